// Streaming decode step of the Tensor Cache layer: one pass over each head's
// ring buffer and memory matrix.
//
// "Tensor Cache: Eviction-conditioned Associative Memory for Transformers",
// §3.2 Fig. 2: (2) evict the pair in slot pos = t mod W, (3) write it into A
// (A <- lambda A + eta k_old v_old^T), (4) store (k_t, v_t) in slot pos,
// (5) read the window by softmax attention and A by m = q A, and fuse
// y = y_local + sigmoid(g) m.
//
// One CTA owns one (b,h) and touches its data exactly once:
//  - A is read, updated and written back in the same pass that forms
//    m = q A' (A' = the updated matrix), with 128-bit loads and stores;
//  - the ring is streamed once with 128-bit non-allocating loads; groups of
//    LPK lanes own one key row each (16 lanes for a 128-wide bf16 row), the
//    scores are reduced with warp shuffles and each group keeps an online
//    softmax (running max, sum and output slice) over its keys;
//  - slot pos is read from the new (k_t, v_t) instead of the ring, and the
//    ring write of slot pos happens after every load of this CTA is done.
// The step is HBM bound: per head it moves W*(d_k+d_v) ring elements and
// 2*d_k*d_v*4 bytes of A.

#include "tc_internal.cuh"

namespace tc {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 8;  // keys per group in flight

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(DecodeParams p) {
    constexpr int VEC = Vec16<T>::N;          // elements per 16-byte load
    constexpr int LPK = D / VEC;              // lanes per key row
    static_assert(LPK >= 1 && LPK <= 32 && (32 % LPK) == 0, "row must map onto a warp");
    constexpr int GPW = 32 / LPK;             // key groups per warp
    constexpr int NG = kWarps * GPW;          // key groups per CTA
    constexpr int CG = D / 4;                 // float4 column groups of A
    constexpr int RG = kThreads / CG;         // row groups of A
    constexpr int RPT = (D + RG - 1) / RG;    // A rows per thread

    __shared__ float s_q[D], s_kn[D], s_vn[D], s_ko[D], s_vo[D];
    __shared__ float s_mp[RG][D];
    __shared__ float s_pd[RG][D];  // delta rule: partial predictions k_old^T A
    __shared__ float s_gm[NG], s_gl[NG];
    __shared__ __align__(16) float s_acc[NG][D];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % p.H);
    const int64_t W = p.W;
    // ragged batches: each batch row has its own clock; a negative clock is an
    // empty row, which this step leaves untouched
    const int64_t t = p.t_rows ? p.t_rows[bh / p.H] : p.t;
    if (t < 0) return;
    const int64_t pos = t % W;
    const bool evict = t >= W;
    const int64_t n = evict ? W : t + 1;  // filled slots after the insert

    const T *q = reinterpret_cast<const T *>(p.q) + bh * D;
    const T *kn = reinterpret_cast<const T *>(p.k) + bh * D;
    const T *vn = reinterpret_cast<const T *>(p.v) + bh * D;
    T *ring_k = reinterpret_cast<T *>(p.ring_k) + bh * W * D;
    T *ring_v = reinterpret_cast<T *>(p.ring_v) + bh * W * D;

    for (int c = tid; c < D; c += kThreads) {
        s_q[c] = to_f32(q[c]);
        s_kn[c] = to_f32(kn[c]);
        s_vn[c] = to_f32(vn[c]);
        s_ko[c] = evict ? to_f32(ring_k[pos * D + c]) : 0.f;
        s_vo[c] = evict ? to_f32(ring_v[pos * D + c]) : 0.f;
    }
    __syncthreads();

    // ---- L2: A' = lambda A + eta k_old v_old^T (if evicting); m = q A' ----
    {
        const float lam = p.lam[h], eta = p.eta[h];
        float4 *A4 = reinterpret_cast<float4 *>(p.A + bh * D * D);
        const int cg = tid % CG, rg = tid / CG;
        float4 a[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = rg + i * RG;
            if (r < D) a[i] = A4[r * CG + cg];
        }
        float4 mp = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 vo = reinterpret_cast<const float4 *>(s_vo)[cg];
        if (p.write_rule == TC_WRITE_DELTA && evict) {
            // delta rule: the written value is v_old - k_old^T A, with A read
            // before this write (uniform branch: rule and clock are per CTA)
            float4 pp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int r = rg + i * RG;
                if (r < D) {
                    const float kr = s_ko[r];
                    pp.x = fmaf(kr, a[i].x, pp.x);
                    pp.y = fmaf(kr, a[i].y, pp.y);
                    pp.z = fmaf(kr, a[i].z, pp.z);
                    pp.w = fmaf(kr, a[i].w, pp.w);
                }
            }
            reinterpret_cast<float4 *>(&s_pd[rg][0])[cg] = pp;
            __syncthreads();
#pragma unroll
            for (int g = 0; g < RG; ++g) {
                const float4 x = reinterpret_cast<const float4 *>(&s_pd[g][0])[cg];
                vo.x -= x.x;
                vo.y -= x.y;
                vo.z -= x.z;
                vo.w -= x.w;
            }
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = rg + i * RG;
            if (r < D) {
                float4 x = a[i];
                if (evict) {
                    const float ek = eta * s_ko[r];
                    x.x = fmaf(lam, x.x, ek * vo.x);
                    x.y = fmaf(lam, x.y, ek * vo.y);
                    x.z = fmaf(lam, x.z, ek * vo.z);
                    x.w = fmaf(lam, x.w, ek * vo.w);
                    A4[r * CG + cg] = x;
                }
                const float qr = s_q[r];
                mp.x = fmaf(qr, x.x, mp.x);
                mp.y = fmaf(qr, x.y, mp.y);
                mp.z = fmaf(qr, x.z, mp.z);
                mp.w = fmaf(qr, x.w, mp.w);
            }
        }
        reinterpret_cast<float4 *>(&s_mp[rg][0])[cg] = mp;
    }

    // ---- L1: softmax attention over the filled ring slots -------------------
    const int gi = warp * GPW + lane / LPK;   // key group
    const int li = lane % LPK;                // slice of the row this lane owns
    const unsigned gmask = (LPK == 32) ? 0xffffffffu : (((1u << LPK) - 1u) << (lane / LPK * LPK));
    float qf[VEC], acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        qf[e] = s_q[li * VEC + e];
        acc[e] = 0.f;
    }
    const float scale = rsqrtf((float)D) * 1.4426950408889634f;  // log2(e)/sqrt(d_k)
    float m_run = -INFINITY, l_run = 0.f;

    for (int64_t base = 0; base < n; base += (int64_t)NG * kUnroll) {
        uint4 kr[kUnroll], vr[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t j = base + (int64_t)u * NG + gi;
            if (j < n) {
                kr[u] = ldg_nc_v4(ring_k + j * D + li * VEC);
                vr[u] = ldg_nc_v4(ring_v + j * D + li * VEC);
            }
        }
        float s[kUnroll];
        float bmax = -INFINITY;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t j = base + (int64_t)u * NG + gi;
            float kf[VEC];
            Vec16<T>::unpack(kr[u], kf);
            if (j == pos) {
#pragma unroll
                for (int e = 0; e < VEC; ++e) kf[e] = s_kn[li * VEC + e];
            }
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) d = fmaf(qf[e], kf[e], d);
#pragma unroll
            for (int off = LPK / 2; off >= 1; off >>= 1) d += __shfl_xor_sync(gmask, d, off);
            s[u] = (j < n) ? d * scale : -INFINITY;
            bmax = fmaxf(bmax, s[u]);
        }
        const float m_new = fmaxf(m_run, bmax);
        if (m_new == -INFINITY) continue;  // this group had no keys in the block
        const float corr = exp2f(m_run - m_new);
        l_run *= corr;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] *= corr;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t j = base + (int64_t)u * NG + gi;
            const float pj = exp2f(s[u] - m_new);
            float vf[VEC];
            Vec16<T>::unpack(vr[u], vf);
            if (j == pos) {
#pragma unroll
                for (int e = 0; e < VEC; ++e) vf[e] = s_vn[li * VEC + e];
            }
            if (j < n) {
                l_run += pj;
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[e] = fmaf(pj, vf[e], acc[e]);
            }
        }
        m_run = m_new;
    }
    if (li == 0) {
        s_gm[gi] = m_run;
        s_gl[gi] = l_run;
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) s_acc[gi][li * VEC + e] = acc[e];
    __syncthreads();

    // ---- combine the groups, fuse with the memory read, store ----------------
    const float gate = sigmoidf_acc(p.g[h]);
    T *y = reinterpret_cast<T *>(p.y) + bh * D;
    for (int c = tid; c < D; c += kThreads) {
        float M = -INFINITY;
        for (int gg = 0; gg < NG; ++gg) M = fmaxf(M, s_gm[gg]);
        float num = 0.f, den = 0.f;
        for (int gg = 0; gg < NG; ++gg) {
            const float w = exp2f(s_gm[gg] - M);
            num = fmaf(w, s_acc[gg][c], num);
            den = fmaf(w, s_gl[gg], den);
        }
        float m = 0.f;
        for (int r = 0; r < RG; ++r) m += s_mp[r][c];
        y[c] = from_f32<T>(num / den + gate * m);
    }
    // every load of slot pos above has completed: now overwrite it (step 4)
    for (int c = tid; c < D; c += kThreads) {
        ring_k[pos * D + c] = kn[c];
        ring_v[pos * D + c] = vn[c];
    }
}

template <typename T>
cudaError_t launch_t(const DecodeParams &p, int64_t BH, cudaStream_t s) {
    const dim3 grid((unsigned)BH), block(kThreads);
    switch (p.dk) {
        case 16: decode_kernel<T, 16><<<grid, block, 0, s>>>(p); break;
        case 32: decode_kernel<T, 32><<<grid, block, 0, s>>>(p); break;
        case 64: decode_kernel<T, 64><<<grid, block, 0, s>>>(p); break;
        case 128: decode_kernel<T, 128><<<grid, block, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

bool decode_supported(int dk, int dv, tc_dtype dtype) {
    (void)dtype;
    return dk == dv && (dk == 16 || dk == 32 || dk == 64 || dk == 128);
}

__global__ void advance_clocks_kernel(int64_t *t_rows, int64_t B) {
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < B;
         b += (int64_t)gridDim.x * blockDim.x)
        if (t_rows[b] >= 0) t_rows[b] += 1;
}

cudaError_t launch_advance_clocks(int64_t *t_rows, int64_t B, cudaStream_t s) {
    const int64_t blocks = (B + 255) / 256;
    advance_clocks_kernel<<<(unsigned)(blocks < 1024 ? blocks : 1024), 256, 0, s>>>(t_rows, B);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams &p, tc_dtype dtype, int64_t BH, cudaStream_t s) {
    if (BH == 0) return cudaSuccess;
    return dtype == TC_BF16 ? launch_t<__nv_bfloat16>(p, BH, s) : launch_t<float>(p, BH, s);
}

}  // namespace tc
