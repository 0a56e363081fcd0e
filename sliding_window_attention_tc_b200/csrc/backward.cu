// Backward of the Tensor Cache layer (outer-product write).
//
// "Tensor Cache: Eviction-conditioned Associative Memory for Transformers":
// the pages train lambda, eta and g end to end through the chunk scan (§2
// training considerations).  For L = sum_t <dy_t, y_t> with
//   y_t = y_local_t + s m_t,  s = sigmoid(g),  m_t = q_t A_t,
//   A_t = lam A_{t-1} + eta k_{t-W} v_{t-W}^T (t >= W), A_t = A_{t-1} otherwise,
// the gradients split into two parts.
//
// Window (L1), the softmax backward over the keys t-W+1 .. t:
//   p = softmax(q k / sqrt(dk)), dp_j = <dy_t, v_j>, D_t = <dy_t, y_local_t>,
//   ds_j = p_j (dp_j - D_t); dq_t += sum_j ds_j k_j / sqrt(dk),
//   dk_j += ds_j q_t / sqrt(dk), dv_j += p_j dy_t.
//   For bf16 with d_k = d_v = 64 two tensor-core kernels do this
//   (backward_sm100.cu); otherwise, in float32 SIMT, bwd_rows_kernel (a warp
//   per 4 query rows) writes dq and the per-row log-sum-exp and D_t, and
//   bwd_keys_kernel (a warp per 4 key rows, over the W queries that see
//   them) writes dk and dv.
//
// Memory (L2), a reverse scan of G_t = dL/dA_t:
//   G_t = q_t^T (s dy_t) + [step t+1 writes] lam G_{t+1}, and each write at
//   step t (eviction e = t - W) gives dk_e += eta G_t v_e,
//   dv_e += eta G_t^T k_e, deta += <G_t, k_e v_e^T>, dlam += <G_t, A_{t-1}>;
//   also dq_t += A_t (s dy_t) and dg += s (1 - s) <dy_t, q_t A_t>.
//   Chunked over the evictions (the transpose of the forward chunk scan):
//   l2b_sums_kernel computes per chunk the state increment and the chunk's
//   summary of q^T (s dy); l2b_scan_kernel scans both over the chunks, one
//   thread per state element, giving each chunk's start state A_c and the
//   G that the later chunks pass back (H_c); l2b_chunk_kernel then forms the
//   chunk's gradients from C x C products in shared memory; the
//   bwd_reduce_kernel sums the lambda, eta, g partials over the batch and
//   the chunks in a fixed order.  No atomics: the gradients are the same bit
//   for bit on every run.

#include <cuda_runtime.h>

#include <cstdint>

#include "tc.h"
#include "tc_internal.cuh"

namespace tc {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxD = 128;
constexpr int kKT = 32;               // key / query tile of the L1 kernels
constexpr float kLog2e = 1.4426950408889634f;

// Evictions per chunk of the memory backward.  The tensor-core chunk kernel
// (bf16, d = 64) takes 128, one MMA tile of rows.  The SIMT one takes 32,
// which keeps it at about 75 KB of shared memory for d = 64 (three CTAs per
// SM) and its triangular in-chunk work small.
int l2b_chunk(const tc_prefill_desc &d) { return backward_memory_tc_supported(d) ? 128 : 32; }

struct BwdParams {
    const void *q, *k, *v, *dy;
    const float *lam, *eta, *g;
    float *gq, *gk, *gv;    // gradients of q, k, v (float32, layout of the inputs)
    float *lse, *Dt;        // [BH][T] per query row (log2 domain), <dy, y_local>
    int64_t stat_stride;    // row stride of lse, Dt (T, or the tensor-core path's Tp)
    float *Ac, *Hc;         // [BH][nC][dk*dv]: increments, then chunk start states A_c;
                            // summaries, then the G passed back from later chunks H_c
    float *part;            // [BH][nC][3]: dlam, deta, dg partials
    float *dlam, *deta, *dg;
    int64_t B, H, T, W;
    int dk, dv;
    int C;                  // evictions per chunk of the memory part
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---------------------------------------------------------------------------
// Register tiling of the window kernels.  A warp owns kQR query rows (or key
// rows): every key (or query) value read from shared memory serves kQR
// FMAs, and the dot products read 16 bytes at a time.  Shared rows are
// padded to a 16-byte stride whose quads fall in distinct banks for 8
// consecutive lanes; the padding columns are zero, so dots over them add 0.
constexpr int kQR = 4;                        // rows per warp
constexpr int kTileR = (kThreads / 32) * kQR;  // rows per CTA

__host__ __device__ __forceinline__ int pad_stride(int d) {
    int s = (d + 3) & ~3;
    if (((s >> 2) & 1) == 0) s += 4;  // odd number of quads: conflict-free float4 rows
    return s;
}

// n rows of width d from global (row stride d) into shared rows of stride sp,
// zero past n rows of src_rows and in the padding columns.
template <typename Tin>
__device__ __forceinline__ void load_rows(float *dst, int sp, const Tin *src, int64_t row0,
                                          int64_t n_valid, int n_rows, int d, int tid) {
    const int lane = tid & 31;
    for (int rr = tid >> 5; rr < n_rows; rr += kThreads / 32) {
        const bool ok = rr < n_valid;
        const Tin *s = src + (row0 + rr) * d;
        for (int c = lane; c < sp; c += 32) dst[rr * sp + c] = (ok && c < d) ? to_f32(s[c]) : 0.f;
    }
}

// Four dot products of one lane's row `a` (stride-1, padded to quads) with four
// broadcast rows b[i] (same padding), over dp4 columns.
__device__ __forceinline__ void dot4(const float *a, const float *b, int sb, int dp4, float (&out)[kQR]) {
#pragma unroll
    for (int i = 0; i < kQR; ++i) out[i] = 0.f;
    for (int r = 0; r < dp4; r += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(a + r);
#pragma unroll
        for (int i = 0; i < kQR; ++i) {
            const float4 y = *reinterpret_cast<const float4 *>(b + i * sb + r);
            out[i] = fmaf(x.x, y.x, out[i]);
            out[i] = fmaf(x.y, y.y, out[i]);
            out[i] = fmaf(x.z, y.z, out[i]);
            out[i] = fmaf(x.w, y.w, out[i]);
        }
    }
}

// dq (window part), log-sum-exp and D_t; a warp owns kQR query rows, a lane
// one key of the current 32-key tile (scores) or output columns lane, lane+32,
// ... (products with V and K).
template <typename Tin, int CPL>  // CPL: output columns per lane, >= d / 32
__global__ void __launch_bounds__(kThreads) bwd_rows_kernel(BwdParams p) {
    extern __shared__ __align__(16) float shr[];
    const int dk = p.dk, dv = p.dv;
    const int skp = pad_stride(dk), svp = pad_stride(dv);
    const int dk4 = (dk + 3) & ~3, dv4 = (dv + 3) & ~3;
    float *sk = shr;                      // [kKT][skp]
    float *sv = sk + kKT * skp;           // [kKT][svp]
    float *sq = sv + kKT * svp;           // [kTileR][skp]
    float *sdy = sq + kTileR * skp;       // [kTileR][svp]
    float *spt = sdy + kTileR * svp;      // [warps][kKT][kQR]: P or dS of the warp's rows
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int64_t T = p.T, W = p.W;
    const int64_t t0 = (int64_t)blockIdx.x * kTileR;  // first row of the CTA
    const int64_t tw = t0 + warp * kQR;               // first row of the warp
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T * dk;
    const Tin *kb = reinterpret_cast<const Tin *>(p.k) + bh * T * dk;
    const Tin *vb = reinterpret_cast<const Tin *>(p.v) + bh * T * dv;
    const Tin *db = reinterpret_cast<const Tin *>(p.dy) + bh * T * dv;
    const int64_t n_here = T - t0 < kTileR ? T - t0 : kTileR;
    load_rows(sq, skp, qb, t0, n_here, kTileR, dk, tid);
    load_rows(sdy, svp, db, t0, n_here, kTileR, dv, tid);
    float *my_p = spt + warp * kKT * kQR;
    const float scale2 = kLog2e / sqrtf((float)dk);
    const int64_t t_last = (t0 + kTileR - 1 < T - 1) ? t0 + kTileR - 1 : T - 1;
    const int64_t lo = t0 - W + 1 > 0 ? t0 - W + 1 : 0;
    const float *q_w = sq + warp * kQR * skp, *dy_w = sdy + warp * kQR * svp;

    // pass 1: softmax statistics and y_local (online), per row
    float m_run[kQR], l_run[kQR], acc[kQR][CPL];
#pragma unroll
    for (int i = 0; i < kQR; ++i) {
        m_run[i] = -INFINITY;
        l_run[i] = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[i][c] = 0.f;
    }
    for (int64_t j0 = lo; j0 <= t_last; j0 += kKT) {
        const int nt = (int)((t_last - j0 + 1 < kKT) ? t_last - j0 + 1 : kKT);
        __syncthreads();
        load_rows(sk, skp, kb, j0, nt, kKT, dk, tid);
        load_rows(sv, svp, vb, j0, nt, kKT, dv, tid);
        __syncthreads();
        const int64_t j = j0 + lane;
        float dot[kQR];
        dot4(sk + lane * skp, q_w, skp, dk4, dot);
        float pr[kQR];
#pragma unroll
        for (int i = 0; i < kQR; ++i) {
            const int64_t t = tw + i;
            const bool in_win = t < T && lane < nt && j > t - W && j <= t;
            const float s = in_win ? dot[i] * scale2 : -INFINITY;
            const float m_new = fmaxf(m_run[i], warp_max(s));
            if (m_new == -INFINITY) {  // no key of this tile in the row's window yet
                pr[i] = 0.f;
                continue;
            }
            const float corr = exp2f(m_run[i] - m_new);
            pr[i] = exp2f(s - m_new);
            l_run[i] = l_run[i] * corr + warp_sum(pr[i]);
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[i][c] *= corr;
            m_run[i] = m_new;
        }
        *reinterpret_cast<float4 *>(my_p + lane * kQR) = make_float4(pr[0], pr[1], pr[2], pr[3]);
        __syncwarp();
        for (int jj = 0; jj < nt; ++jj) {
            const float4 pb = *reinterpret_cast<const float4 *>(my_p + jj * kQR);
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int col = lane + 32 * c;
                if (col < dv) {
                    const float vv = sv[jj * svp + col];
                    acc[0][c] = fmaf(pb.x, vv, acc[0][c]);
                    acc[1][c] = fmaf(pb.y, vv, acc[1][c]);
                    acc[2][c] = fmaf(pb.z, vv, acc[2][c]);
                    acc[3][c] = fmaf(pb.w, vv, acc[3][c]);
                }
            }
        }
        __syncwarp();
    }
    float lse2[kQR], Dt[kQR];
#pragma unroll
    for (int i = 0; i < kQR; ++i) {
        const int64_t t = tw + i;
        lse2[i] = m_run[i] + log2f(l_run[i]);
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int col = lane + 32 * c;
            if (col < dv) d = fmaf(dy_w[i * svp + col], acc[i][c] / l_run[i], d);
        }
        Dt[i] = warp_sum(d);
        if (t < T && lane == 0) {
            p.lse[bh * p.stat_stride + t] = lse2[i];
            p.Dt[bh * p.stat_stride + t] = Dt[i];
        }
    }
    // pass 2: ds_j = p_j (dp_j - D_t); dq_t = sum_j ds_j k_j / sqrt(dk)
    float dqa[kQR][CPL];
#pragma unroll
    for (int i = 0; i < kQR; ++i)
#pragma unroll
        for (int c = 0; c < CPL; ++c) dqa[i][c] = 0.f;
    const float inv_sqrt = 1.f / sqrtf((float)dk);
    for (int64_t j0 = lo; j0 <= t_last; j0 += kKT) {
        const int nt = (int)((t_last - j0 + 1 < kKT) ? t_last - j0 + 1 : kKT);
        __syncthreads();
        load_rows(sk, skp, kb, j0, nt, kKT, dk, tid);
        load_rows(sv, svp, vb, j0, nt, kKT, dv, tid);
        __syncthreads();
        const int64_t j = j0 + lane;
        float dot[kQR], dp[kQR], ds[kQR];
        dot4(sk + lane * skp, q_w, skp, dk4, dot);
        dot4(sv + lane * svp, dy_w, svp, dv4, dp);
#pragma unroll
        for (int i = 0; i < kQR; ++i) {
            const int64_t t = tw + i;
            const bool in_win = t < T && lane < nt && j > t - W && j <= t;
            ds[i] = in_win ? exp2f(dot[i] * scale2 - lse2[i]) * (dp[i] - Dt[i]) : 0.f;
        }
        *reinterpret_cast<float4 *>(my_p + lane * kQR) = make_float4(ds[0], ds[1], ds[2], ds[3]);
        __syncwarp();
        for (int jj = 0; jj < nt; ++jj) {
            const float4 db4 = *reinterpret_cast<const float4 *>(my_p + jj * kQR);
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int r = lane + 32 * c;
                if (r < dk) {
                    const float kk = sk[jj * skp + r];
                    dqa[0][c] = fmaf(db4.x, kk, dqa[0][c]);
                    dqa[1][c] = fmaf(db4.y, kk, dqa[1][c]);
                    dqa[2][c] = fmaf(db4.z, kk, dqa[2][c]);
                    dqa[3][c] = fmaf(db4.w, kk, dqa[3][c]);
                }
            }
        }
        __syncwarp();
    }
#pragma unroll
    for (int i = 0; i < kQR; ++i) {
        const int64_t t = tw + i;
        if (t >= T) continue;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int r = lane + 32 * c;
            if (r < dk) p.gq[(bh * T + t) * dk + r] = dqa[i][c] * inv_sqrt;
        }
    }
}

// ---------------------------------------------------------------------------
// dk, dv (window part); a warp owns kQR key rows j over the queries
// t = j .. j+W-1, a lane one query of the current 32-query tile (scores) or
// output columns lane, lane+32, ... (products with Q and dY).
template <typename Tin, int CPL>  // CPL: output columns per lane, >= d / 32
__global__ void __launch_bounds__(kThreads) bwd_keys_kernel(BwdParams p) {
    extern __shared__ __align__(16) float shr[];
    const int dk = p.dk, dv = p.dv;
    const int skp = pad_stride(dk), svp = pad_stride(dv);
    const int dk4 = (dk + 3) & ~3, dv4 = (dv + 3) & ~3;
    float *sq = shr;                      // [kKT][skp]   queries of the tile
    float *sdy = sq + kKT * skp;          // [kKT][svp]
    float *sk = sdy + kKT * svp;          // [kTileR][skp] keys of the CTA
    float *sv = sk + kTileR * skp;        // [kTileR][svp]
    float *spt = sv + kTileR * svp;       // [warps][kKT][2 kQR]: P and dS of the warp's keys
    float *slse = spt + (kThreads / 32) * kKT * 2 * kQR;  // [kKT]
    float *sD = slse + kKT;                               // [kKT]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int64_t T = p.T, W = p.W;
    const int64_t j0k = (int64_t)blockIdx.x * kTileR;  // first key of the CTA
    const int64_t jw = j0k + warp * kQR;               // first key of the warp
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T * dk;
    const Tin *kb = reinterpret_cast<const Tin *>(p.k) + bh * T * dk;
    const Tin *vb = reinterpret_cast<const Tin *>(p.v) + bh * T * dv;
    const Tin *db = reinterpret_cast<const Tin *>(p.dy) + bh * T * dv;
    const int64_t n_here = T - j0k < kTileR ? T - j0k : kTileR;
    load_rows(sk, skp, kb, j0k, n_here, kTileR, dk, tid);
    load_rows(sv, svp, vb, j0k, n_here, kTileR, dv, tid);
    float *my_p = spt + warp * kKT * 2 * kQR;
    const float scale2 = kLog2e / sqrtf((float)dk);
    const float inv_sqrt = 1.f / sqrtf((float)dk);
    // queries that see any key of this CTA: j0k .. j0k + kTileR - 1 + W - 1
    const int64_t q_hi_all = j0k + kTileR - 1 + W - 1 < T - 1 ? j0k + kTileR - 1 + W - 1 : T - 1;
    const float *k_w = sk + warp * kQR * skp, *v_w = sv + warp * kQR * svp;
    float dka[kQR][CPL], dva[kQR][CPL];
#pragma unroll
    for (int i = 0; i < kQR; ++i)
#pragma unroll
        for (int c = 0; c < CPL; ++c) dka[i][c] = dva[i][c] = 0.f;
    for (int64_t q0 = j0k; q0 <= q_hi_all; q0 += kKT) {
        const int nt = (int)((q_hi_all - q0 + 1 < kKT) ? q_hi_all - q0 + 1 : kKT);
        __syncthreads();
        load_rows(sq, skp, qb, q0, nt, kKT, dk, tid);
        load_rows(sdy, svp, db, q0, nt, kKT, dv, tid);
        if (tid < nt) {
            slse[tid] = p.lse[bh * p.stat_stride + q0 + tid];
            sD[tid] = p.Dt[bh * p.stat_stride + q0 + tid];
        }
        __syncthreads();
        const int64_t t = q0 + lane;
        float dot[kQR], dp[kQR], pj[kQR], ds[kQR];
        dot4(sq + lane * skp, k_w, skp, dk4, dot);
        dot4(sdy + lane * svp, v_w, svp, dv4, dp);
        const float lse_t = lane < nt ? slse[lane] : 0.f, D_t = lane < nt ? sD[lane] : 0.f;
#pragma unroll
        for (int i = 0; i < kQR; ++i) {
            const int64_t j = jw + i;
            const bool sees = j < T && lane < nt && t >= j && t < j + W;
            pj[i] = sees ? exp2f(dot[i] * scale2 - lse_t) : 0.f;
            ds[i] = pj[i] * (dp[i] - D_t);
        }
        *reinterpret_cast<float4 *>(my_p + lane * 2 * kQR) = make_float4(pj[0], pj[1], pj[2], pj[3]);
        *reinterpret_cast<float4 *>(my_p + lane * 2 * kQR + kQR) = make_float4(ds[0], ds[1], ds[2], ds[3]);
        __syncwarp();
        for (int tt = 0; tt < nt; ++tt) {
            const float4 pb = *reinterpret_cast<const float4 *>(my_p + tt * 2 * kQR);
            const float4 dsb = *reinterpret_cast<const float4 *>(my_p + tt * 2 * kQR + kQR);
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int r = lane + 32 * c;
                if (r < dk) {
                    const float qq = sq[tt * skp + r];
                    dka[0][c] = fmaf(dsb.x, qq, dka[0][c]);
                    dka[1][c] = fmaf(dsb.y, qq, dka[1][c]);
                    dka[2][c] = fmaf(dsb.z, qq, dka[2][c]);
                    dka[3][c] = fmaf(dsb.w, qq, dka[3][c]);
                }
                if (r < dv) {
                    const float yy = sdy[tt * svp + r];
                    dva[0][c] = fmaf(pb.x, yy, dva[0][c]);
                    dva[1][c] = fmaf(pb.y, yy, dva[1][c]);
                    dva[2][c] = fmaf(pb.z, yy, dva[2][c]);
                    dva[3][c] = fmaf(pb.w, yy, dva[3][c]);
                }
            }
        }
        __syncwarp();
    }
#pragma unroll
    for (int i = 0; i < kQR; ++i) {
        const int64_t j = jw + i;
        if (j >= T) continue;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int r = lane + 32 * c;
            if (r < dk) p.gk[(bh * T + j) * dk + r] = dka[i][c] * inv_sqrt;
            if (r < dv) p.gv[(bh * T + j) * dv + r] = dva[i][c];
        }
    }
}

// Dynamic shared memory of the two window kernels.
__host__ __forceinline__ size_t rows_smem(int dk, int dv) {
    return (size_t)((kKT + kTileR) * (pad_stride(dk) + pad_stride(dv)) + (kThreads / 32) * kKT * kQR) *
           sizeof(float);
}
__host__ __forceinline__ size_t keys_smem(int dk, int dv) {
    return (size_t)((kKT + kTileR) * (pad_stride(dk) + pad_stride(dv)) +
                    (kThreads / 32) * kKT * 2 * kQR + 2 * kKT) *
           sizeof(float);
}

// ---------------------------------------------------------------------------
// Memory part, chunked.  Chunk c of row bh holds evictions e = cC .. cC+L-1
// (L <= C); index i, j, s within it.  Reads at t = e + W: qt_s = q_t,
// dt_s = s dy_t.  pw(n) = lam^n.

// lam^n for n = 0 .. n_max into shared memory (lam^0 = 1 also for lam = 0).
__device__ __forceinline__ void lam_powers(float *pw, int n_max, float lam) {
    const double l2l = log2((double)lam);
    for (int n = threadIdx.x; n <= n_max; n += blockDim.x)
        pw[n] = n == 0 ? 1.f : (float)exp2((double)n * l2l);
}

// Rows r0 .. r0+n-1 (of width d, row stride d in global) into shared rows of
// stride sp; a row index past `valid` reads as zeros.
template <typename Tin>
__device__ __forceinline__ void stage_rows(float *dst, int sp, const Tin *src, int64_t r0, int n,
                                           int valid, int d, float scale) {
    for (int x = threadIdx.x; x < n * d; x += blockDim.x) {
        const int rr = x / d, c = x % d;
        dst[rr * sp + c] = rr < valid ? scale * to_f32(src[(r0 + rr) * d + c]) : 0.f;
    }
}

// Per chunk: the state increment dA_c = sum_i eta lam^(L-1-i) k_i v_i^T (into
// Ac) and the summary X_c = sum_s lam^s qt_s^T dt_s (into Hc).
template <typename Tin>
__global__ void __launch_bounds__(kThreads) l2b_sums_kernel(BwdParams p) {
    extern __shared__ float sh[];
    const int dk = p.dk, dv = p.dv, C = p.C;
    const int64_t bh = blockIdx.y, T = p.T, W = p.W, E = T - W;
    const int c = blockIdx.x, h = (int)(bh % p.H);
    const int64_t e0 = (int64_t)c * C;
    const int L = (int)(E - e0 < C ? E - e0 : C);
    const int nC = (int)((E + C - 1) / C);
    const float lam = p.lam[h], eta = p.eta[h];
    const float sg = 1.f / (1.f + expf(-p.g[h]));
    float *sK = sh, *sV = sK + C * dk, *sQ = sV + C * dv, *sD = sQ + C * dk, *pw = sD + C * dv;
    const Tin *kb = reinterpret_cast<const Tin *>(p.k) + bh * T * dk;
    const Tin *vb = reinterpret_cast<const Tin *>(p.v) + bh * T * dv;
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T * dk;
    const Tin *db = reinterpret_cast<const Tin *>(p.dy) + bh * T * dv;
    stage_rows(sK, dk, kb, e0, C, L, dk, 1.f);
    stage_rows(sV, dv, vb, e0, C, L, dv, 1.f);
    stage_rows(sQ, dk, qb, e0 + W, C, L, dk, 1.f);
    stage_rows(sD, dv, db, e0 + W, C, L, dv, sg);
    lam_powers(pw, C, lam);
    __syncthreads();
    float *outA = p.Ac + ((size_t)bh * nC + c) * dk * dv;
    float *outX = p.Hc + ((size_t)bh * nC + c) * dk * dv;
    const int tm = (dk + 3) / 4, tn = (dv + 3) / 4;
    for (int t = threadIdx.x; t < tm * tn; t += blockDim.x) {
        const int r0 = 4 * (t / tn), c0 = 4 * (t % tn);
        float acc[4][4];
        tile44(L, r0, c0, [&](int r, int i) { return r < dk ? pw[L - 1 - i] * sK[i * dk + r] : 0.f; },
               [&](int i, int cc) { return cc < dv ? sV[i * dv + cc] : 0.f; }, acc);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (r0 + u < dk && c0 + w < dv) outA[(r0 + u) * dv + c0 + w] = eta * acc[u][w];
        tile44(L, r0, c0, [&](int r, int i) { return r < dk ? pw[i] * sQ[i * dk + r] : 0.f; },
               [&](int i, int cc) { return cc < dv ? sD[i * dv + cc] : 0.f; }, acc);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (r0 + u < dk && c0 + w < dv) outX[(r0 + u) * dv + c0 + w] = acc[u][w];
    }
}

// Per (row, state element), over the chunks: A_c = state before chunk c's
// writes (forward), H_c = G at the start of chunk c+1 (backward), in place.
// Values are read kScanBatch chunks ahead of their use, so each thread keeps
// several loads in flight instead of one.
constexpr int kScanBatch = 8;
__global__ void __launch_bounds__(kThreads) l2b_scan_kernel(BwdParams p) {
    __shared__ float decay[2];  // lam^C, lam^(length of the last chunk)
    const int dk = p.dk, dv = p.dv, C = p.C;
    const int64_t bh = blockIdx.y, E = p.T - p.W;
    const int nC = (int)((E + C - 1) / C);
    if (threadIdx.x < 2) {
        const double l2l = log2((double)p.lam[bh % p.H]);
        const int n = threadIdx.x == 0 ? C : (int)(E - (int64_t)(nC - 1) * C);
        decay[threadIdx.x] = (float)exp2((double)n * l2l);
    }
    __syncthreads();
    const int x = blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= dk * dv) return;
    const float pC = decay[0], pLast = decay[1];
    const size_t stride = (size_t)dk * dv;
    float *__restrict__ Ac = p.Ac + (size_t)bh * nC * stride + x;
    float *__restrict__ Hc = p.Hc + (size_t)bh * nC * stride + x;
    float A = 0.f;
    for (int c0 = 0; c0 < nC; c0 += kScanBatch) {
        float d[kScanBatch];
#pragma unroll
        for (int u = 0; u < kScanBatch; ++u) d[u] = c0 + u < nC ? Ac[(size_t)(c0 + u) * stride] : 0.f;
#pragma unroll
        for (int u = 0; u < kScanBatch; ++u) {
            const int c = c0 + u;
            if (c < nC) {
                Ac[(size_t)c * stride] = A;
                A = fmaf(c == nC - 1 ? pLast : pC, A, d[u]);
            }
        }
    }
    float H = 0.f;
    for (int c0 = nC - 1; c0 >= 0; c0 -= kScanBatch) {
        float xs[kScanBatch];
#pragma unroll
        for (int u = 0; u < kScanBatch; ++u) xs[u] = c0 - u >= 0 ? Hc[(size_t)(c0 - u) * stride] : 0.f;
#pragma unroll
        for (int u = 0; u < kScanBatch; ++u) {
            const int c = c0 - u;
            if (c >= 0) {
                Hc[(size_t)c * stride] = H;
                H = fmaf(c == nC - 1 ? pLast : pC, H, xs[u]);
            }
        }
    }
}

// Per chunk, with A = A_c and H = H_c (rows of K, V, qt, dt staged):
//   dk_i = eta [pw(L-i) H v_i + sum_{s>=i} pw(s-i) (dt_s.v_i) qt_s]
//   dv_i = eta [pw(L-i) H^T k_i + sum_{s>=i} pw(s-i) (qt_s.k_i) dt_s]
//   dq_s = pw(s+1) A dt_s + eta sum_{j<=s} pw(s-j) (dt_s.v_j) k_j
//   m_s  = pw(s+1) qt_s A + eta sum_{j<=s} pw(s-j) (qt_s.k_j) v_j
//   deta += sum_i <k_i, dk_i> / eta,  dg += (1 - sig) sum_s <dt_s, m_s>,
//   dlam += L pw(L) <H, A> + sum_s (s+1) pw(s) <qt_s A, dt_s>
//         + eta sum_j (L-1-j) pw(L-1-j) <k_j, H v_j>
//         + eta sum_{j<s} (s-j) pw(s-1-j) (qt_s.k_j) (dt_s.v_j)
// (sum over the chunk's steps e of <G_e, A_{e-1}>, with G_e and A_{e-1}
// written out in the chunk's terms).  The increments of dq, dk, dv are added
// to the window part's results; each row belongs to one chunk.
template <typename Tin>
__global__ void __launch_bounds__(kThreads) l2b_chunk_kernel(BwdParams p) {
    extern __shared__ float sh[];
    const int dk = p.dk, dv = p.dv, C = p.C;
    const int sk = dk + 1, sv = dv + 1, sc = C + 1;  // padded strides
    const int64_t bh = blockIdx.y, T = p.T, W = p.W, E = T - W;
    const int c = blockIdx.x, h = (int)(bh % p.H);
    const int64_t e0 = (int64_t)c * C;
    const int L = (int)(E - e0 < C ? E - e0 : C);
    const int nC = (int)((E + C - 1) / C);
    const float eta = p.eta[h];
    const float sg = 1.f / (1.f + expf(-p.g[h]));
    float *sK = sh, *sV = sK + C * sk, *sQ = sV + C * sv, *sD = sQ + C * sk;
    float *sA = sD + C * sv, *sH = sA + dk * sv, *sQK = sH + dk * sv, *sDV = sQK + C * sc;
    float *pw = sDV + C * sc, *sred = pw + C + 2;
    const Tin *kb = reinterpret_cast<const Tin *>(p.k) + bh * T * dk;
    const Tin *vb = reinterpret_cast<const Tin *>(p.v) + bh * T * dv;
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T * dk;
    const Tin *db = reinterpret_cast<const Tin *>(p.dy) + bh * T * dv;
    stage_rows(sK, sk, kb, e0, C, L, dk, 1.f);
    stage_rows(sV, sv, vb, e0, C, L, dv, 1.f);
    stage_rows(sQ, sk, qb, e0 + W, C, L, dk, 1.f);
    stage_rows(sD, sv, db, e0 + W, C, L, dv, sg);
    const float *gA = p.Ac + ((size_t)bh * nC + c) * dk * dv;
    const float *gH = p.Hc + ((size_t)bh * nC + c) * dk * dv;
    for (int x = threadIdx.x; x < dk * dv; x += blockDim.x) {
        sA[(x / dv) * sv + x % dv] = gA[x];
        sH[(x / dv) * sv + x % dv] = gH[x];
    }
    lam_powers(pw, C + 1, p.lam[h]);
    __syncthreads();
    // QK[s][j] = qt_s . k_j, DV[s][j] = dt_s . v_j
    const int tc_ = (C + 3) / 4;
    for (int t = threadIdx.x; t < tc_ * tc_; t += blockDim.x) {
        const int s0 = 4 * (t / tc_), j0 = 4 * (t % tc_);
        float acc[4][4];
        tile44(dk, s0, j0, [&](int s, int r) { return sQ[s * sk + r]; },
               [&](int r, int j) { return sK[j * sk + r]; }, acc);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) sQK[(s0 + u) * sc + j0 + w] = acc[u][w];
        tile44(dv, s0, j0, [&](int s, int cc) { return sD[s * sv + cc]; },
               [&](int cc, int j) { return sV[j * sv + cc]; }, acc);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) sDV[(s0 + u) * sc + j0 + w] = acc[u][w];
    }
    __syncthreads();
    float p_lam = 0.f, p_eta = 0.f, p_g = 0.f;  // this thread's partials
    float *gq = p.gq + (bh * T + e0 + W) * dk, *gk = p.gk + (bh * T + e0) * dk;
    float *gv = p.gv + (bh * T + e0) * dv;
    const int tL = (L + 3) / 4, tk = (dk + 3) / 4, tv = (dv + 3) / 4;
    // dk and the <k, H v> terms: rows i, columns r
    for (int t = threadIdx.x; t < tL * tk; t += blockDim.x) {
        const int i0 = 4 * (t / tk), r0 = 4 * (t % tk);
        float hv[4][4], in[4][4];
        tile44(dv, i0, r0, [&](int i, int cc) { return sV[i * sv + cc]; },
               [&](int cc, int r) { return r < dk ? sH[r * sv + cc] : 0.f; }, hv);
        tile44(L, i0, r0, [&](int i, int s) { return s >= i ? pw[s - i] * sDV[s * sc + i] : 0.f; },
               [&](int s, int r) { return r < dk ? sQ[s * sk + r] : 0.f; }, in);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            if (i >= L) continue;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int r = r0 + w;
                if (r >= dk) continue;
                const float dkr = pw[L - i] * hv[u][w] + in[u][w];  // dk_i[r] / eta
                gk[(size_t)i * dk + r] += eta * dkr;
                p_eta = fmaf(sK[i * sk + r], dkr, p_eta);
                p_lam = fmaf(eta * (float)(L - 1 - i) * pw[L - 1 - i] * sK[i * sk + r], hv[u][w], p_lam);
            }
        }
    }
    // dv: rows i, columns cc
    for (int t = threadIdx.x; t < tL * tv; t += blockDim.x) {
        const int i0 = 4 * (t / tv), c0 = 4 * (t % tv);
        float hk[4][4], in[4][4];
        tile44(dk, i0, c0, [&](int i, int r) { return sK[i * sk + r]; },
               [&](int r, int cc) { return cc < dv ? sH[r * sv + cc] : 0.f; }, hk);
        tile44(L, i0, c0, [&](int i, int s) { return s >= i ? pw[s - i] * sQK[s * sc + i] : 0.f; },
               [&](int s, int cc) { return cc < dv ? sD[s * sv + cc] : 0.f; }, in);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            if (i >= L) continue;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (c0 + w < dv) gv[(size_t)i * dv + c0 + w] += eta * (pw[L - i] * hk[u][w] + in[u][w]);
        }
    }
    // dq: rows s, columns r
    for (int t = threadIdx.x; t < tL * tk; t += blockDim.x) {
        const int s0 = 4 * (t / tk), r0 = 4 * (t % tk);
        float ad[4][4], in[4][4];
        tile44(dv, s0, r0, [&](int s, int cc) { return sD[s * sv + cc]; },
               [&](int cc, int r) { return r < dk ? sA[r * sv + cc] : 0.f; }, ad);
        tile44(L, s0, r0, [&](int s, int j) { return j <= s ? pw[s - j] * sDV[s * sc + j] : 0.f; },
               [&](int j, int r) { return r < dk ? sK[j * sk + r] : 0.f; }, in);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            if (s >= L) continue;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (r0 + w < dk) gq[(size_t)s * dk + r0 + w] += pw[s + 1] * ad[u][w] + eta * in[u][w];
        }
    }
    // m (for dg) and the <qt A, dt> terms: rows s, columns cc
    for (int t = threadIdx.x; t < tL * tv; t += blockDim.x) {
        const int s0 = 4 * (t / tv), c0 = 4 * (t % tv);
        float qa[4][4], in[4][4];
        tile44(dk, s0, c0, [&](int s, int r) { return sQ[s * sk + r]; },
               [&](int r, int cc) { return cc < dv ? sA[r * sv + cc] : 0.f; }, qa);
        tile44(L, s0, c0, [&](int s, int j) { return j <= s ? pw[s - j] * sQK[s * sc + j] : 0.f; },
               [&](int j, int cc) { return cc < dv ? sV[j * sv + cc] : 0.f; }, in);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            if (s >= L) continue;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int cc = c0 + w;
                if (cc >= dv) continue;
                const float m = pw[s + 1] * qa[u][w] + eta * in[u][w];
                p_g = fmaf(sD[s * sv + cc], m, p_g);
                p_lam = fmaf((float)(s + 1) * pw[s] * qa[u][w], sD[s * sv + cc], p_lam);
            }
        }
    }
    // the pair terms and <H, A>
    for (int x = threadIdx.x; x < L * L; x += blockDim.x) {
        const int s = x / L, j = x % L;
        if (j < s)
            p_lam = fmaf(eta * (float)(s - j) * pw[s - 1 - j] * sQK[s * sc + j], sDV[s * sc + j], p_lam);
    }
    for (int x = threadIdx.x; x < dk * dv; x += blockDim.x)
        p_lam = fmaf((float)L * pw[L] * sH[(x / dv) * sv + x % dv], sA[(x / dv) * sv + x % dv], p_lam);
    p_g *= 1.f - sg;
    // fixed-order block sum of the three partials
    p_lam = warp_sum(p_lam);
    p_eta = warp_sum(p_eta);
    p_g = warp_sum(p_g);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        sred[warp * 3] = p_lam;
        sred[warp * 3 + 1] = p_eta;
        sred[warp * 3 + 2] = p_g;
    }
    __syncthreads();
    if (threadIdx.x < 3) {
        float a = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) a += sred[w * 3 + threadIdx.x];
        p.part[((size_t)bh * nC + c) * 3 + threadIdx.x] = a;
    }
}

__host__ __forceinline__ size_t l2b_chunk_smem(int dk, int dv, int C) {
    return (size_t)(C * (dk + 1) * 2 + C * (dv + 1) * 2 + 2 * dk * (dv + 1) + 2 * C * (C + 1) + C + 2 +
                    3 * (kThreads / 32)) * sizeof(float);
}
__host__ __forceinline__ size_t l2b_sums_smem(int dk, int dv, int C) {
    return (size_t)(2 * C * dk + 2 * C * dv + C + 1) * sizeof(float);
}

// dlam, deta, dg per head: the (b, h, chunk) partials summed over the batch
// and the chunks in a fixed order (zero when nothing is evicted).
__global__ void bwd_reduce_kernel(BwdParams p, int nC) {
    const int64_t h = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= p.H) return;
    float a = 0.f, b_ = 0.f, c = 0.f;
    for (int64_t b = 0; b < p.B; ++b)
        for (int x = 0; x < nC; ++x) {
            const float *pp = p.part + ((b * p.H + h) * nC + x) * 3;
            a += pp[0];
            b_ += pp[1];
            c += pp[2];
        }
    p.dlam[h] = a;
    p.deta[h] = b_;
    p.dg[h] = c;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Chunks of the memory backward: ceil(E / C) over the E = T - W evictions.
int64_t l2b_chunks(const tc_prefill_desc &d) {
    const int64_t E = d.T > d.W ? d.T - d.W : 0;
    const int C = l2b_chunk(d);
    return (E + C - 1) / C;
}

struct BwdLayout {
    size_t lse, Dt, Ac, Hc, part, total;
};
BwdLayout bwd_layout(const tc_prefill_desc &d) {
    const int64_t BH = d.B * d.H, nC = l2b_chunks(d);
    const size_t mats = (size_t)(BH * nC) * d.dk * d.dv * sizeof(float);
    const size_t stats = (size_t)(BH * backward_stat_stride(d.T)) * sizeof(float);
    BwdLayout L;
    L.lse = 0;
    L.Dt = L.lse + align256(stats);
    L.Ac = L.Dt + align256(stats);
    L.Hc = L.Ac + align256(mats);
    L.part = L.Hc + align256(mats);
    L.total = L.part + align256((size_t)(BH * nC * 3) * sizeof(float));
    return L;
}

// The two window kernels, CPL output columns per lane.
template <typename Tin, int CPL>
cudaError_t launch_window(const BwdParams &p, cudaStream_t s) {
    const dim3 grid((unsigned)((p.T + kTileR - 1) / kTileR), (unsigned)(p.B * p.H));
    const size_t s_rows = rows_smem(p.dk, p.dv), s_keys = keys_smem(p.dk, p.dv);
    cudaError_t e = cudaFuncSetAttribute(bwd_rows_kernel<Tin, CPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_rows);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_keys_kernel<Tin, CPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)s_keys);
    if (e != cudaSuccess) return e;
    bwd_rows_kernel<Tin, CPL><<<grid, kThreads, s_rows, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_keys_kernel<Tin, CPL><<<grid, kThreads, s_keys, s>>>(p);
    return cudaGetLastError();
}

// Memory part and the final reduction of the scalar gradients.
template <typename Tin>
cudaError_t launch_memory(const tc_prefill_desc &d, const BwdParams &p, int *status,
                          unsigned long long wait_ns, cudaStream_t s) {
    const int64_t BH = p.B * p.H;
    // memory part, chunked: sums, scan over the chunks, per-chunk gradients
    const int C = p.C;
    const int64_t E = p.T > p.W ? p.T - p.W : 0;
    const int nC = (int)((E + C - 1) / C);
    const bool tc_chunk = backward_memory_tc_supported(d);
    cudaError_t e = cudaSuccess;
    if (nC > 0) {
        const size_t s_sums = l2b_sums_smem(p.dk, p.dv, C), s_chunk = l2b_chunk_smem(p.dk, p.dv, C);
        if (!tc_chunk) {
            e = cudaFuncSetAttribute(l2b_sums_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)s_sums);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(l2b_chunk_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)s_chunk);
            if (e != cudaSuccess) return e;
        }
        const dim3 grid((unsigned)nC, (unsigned)BH);
        if (tc_chunk) {
            e = launch_backward_sums_tc(d, p.q, p.k, p.v, p.dy, p.lam, p.eta, p.g, p.Ac, p.Hc, status,
                                        wait_ns, s);
        } else {
            l2b_sums_kernel<Tin><<<grid, kThreads, s_sums, s>>>(p);
            e = cudaGetLastError();
        }
        if (e != cudaSuccess) return e;
        l2b_scan_kernel<<<dim3((unsigned)((p.dk * p.dv + kThreads - 1) / kThreads), (unsigned)BH),
                          kThreads, 0, s>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (tc_chunk) {
            e = launch_backward_chunks_tc(d, p.q, p.k, p.v, p.dy, p.lam, p.eta, p.g, p.Ac, p.Hc, p.gq,
                                          p.gk, p.gv, p.part, status, wait_ns, s);
        } else {
            l2b_chunk_kernel<Tin><<<grid, kThreads, s_chunk, s>>>(p);
            e = cudaGetLastError();
        }
        if (e != cudaSuccess) return e;
    }
    bwd_reduce_kernel<<<(unsigned)((p.H + 127) / 128), 128, 0, s>>>(p, nC);
    return cudaGetLastError();
}

// The whole backward: window part (tensor cores where they take the shape),
// then the memory part.
template <typename Tin>
cudaError_t launch_t(const tc_prefill_desc &d, const BwdParams &p, int *status,
                     unsigned long long wait_ns, cudaStream_t s) {
    if (p.T > 0) {
        cudaError_t e;
        if (backward_window_tc_supported(d))
            e = launch_backward_window_tc(d, p.q, p.k, p.v, p.dy, p.gq, p.gk, p.gv, p.lse, p.Dt, status,
                                          wait_ns, s);
        else
            e = (p.dk <= 64 && p.dv <= 64) ? launch_window<Tin, 2>(p, s)
                                           : launch_window<Tin, kMaxD / 32>(p, s);
        if (e != cudaSuccess) return e;
    }
    return launch_memory<Tin>(d, p, status, wait_ns, s);
}

}  // namespace

size_t backward_workspace_bytes(const tc_prefill_desc &d) { return bwd_layout(d).total; }

cudaError_t launch_backward(const tc_prefill_desc &d, const void *q, const void *k, const void *v,
                            const float *lam, const float *eta, const float *g, const void *dy,
                            float *dq, float *dk, float *dv, float *dlam, float *deta, float *dg,
                            void *workspace, int *status, unsigned long long wait_ns,
                            cudaStream_t s) {
    const BwdLayout L = bwd_layout(d);
    char *ws = static_cast<char *>(workspace);
    BwdParams p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.dy = dy;
    p.lam = lam;
    p.eta = eta;
    p.g = g;
    p.gq = dq;
    p.gk = dk;
    p.gv = dv;
    p.lse = reinterpret_cast<float *>(ws + L.lse);
    p.Dt = reinterpret_cast<float *>(ws + L.Dt);
    p.Ac = reinterpret_cast<float *>(ws + L.Ac);
    p.Hc = reinterpret_cast<float *>(ws + L.Hc);
    p.part = reinterpret_cast<float *>(ws + L.part);
    p.dlam = dlam;
    p.deta = deta;
    p.dg = dg;
    p.B = d.B;
    p.H = d.H;
    p.T = d.T;
    p.W = d.W;
    p.dk = (int)d.dk;
    p.dv = (int)d.dv;
    p.stat_stride = backward_window_tc_supported(d) ? backward_stat_stride(d.T) : d.T;
    p.C = l2b_chunk(d);
    return d.dtype == TC_BF16 ? launch_t<__nv_bfloat16>(d, p, status, wait_ns, s)
                              : launch_t<float>(d, p, status, wait_ns, s);
}

int backward_launch_count(const tc_prefill_desc &d) {
    const int window = d.T > 0 ? 2 : 0;
    return window + (l2b_chunks(d) > 0 ? 3 : 0) + 1;
}

}  // namespace tc
