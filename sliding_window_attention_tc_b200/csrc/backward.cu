// Backward of the Tensor Cache layer (outer-product write), float32 SIMT.
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
//   bwd_rows_kernel (a warp per query row) writes dq and the per-row
//   log-sum-exp and D_t; bwd_keys_kernel (a warp per key row, over the W
//   queries that see it) writes dk and dv.
//
// Memory (L2), a reverse scan of G_t = dL/dA_t:
//   G_t = q_t^T (s dy_t) + [step t+1 writes] lam G_{t+1}, and each write at
//   step t (eviction e = t - W) gives dk_e += eta G_t v_e,
//   dv_e += eta G_t^T k_e, deta += <G_t, k_e v_e^T>, dlam += <G_t, A_{t-1}>;
//   also dq_t += A_t (s dy_t) and dg += s (1 - s) <dy_t, q_t A_t>.
//   bwd_l2_kernel (CTAs of 8 rows of A per (b,h)) replays A from
//   checkpoints every kCk tokens and walks the tokens backwards; it adds to
//   dq, dk, dv and leaves partials of dlam, deta, dg, which
//   bwd_reduce_kernel sums over the batch and the row blocks in a fixed order.

#include <cuda_runtime.h>

#include <cstdint>

#include "tc.h"
#include "tc_internal.cuh"

namespace tc {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxD = 128;
constexpr int kRows = kThreads / 32;  // query or key rows per CTA in the L1 kernels
constexpr int kKT = 32;               // key / query tile of the L1 kernels
constexpr int kCk = 64;               // checkpoint interval of the L2 replay
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
    const void *q, *k, *v, *dy;
    const float *lam, *eta, *g;
    float *gq, *gk, *gv;    // gradients of q, k, v (float32, layout of the inputs)
    float *lse, *Dt;        // [BH][T] per query row (log2 domain), <dy, y_local>
    float *ckpt, *seg;      // L2 replay: [BH][nCk][dk*dv], [BH][kCk][dk*dv]
    float *part;            // [BH][3]: dlam, deta, dg
    float *dlam, *deta, *dg;
    int64_t B, H, T, W;
    int dk, dv;
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
// dq (window part), log-sum-exp and D_t, one warp per query row.
template <typename Tin>
__global__ void __launch_bounds__(kThreads) bwd_rows_kernel(BwdParams p) {
    constexpr int CPL = kMaxD / 32;
    __shared__ float sk[kKT][kMaxD + 1], sv[kKT][kMaxD + 1];
    __shared__ float sq[kRows][kMaxD], sdy[kRows][kMaxD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int dk = p.dk, dv = p.dv;
    const int64_t T = p.T, W = p.W;
    const int64_t t0 = (int64_t)blockIdx.x * kRows, t = t0 + warp;
    const bool row_ok = t < T;
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T * dk;
    const Tin *kb = reinterpret_cast<const Tin *>(p.k) + bh * T * dk;
    const Tin *vb = reinterpret_cast<const Tin *>(p.v) + bh * T * dv;
    const Tin *db = reinterpret_cast<const Tin *>(p.dy) + bh * T * dv;
    for (int x = tid; x < kRows * dk; x += kThreads) {
        const int64_t tt = t0 + x / dk;
        sq[x / dk][x % dk] = tt < T ? to_f32(qb[tt * dk + x % dk]) : 0.f;
    }
    for (int x = tid; x < kRows * dv; x += kThreads) {
        const int64_t tt = t0 + x / dv;
        sdy[x / dv][x % dv] = tt < T ? to_f32(db[tt * dv + x % dv]) : 0.f;
    }
    const float scale2 = kLog2e / sqrtf((float)dk);
    const int64_t win_lo = t - W + 1 > 0 ? t - W + 1 : 0;
    const int64_t t_last = (t0 + kRows - 1 < T - 1) ? t0 + kRows - 1 : T - 1;
    const int64_t lo = t0 - W + 1 > 0 ? t0 - W + 1 : 0;

    // pass 1: softmax statistics and y_local (online)
    float m_run = -INFINITY, l_run = 0.f, acc[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = 0.f;
    for (int64_t j0 = lo; j0 <= t_last; j0 += kKT) {
        const int nt = (int)((t_last - j0 + 1 < kKT) ? t_last - j0 + 1 : kKT);
        __syncthreads();
        for (int x = tid; x < nt * dk; x += kThreads) sk[x / dk][x % dk] = to_f32(kb[(j0 + x / dk) * dk + x % dk]);
        for (int x = tid; x < nt * dv; x += kThreads) sv[x / dv][x % dv] = to_f32(vb[(j0 + x / dv) * dv + x % dv]);
        __syncthreads();
        if (!row_ok) continue;
        const int64_t j = j0 + lane;
        const bool in_win = lane < nt && j >= win_lo && j <= t;
        float dot = 0.f;
        if (in_win)
            for (int r = 0; r < dk; ++r) dot = fmaf(sq[warp][r], sk[lane][r], dot);
        const float s = in_win ? dot * scale2 : -INFINITY;
        const float m_new = fmaxf(m_run, warp_max(s));
        if (m_new == -INFINITY) continue;
        const float corr = exp2f(m_run - m_new);
        const float pj = exp2f(s - m_new);
        l_run = l_run * corr + warp_sum(pj);
#pragma unroll
        for (int i = 0; i < CPL; ++i) acc[i] *= corr;
        m_run = m_new;
        for (int jj = 0; jj < nt; ++jj) {
            const float pb = __shfl_sync(0xffffffffu, pj, jj);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = lane + 32 * i;
                if (c < dv) acc[i] = fmaf(pb, sv[jj][c], acc[i]);
            }
        }
    }
    float lse2 = 0.f, Dt = 0.f;
    if (row_ok) {
        lse2 = m_run + log2f(l_run);
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < dv) d = fmaf(sdy[warp][c], acc[i] / l_run, d);
        }
        Dt = warp_sum(d);
        if (lane == 0) {
            p.lse[bh * T + t] = lse2;
            p.Dt[bh * T + t] = Dt;
        }
    }
    // pass 2: ds_j = p_j (dp_j - D_t); dq_t = sum_j ds_j k_j / sqrt(dk)
    float dqa[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) dqa[i] = 0.f;
    const float inv_sqrt = 1.f / sqrtf((float)dk);
    for (int64_t j0 = lo; j0 <= t_last; j0 += kKT) {
        const int nt = (int)((t_last - j0 + 1 < kKT) ? t_last - j0 + 1 : kKT);
        __syncthreads();
        for (int x = tid; x < nt * dk; x += kThreads) sk[x / dk][x % dk] = to_f32(kb[(j0 + x / dk) * dk + x % dk]);
        for (int x = tid; x < nt * dv; x += kThreads) sv[x / dv][x % dv] = to_f32(vb[(j0 + x / dv) * dv + x % dv]);
        __syncthreads();
        if (!row_ok) continue;
        const int64_t j = j0 + lane;
        const bool in_win = lane < nt && j >= win_lo && j <= t;
        float ds = 0.f;
        if (in_win) {
            float dot = 0.f, dp = 0.f;
            for (int r = 0; r < dk; ++r) dot = fmaf(sq[warp][r], sk[lane][r], dot);
            for (int c = 0; c < dv; ++c) dp = fmaf(sdy[warp][c], sv[lane][c], dp);
            ds = exp2f(dot * scale2 - lse2) * (dp - Dt);
        }
        for (int jj = 0; jj < nt; ++jj) {
            const float db_ = __shfl_sync(0xffffffffu, ds, jj);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int r = lane + 32 * i;
                if (r < dk) dqa[i] = fmaf(db_, sk[jj][r], dqa[i]);
            }
        }
    }
    if (row_ok) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int r = lane + 32 * i;
            if (r < dk) p.gq[(bh * T + t) * dk + r] = dqa[i] * inv_sqrt;
        }
    }
}

// ---------------------------------------------------------------------------
// dk, dv (window part), one warp per key row j over the queries t = j .. j+W-1.
template <typename Tin>
__global__ void __launch_bounds__(kThreads) bwd_keys_kernel(BwdParams p) {
    constexpr int CPL = kMaxD / 32;
    __shared__ float sq[kKT][kMaxD + 1], sdy[kKT][kMaxD + 1];
    __shared__ float slse[kKT], sD[kKT];
    __shared__ float sk[kRows][kMaxD], sv[kRows][kMaxD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int dk = p.dk, dv = p.dv;
    const int64_t T = p.T, W = p.W;
    const int64_t j0k = (int64_t)blockIdx.x * kRows, j = j0k + warp;
    const bool row_ok = j < T;
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T * dk;
    const Tin *kb = reinterpret_cast<const Tin *>(p.k) + bh * T * dk;
    const Tin *vb = reinterpret_cast<const Tin *>(p.v) + bh * T * dv;
    const Tin *db = reinterpret_cast<const Tin *>(p.dy) + bh * T * dv;
    for (int x = tid; x < kRows * dk; x += kThreads) {
        const int64_t jj = j0k + x / dk;
        sk[x / dk][x % dk] = jj < T ? to_f32(kb[jj * dk + x % dk]) : 0.f;
    }
    for (int x = tid; x < kRows * dv; x += kThreads) {
        const int64_t jj = j0k + x / dv;
        sv[x / dv][x % dv] = jj < T ? to_f32(vb[jj * dv + x % dv]) : 0.f;
    }
    const float scale2 = kLog2e / sqrtf((float)dk);
    const float inv_sqrt = 1.f / sqrtf((float)dk);
    // queries that see any key of this CTA: j0k .. j0k + kRows - 1 + W - 1
    const int64_t q_hi_all = j0k + kRows - 1 + W - 1 < T - 1 ? j0k + kRows - 1 + W - 1 : T - 1;
    const int64_t q_hi = j + W - 1 < T - 1 ? j + W - 1 : T - 1;
    float dka[CPL], dva[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) dka[i] = dva[i] = 0.f;
    for (int64_t q0 = j0k; q0 <= q_hi_all; q0 += kKT) {
        const int nt = (int)((q_hi_all - q0 + 1 < kKT) ? q_hi_all - q0 + 1 : kKT);
        __syncthreads();
        for (int x = tid; x < nt * dk; x += kThreads) sq[x / dk][x % dk] = to_f32(qb[(q0 + x / dk) * dk + x % dk]);
        for (int x = tid; x < nt * dv; x += kThreads) sdy[x / dv][x % dv] = to_f32(db[(q0 + x / dv) * dv + x % dv]);
        if (tid < nt) {
            slse[tid] = p.lse[bh * T + q0 + tid];
            sD[tid] = p.Dt[bh * T + q0 + tid];
        }
        __syncthreads();
        if (!row_ok) continue;
        const int64_t t = q0 + lane;
        const bool sees = lane < nt && t >= j && t <= q_hi;
        float pj = 0.f, ds = 0.f;
        if (sees) {
            float dot = 0.f, dp = 0.f;
            for (int r = 0; r < dk; ++r) dot = fmaf(sq[lane][r], sk[warp][r], dot);
            for (int c = 0; c < dv; ++c) dp = fmaf(sdy[lane][c], sv[warp][c], dp);
            pj = exp2f(dot * scale2 - slse[lane]);
            ds = pj * (dp - sD[lane]);
        }
        for (int tt = 0; tt < nt; ++tt) {
            const float pb = __shfl_sync(0xffffffffu, pj, tt);
            const float dsb = __shfl_sync(0xffffffffu, ds, tt);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int r = lane + 32 * i;
                if (r < dk) dka[i] = fmaf(dsb, sq[tt][r], dka[i]);
                if (r < dv) dva[i] = fmaf(pb, sdy[tt][r], dva[i]);
            }
        }
    }
    if (row_ok) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int r = lane + 32 * i;
            if (r < dk) p.gk[(bh * T + j) * dk + r] = dka[i] * inv_sqrt;
            if (r < dv) p.gv[(bh * T + j) * dv + r] = dva[i];
        }
    }
}

// ---------------------------------------------------------------------------
// L2 reverse scan.  Row r of G_t = dL/dA_t and of A_t only involves q_t[r],
// k_e[r] and whole rows of dy / v, so each (b,h) is split over CTAs of
// kRows rows (one row per warp; lane l owns columns l, l+32, ...).  A is
// replayed from checkpoints every kCk tokens; a segment's q, dy, k, v are
// staged in shared memory once.  dv_e sums over all rows: the CTAs of a head
// add their parts with atomics.
template <typename Tin>
__global__ void __launch_bounds__(kThreads) bwd_l2_kernel(BwdParams p) {
    constexpr int CPL = kMaxD / 32;
    extern __shared__ float sh[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % p.H);
    const int dk = p.dk, dv = p.dv;
    const int r0 = blockIdx.x * kRows, r = r0 + warp;
    const bool row_ok = r < dk;
    const int64_t T = p.T, W = p.W;
    const float lam = p.lam[h], eta = p.eta[h];
    const float sg = 1.f / (1.f + expf(-p.g[h]));
    // shared: q rows [kCk][kRows], k rows [kCk][kRows], dy [kCk][dv], v [kCk][dv], column sums [kRows][dv]
    float *sQ = sh, *sK = sQ + kCk * kRows, *sDY = sK + kCk * kRows, *sV = sDY + kCk * dv;
    float *scol = sV + kCk * dv;
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T * dk;
    const Tin *kb = reinterpret_cast<const Tin *>(p.k) + bh * T * dk;
    const Tin *vb = reinterpret_cast<const Tin *>(p.v) + bh * T * dv;
    const Tin *db = reinterpret_cast<const Tin *>(p.dy) + bh * T * dv;
    const int64_t nCk = (T + kCk - 1) / kCk;
    const int nrs = gridDim.x;
    // this CTA's slices: [nCk][kRows][dv] checkpoints, [kCk][kRows][dv] segment
    float *ck = p.ckpt + ((bh * nrs + blockIdx.x) * nCk) * (int64_t)kRows * dv;
    float *seg = p.seg + ((bh * nrs + blockIdx.x) * (int64_t)kCk) * kRows * dv;
    auto at = [&](int jx) { return warp * dv + lane + 32 * jx; };  // element of a [kRows][dv] slab
    auto col_ok = [&](int jx) { return lane + 32 * jx < dv; };

    // stage q, dy (tokens tb..te-1) and k, v of their evictions
    auto stage = [&](int64_t tb, int64_t te, bool with_q) {
        __syncthreads();
        const int n = (int)(te - tb);
        for (int x = tid; x < n * kRows; x += kThreads) {
            const int64_t t = tb + x / kRows;
            const int rr = r0 + x % kRows;
            sK[x] = (t >= W && rr < dk) ? to_f32(kb[(t - W) * dk + rr]) : 0.f;
            if (with_q) sQ[x] = rr < dk ? to_f32(qb[t * dk + rr]) : 0.f;
        }
        for (int x = tid; x < n * dv; x += kThreads) {
            const int64_t t = tb + x / dv;
            sV[x] = t >= W ? to_f32(vb[(t - W) * dv + x % dv]) : 0.f;
            if (with_q) sDY[x] = to_f32(db[t * dv + x % dv]);
        }
        __syncthreads();
    };

    float A[CPL];
#pragma unroll
    for (int jx = 0; jx < CPL; ++jx) A[jx] = 0.f;
    // forward replay: checkpoints of A before every kCk-th token
    for (int64_t s = 0; s < nCk; ++s) {
        const int64_t tb = s * kCk, te = tb + kCk < T ? tb + kCk : T;
#pragma unroll
        for (int jx = 0; jx < CPL; ++jx)
            if (col_ok(jx)) ck[s * kRows * dv + at(jx)] = A[jx];
        stage(tb, te, false);
        for (int64_t t = tb; t < te; ++t) {
            if (t < W) continue;
            const float ek = eta * sK[(t - tb) * kRows + warp];
#pragma unroll
            for (int jx = 0; jx < CPL; ++jx)
                if (col_ok(jx)) A[jx] = fmaf(lam, A[jx], ek * sV[(t - tb) * dv + lane + 32 * jx]);
        }
    }

    float G[CPL];
#pragma unroll
    for (int jx = 0; jx < CPL; ++jx) G[jx] = 0.f;
    float pl = 0.f, pe = 0.f, pg = 0.f;  // dlam, deta, dg partials
    for (int64_t s = nCk - 1; s >= 0; --s) {
        const int64_t tb = s * kCk, te = tb + kCk < T ? tb + kCk : T;
        stage(tb, te, true);
        // replay the segment, keeping every A_t of this CTA's rows
#pragma unroll
        for (int jx = 0; jx < CPL; ++jx)
            if (col_ok(jx)) A[jx] = ck[s * kRows * dv + at(jx)];
        for (int64_t t = tb; t < te; ++t) {
            if (t >= W) {
                const float ek = eta * sK[(t - tb) * kRows + warp];
#pragma unroll
                for (int jx = 0; jx < CPL; ++jx)
                    if (col_ok(jx)) A[jx] = fmaf(lam, A[jx], ek * sV[(t - tb) * dv + lane + 32 * jx]);
            }
#pragma unroll
            for (int jx = 0; jx < CPL; ++jx)
                if (col_ok(jx)) seg[(t - tb) * kRows * dv + at(jx)] = A[jx];
        }
        for (int64_t t = te - 1; t >= tb; --t) {
            const int i = (int)(t - tb);
            const float qr = sQ[i * kRows + warp];
            // dq_t[r] += sum_c A_t[r][c] dm_t[c];  dg partial (1 - s) q_t[r] (that)
            float acc = 0.f;
#pragma unroll
            for (int jx = 0; jx < CPL; ++jx)
                if (col_ok(jx)) acc = fmaf(seg[i * kRows * dv + at(jx)], sg * sDY[i * dv + lane + 32 * jx], acc);
            acc = warp_sum(acc);
            if (row_ok && lane == 0) p.gq[(bh * T + t) * dk + r] += acc;
            pg = fmaf((1.f - sg) * qr, acc, pg);
            // G += q_t (x) dm_t
#pragma unroll
            for (int jx = 0; jx < CPL; ++jx)
                if (col_ok(jx)) G[jx] = fmaf(qr, sg * sDY[i * dv + lane + 32 * jx], G[jx]);
            if (t >= W) {
                const int64_t e = t - W;
                const float kr = sK[i * kRows + warp];
                float a2 = 0.f;
#pragma unroll
                for (int jx = 0; jx < CPL; ++jx) {
                    if (!col_ok(jx)) continue;
                    a2 = fmaf(G[jx], sV[i * dv + lane + 32 * jx], a2);
                    const float Ap = t > tb ? seg[(i - 1) * kRows * dv + at(jx)]
                                            : ck[s * kRows * dv + at(jx)];
                    pl = fmaf(G[jx], Ap, pl);
                    scol[at(jx)] = G[jx] * kr;
                }
                a2 = warp_sum(a2);
                if (row_ok && lane == 0) p.gk[(bh * T + e) * dk + r] += eta * a2;
                pe = fmaf(kr, a2, pe);
                __syncthreads();
                for (int c = tid; c < dv; c += kThreads) {
                    float sum = 0.f;
                    for (int w = 0; w < kRows; ++w) sum += scol[w * dv + c];
                    atomicAdd(&p.gv[(bh * T + e) * dv + c], eta * sum);
                }
                __syncthreads();
#pragma unroll
                for (int jx = 0; jx < CPL; ++jx) G[jx] *= lam;
            }
        }
    }
    // partials of this CTA: pl differs per lane; pe and pg are equal in all
    // lanes of a warp (only lane 0's count); rows past dk hold zeros
    __shared__ float sred[3][kRows];
    pl = warp_sum(pl);
    if (lane == 0) {
        sred[0][warp] = pl;
        sred[1][warp] = pe;
        sred[2][warp] = pg;
    }
    __syncthreads();
    if (tid < 3) {
        float a = 0.f;
        for (int w = 0; w < kRows; ++w) a += sred[tid][w];
        p.part[(bh * nrs + blockIdx.x) * 3 + tid] = a;
    }
}

// dlam, deta, dg per head: the (b,h) partials summed over the batch in a
// fixed order.
__global__ void bwd_reduce_kernel(BwdParams p, int nrs) {
    const int64_t h = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= p.H) return;
    float a = 0.f, b_ = 0.f, c = 0.f;
    for (int64_t b = 0; b < p.B; ++b)
        for (int x = 0; x < nrs; ++x) {
            const float *pp = p.part + ((b * p.H + h) * nrs + x) * 3;
            a += pp[0];
            b_ += pp[1];
            c += pp[2];
        }
    p.dlam[h] = a;
    p.deta[h] = b_;
    p.dg[h] = c;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdLayout {
    size_t lse, Dt, ckpt, seg, part, total;
};
BwdLayout bwd_layout(const tc_prefill_desc &d) {
    const int64_t BH = d.B * d.H, nrs = (d.dk + kRows - 1) / kRows;
    const int64_t slab = nrs * kRows * d.dv;  // rows of A / G padded to whole CTAs
    const int64_t nCk = (d.T + kCk - 1) / kCk;
    BwdLayout L;
    L.lse = 0;
    L.Dt = L.lse + align256((size_t)(BH * d.T) * sizeof(float));
    L.ckpt = L.Dt + align256((size_t)(BH * d.T) * sizeof(float));
    L.seg = L.ckpt + align256((size_t)(BH * nCk * slab) * sizeof(float));
    L.part = L.seg + align256((size_t)(BH * kCk * slab) * sizeof(float));
    L.total = L.part + align256((size_t)(BH * nrs * 3) * sizeof(float));
    return L;
}

template <typename Tin>
cudaError_t launch_t(const BwdParams &p, cudaStream_t s) {
    const int64_t BH = p.B * p.H;
    if (p.T > 0) {
        const dim3 grid((unsigned)((p.T + kRows - 1) / kRows), (unsigned)BH);
        bwd_rows_kernel<Tin><<<grid, kThreads, 0, s>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        bwd_keys_kernel<Tin><<<grid, kThreads, 0, s>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int nrs = (p.dk + kRows - 1) / kRows;
    const size_t smem = (size_t)(2 * kCk * kRows + 2 * kCk * p.dv + kRows * p.dv) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_l2_kernel<Tin>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_l2_kernel<Tin><<<dim3((unsigned)nrs, (unsigned)BH), kThreads, smem, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_reduce_kernel<<<(unsigned)((p.H + 127) / 128), 128, 0, s>>>(p, nrs);
    return cudaGetLastError();
}

}  // namespace

size_t backward_workspace_bytes(const tc_prefill_desc &d) { return bwd_layout(d).total; }

cudaError_t launch_backward(const tc_prefill_desc &d, const void *q, const void *k, const void *v,
                            const float *lam, const float *eta, const float *g, const void *dy,
                            float *dq, float *dk, float *dv, float *dlam, float *deta, float *dg,
                            void *workspace, cudaStream_t s) {
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
    p.ckpt = reinterpret_cast<float *>(ws + L.ckpt);
    p.seg = reinterpret_cast<float *>(ws + L.seg);
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
    return d.dtype == TC_BF16 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace tc
