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
//   bwd_rows_kernel (a warp per 4 query rows) writes dq and the per-row
//   log-sum-exp and D_t; bwd_keys_kernel (a warp per 4 key rows, over the W
//   queries that see them) writes dk and dv.
//
// Memory (L2), a reverse scan of G_t = dL/dA_t:
//   G_t = q_t^T (s dy_t) + [step t+1 writes] lam G_{t+1}, and each write at
//   step t (eviction e = t - W) gives dk_e += eta G_t v_e,
//   dv_e += eta G_t^T k_e, deta += <G_t, k_e v_e^T>, dlam += <G_t, A_{t-1}>;
//   also dq_t += A_t (s dy_t) and dg += s (1 - s) <dy_t, q_t A_t>.
//   bwd_l2_kernel (CTAs of 8 rows of A per (b,h), one thread-block cluster
//   per (b,h)) replays A from checkpoints every kCk tokens and walks the
//   tokens backwards; it adds to dq, dk, dv and leaves partials of dlam,
//   deta, dg, which bwd_reduce_kernel sums over the batch and the row blocks
//   in a fixed order.  dv_e sums over all rows of G: each CTA keeps its rows'
//   part for a segment's evictions in shared memory, and the cluster adds
//   the parts rank by rank through distributed shared memory.  No step
//   depends on the order in which CTAs run, so the gradients are the same
//   bit for bit on every run.

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tc.h"
#include "tc_internal.cuh"

namespace tc {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxD = 128;
constexpr int kRows = kThreads / 32;  // rows of A per CTA in the L2 kernel
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
            p.lse[bh * T + t] = lse2[i];
            p.Dt[bh * T + t] = Dt[i];
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
            slse[tid] = p.lse[bh * T + q0 + tid];
            sD[tid] = p.Dt[bh * T + q0 + tid];
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
// L2 reverse scan.  Row r of G_t = dL/dA_t and of A_t only involves q_t[r],
// k_e[r] and whole rows of dy / v, so each (b,h) is split over CTAs of
// kRows rows (one row per warp; lane l owns columns l, l+32, ...).  A is
// replayed from checkpoints every kCk tokens; a segment's q, dy, k, v are
// staged in shared memory once.  dv_e sums over all rows: the CTAs of a head
// are one cluster, and after each segment every CTA adds one slice of the
// segment's evictions over the cluster's parts, rank by rank.
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
    // shared: q rows [kCk][kRows], k rows [kCk][kRows], dy [kCk][dv], v [kCk][dv], column sums
    // [kRows][dv], this CTA's part of dv for the segment's evictions [kCk][dv]
    float *sQ = sh, *sK = sQ + kCk * kRows, *sDY = sK + kCk * kRows, *sV = sDY + kCk * dv;
    float *scol = sV + kCk * dv;
    float *sDV = scol + kRows * dv;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
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
                    sDV[i * dv + c] = sum;
                }
                __syncthreads();
#pragma unroll
                for (int jx = 0; jx < CPL; ++jx) G[jx] *= lam;
            }
        }
        // dv of the segment's evictions e = t - W (t in [max(tb, W), te)): the
        // parts of all row blocks, added in rank order; CTA x of the cluster
        // takes every nrs-th eviction starting at x
        cluster.sync();
        const int64_t t_first = tb > W ? tb : W;
        for (int64_t t = t_first + blockIdx.x; t < te; t += nrs) {
            const int i = (int)(t - tb);
            for (int c = tid; c < dv; c += kThreads) {
                float sum = 0.f;
                for (int q = 0; q < nrs; ++q) sum += cluster.map_shared_rank(sDV, q)[i * dv + c];
                p.gv[(bh * T + (t - W)) * dv + c] += eta * sum;
            }
        }
        cluster.sync();  // the parts are read before the next segment overwrites them
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

template <typename Tin>
cudaError_t launch_t(const BwdParams &p, cudaStream_t s) {
    const int64_t BH = p.B * p.H;
    if (p.T > 0) {
        const cudaError_t e = (p.dk <= 64 && p.dv <= 64) ? launch_window<Tin, 2>(p, s)
                                                          : launch_window<Tin, kMaxD / 32>(p, s);
        if (e != cudaSuccess) return e;
    }
    const int nrs = (p.dk + kRows - 1) / kRows;  // row blocks = CTAs of one cluster (<= 16)
    const size_t smem =
        (size_t)(2 * kCk * kRows + 2 * kCk * p.dv + kRows * p.dv + kCk * p.dv) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_l2_kernel<Tin>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (nrs > 8) {
        e = cudaFuncSetAttribute(bwd_l2_kernel<Tin>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nrs, (unsigned)BH);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)nrs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, bwd_l2_kernel<Tin>, p);
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
