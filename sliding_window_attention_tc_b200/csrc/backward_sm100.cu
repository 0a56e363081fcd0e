// Window (L1) part of the backward on the tensor cores: bf16 q, k, v, dy with
// d_k = d_v = 64.
//
// "Tensor Cache: Eviction-conditioned Associative Memory for Transformers",
// §2 training considerations (the layer is trained end to end through its
// window attention and its memory).  Over the window pairs t - W < j <= t:
//   p_tj = softmax_j(<q_t, k_j> / sqrt(d)),  dp_tj = <dy_t, v_j>,
//   D_t = sum_j p_tj dp_tj  (= <dy_t, y_local_t>),  ds_tj = p_tj (dp_tj - D_t),
//   dq_t = sum_j ds_tj k_j / sqrt(d),  dk_j = sum_t ds_tj q_t / sqrt(d),
//   dv_j = sum_t p_tj dy_t.
//
// Two kernels of one shape.  A CTA owns a block of 128 rows (the TMEM lanes
// and the M of every MMA) and walks the 64-row tiles of the other side that
// share a window pair with them:
//   rows kernel: own = queries (Q, dY), other = keys (K, V).  Pass 1 takes
//     the softmax statistics online (row max, row sum, and D_t from P and
//     dP); pass 2 forms dS and accumulates dQ += dS K.  Writes dq and, per
//     query row, the log-sum-exp (log2 domain) and D_t.
//   keys kernel: own = keys (K, V), other = queries (Q, dY) with their
//     log-sum-exp and D_t; accumulates dV += P^T dY and dK += dS^T Q.
// Per tile, S = own_a x_a^T and dP = own_b x_b^T go to TMEM (fp32) on the
// tensor cores.  The softmax warps turn them into P and dS and write them back
// over S and dP as bf16 pairs split hi + lo (x = hi + lo with both parts
// bf16; the remainder is below 2^-17 |x|).  Those feed the gradient MMAs as
// the TMEM operand A, with the other tile read MN-major as B.  Products of
// the bf16 inputs are exact in the float32 accumulators, so the gradients
// keep float32 accuracy up to the split (a few 1e-6 relative).
//
// Roles (192 threads, two CTAs per SM): warp 0 issues the TMA copies (own
// block once, other tiles through a 4-stage ring), warp 1 issues the MMAs,
// warps 2-5 (one TMEM lane each per thread, row r = 32 (warp % 4) + lane)
// do the element-wise work and the epilogue.  Every wait is bounded: one
// that runs out sets the CTA's abort flag and TC_ERR_DEVICE_TIMEOUT, and
// every role drains and returns.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100_ptx.cuh"
#include "tc.h"
#include "tc_internal.cuh"

namespace tc {
namespace {

using namespace sm100;

constexpr int HDB = 64;              // head size of this path
constexpr int BO = 128;              // own rows per CTA
constexpr int BX = 64;               // rows per other-side tile
constexpr int NSX = 4;               // other-side tile stages
constexpr int kBwdTcThreads = 192;
constexpr float kLog2eF = 1.4426950408889634f;

constexpr uint32_t OWN_TILE = BO * HDB * 2;  // 16 KB
constexpr uint32_t X_TILE = BX * HDB * 2;    // 8 KB
constexpr uint32_t OFF_OWN = 0;                           // own_a, own_b
constexpr uint32_t OFF_XS = 2 * OWN_TILE;                 // NSX x (x_a, x_b)
constexpr uint32_t OFF_ST = OFF_XS + NSX * 2 * X_TILE;    // NSX x (lse[64], D[64]) (keys kernel)
constexpr uint32_t OFF_BARS = OFF_ST + NSX * 2 * BX * 4;
constexpr uint32_t SMEM_BWD_TC = OFF_BARS + 128 + 1024;   // + slack for the 1024-byte alignment

// TMEM columns: S (then P hi/lo), dP (then dS hi/lo), two accumulators.
constexpr uint32_t TMC_S = 0, TMC_DP = 64, TMC_ACC0 = 128, TMC_ACC1 = 192, TMC_COLS = 256;

struct BwdTcParams {
    float *out0, *out1;  // rows kernel: dq; keys kernel: dk, dv  ([BH][T][64] float32)
    float *lse, *Dt;     // [BH][Tp] per query row: log-sum-exp (log2), D_t
    int T, Tp, W;        // W clamped to T
    int *status;
    unsigned long long wait_ns;
};

__device__ __forceinline__ bool warp_wait_b(uint64_t *bar, uint32_t parity, volatile int *abort,
                                            int *status, uint64_t limit) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status, limit));
}

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// x0, x1 -> bf16 pair hi and the bf16 pair of the remainders lo.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16(x0, x1);
    const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
    lo = pack_bf16(x0 - h0, x1 - h1);
}

template <bool KEYS>
__global__ void __launch_bounds__(kBwdTcThreads, 2)
    bwd_window_tc_kernel(const __grid_constant__ CUtensorMap t_own_a,
                         const __grid_constant__ CUtensorMap t_own_b,
                         const __grid_constant__ CUtensorMap t_x_a,
                         const __grid_constant__ CUtensorMap t_x_b,
                         const __grid_constant__ CUtensorMap t_lse,
                         const __grid_constant__ CUtensorMap t_D, BwdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BARS);
    uint64_t *own_full = bars, *x_full = bars + 1, *x_empty = x_full + NSX;
    uint64_t *s_full = x_empty + NSX, *ops_ready = s_full + 1, *acc_full = ops_ready + 1;
    uint64_t *mma_done = acc_full + 1;
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int T = p.T, W = p.W;
    const int bh = blockIdx.y;
    const int o0 = blockIdx.x * BO;  // first own row
    // other-side tiles xs, xs + 64, ... (nX of them); the rows kernel walks them twice
    int xs, nX;
    if (KEYS) {
        xs = o0;
        const int64_t hi = min((int64_t)T - 1, (int64_t)o0 + BO - 2 + W);
        nX = (int)((hi - xs) / BX) + 1;
    } else {
        const int lo = max(0, o0 - W + 1);
        const int hi = min(T - 1, o0 + BO - 1);
        xs = lo & ~(BX - 1);
        nX = (hi - xs) / BX + 1;
    }
    const int N = KEYS ? nX : 2 * nX;

    if (tid == 0) {
        mbar_init(own_full, 1);
        for (int s = 0; s < NSX; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(ops_ready, 4);
        mbar_init(acc_full, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base, TMC_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (tid == 0) {
            tma_prefetch_desc(&t_own_a);
            tma_prefetch_desc(&t_own_b);
            tma_prefetch_desc(&t_x_a);
            tma_prefetch_desc(&t_x_b);
            mbar_expect_tx(own_full, 2 * OWN_TILE);
            tma_load_3d(sm + OFF_OWN, &t_own_a, own_full, 0, o0, bh);
            tma_load_3d(sm + OFF_OWN + OWN_TILE, &t_own_b, own_full, 0, o0, bh);
            int n = 0;
            for (; n < N; ++n) {
                const int s = n % NSX;
                if (!mbar_wait(&x_empty[s], ((n / NSX) & 1) ^ 1, abort, p.status, p.wait_ns)) break;
                const int x0 = xs + BX * (n % nX);
                uint8_t *dst = sm + OFF_XS + s * 2 * X_TILE;
                mbar_expect_tx(&x_full[s], 2 * X_TILE + (KEYS ? 2 * BX * 4 : 0));
                tma_load_3d(dst, &t_x_a, &x_full[s], 0, x0, bh);
                tma_load_3d(dst + X_TILE, &t_x_b, &x_full[s], 0, x0, bh);
                if (KEYS) {
                    float *st = reinterpret_cast<float *>(sm + OFF_ST) + s * 2 * BX;
                    tma_load_2d(st, &t_lse, &x_full[s], x0, bh);
                    tma_load_2d(st + BX, &t_D, &x_full[s], x0, bh);
                }
            }
            // every issued copy lands before the CTA exits
            mbar_wait_drain(own_full, 0);
            for (int st = 0; st < NSX; ++st) {
                const int fills = n > st ? (n - 1 - st) / NSX + 1 : 0;
                if (fills) mbar_wait_drain(&x_full[st], (fills - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Per tile n: S and dP (K = 64 in four steps), then, once the softmax
        // warps have turned them into operands, the gradient MMAs of tile n
        // (issued before S of tile n+1, which overwrites their operands: the
        // tensor core runs one thread's MMAs in issue order).
        const uint32_t id_s = idesc_bf16(128, 64, false, false);
        const uint32_t id_g = idesc_bf16(128, 64, false, true);
        const uint32_t own_a = smem_u32(sm + OFF_OWN), own_b = own_a + OWN_TILE;
        const uint32_t xbase = smem_u32(sm + OFF_XS);
        bool ok = warp_wait_b(own_full, 0, abort, p.status, p.wait_ns);
        bool first_grad = true;
        for (int n = 0; ok && n <= N; ++n) {
            if (n > 0) {
                const int m = n - 1, sp = m % NSX;
                if (!(ok = warp_wait_b(ops_ready, m & 1, abort, p.status, p.wait_ns))) break;
                tc_fence_after();
                if (KEYS || m >= nX) {
                    const uint32_t xa = xbase + sp * 2 * X_TILE, xb = xa + X_TILE;
                    const uint64_t da = sdesc_sw128(xa, X_TILE, 1024);
                    // acc0 += dS x_a: K step k reads dS columns 16k..16k+15,
                    // hi at 32 (k/2) + 8 (k%2), lo 16 columns further
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t col = TMC_DP + 32 * (k >> 1) + 8 * (k & 1);
                        mma_ts_w(tb + TMC_ACC0, tb + col, da + 128 * k, id_g, (first_grad && k == 0) ? 0u : 1u);
                        mma_ts_w(tb + TMC_ACC0, tb + col + 16, da + 128 * k, id_g, 1u);
                    }
                    if (KEYS) {
                        const uint64_t db = sdesc_sw128(xb, X_TILE, 1024);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t col = TMC_S + 32 * (k >> 1) + 8 * (k & 1);
                            mma_ts_w(tb + TMC_ACC1, tb + col, db + 128 * k, id_g,
                                     (first_grad && k == 0) ? 0u : 1u);
                            mma_ts_w(tb + TMC_ACC1, tb + col + 16, db + 128 * k, id_g, 1u);
                        }
                    }
                    first_grad = false;
                }
                mma_commit_w(&x_empty[sp]);
            }
            if (n == N) break;
            const int s = n % NSX;
            if (!(ok = warp_wait_b(&x_full[s], (n / NSX) & 1, abort, p.status, p.wait_ns))) break;
            tc_fence_after();
            const uint32_t xa = xbase + s * 2 * X_TILE, xb = xa + X_TILE;
            const uint64_t oa = sdesc_sw128(own_a, 16, 1024), ob = sdesc_sw128(own_b, 16, 1024);
            const uint64_t ka = sdesc_sw128(xa, 16, 1024), kb = sdesc_sw128(xb, 16, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_ss_w(tb + TMC_S, oa + 2 * k, ka + 2 * k, id_s, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_ss_w(tb + TMC_DP, ob + 2 * k, kb + 2 * k, id_s, k > 0);
            mma_commit_w(s_full);
        }
        if (ok) mma_commit_w(acc_full);
        // nothing may still run on the tensor cores when TMEM is released
        mma_commit_w(mma_done);
        mbar_wait_drain(mma_done, 0);
    } else {
        // ------------------------------------------------------------ softmax side + epilogue
        const int q4 = warp & 3;
        const int r = 32 * q4 + (tid & 31);
        const uint32_t lanes = tb + ((uint32_t)(32 * q4) << 16);
        const float sl2 = kLog2eF * 0.125f;  // log2(e) / sqrt(64)
        const int orow = o0 + r;
        const float *stat = reinterpret_cast<const float *>(sm + OFF_ST);
        // rows kernel: online statistics of query row orow
        float m_run = -INFINITY, l_run = 0.f, d_run = 0.f, lse2 = 0.f, Drow = 0.f;
        bool ok = true;
        for (int n = 0; n < N; ++n) {
            if (!(ok = warp_wait_b(s_full, n & 1, abort, p.status, p.wait_ns))) break;
            tc_fence_after();
            const int x0 = xs + BX * (n % nX);
            // window test of column c: (unsigned)(base - c) < wlim (rows kernel:
            // base - c = t - j) or (unsigned)(c - base) < wlim and c < climit
            // (keys kernel: c - base = t - j, t < T)
            const int base = orow - x0;
            const uint32_t wlim = (KEYS || orow < T) ? (uint32_t)W : 0u;
            const int climit = T - x0;
            if (!KEYS && n < nX) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t sr[32], pr[32];
                    tmem_ld32(lanes + TMC_S + 32 * h, sr);
                    tmem_ld32(lanes + TMC_DP + 32 * h, pr);
                    tmem_wait_ld();
                    float x[32];
                    float mx = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const bool in = (uint32_t)(base - (32 * h + c)) < wlim;
                        x[c] = in ? __uint_as_float(sr[c]) * sl2 : -INFINITY;
                        mx = fmaxf(mx, x[c]);
                    }
                    const float m_new = fmaxf(m_run, mx);
                    if (m_new != -INFINITY) {
                        const float corr = ex2f(m_run - m_new);
                        float sum = 0.f, dsum = 0.f;
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const float e = ex2f(x[c] - m_new);
                            sum += e;
                            dsum = fmaf(e, __uint_as_float(pr[c]), dsum);
                        }
                        l_run = fmaf(l_run, corr, sum);
                        d_run = fmaf(d_run, corr, dsum);
                        m_run = m_new;
                    }
                }
                if (n == nX - 1 && l_run > 0.f) {
                    lse2 = m_run + log2f(l_run);
                    Drow = d_run / l_run;
                }
            } else {
                const float *st = stat + (n % NSX) * 2 * BX;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t sr[32], pr[32];
                    tmem_ld32(lanes + TMC_S + 32 * h, sr);
                    tmem_ld32(lanes + TMC_DP + 32 * h, pr);
                    tmem_wait_ld();
                    uint32_t phi[16], plo[16], dhi[16], dlo[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float pp[2], dd[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int c = 2 * e + u, cc = 32 * h + c;
                            float L, D;
                            bool in;
                            if (KEYS) {
                                L = st[cc];
                                D = st[BX + cc];
                                in = (uint32_t)(cc - base) < wlim && cc < climit;
                            } else {
                                L = lse2;
                                D = Drow;
                                in = (uint32_t)(base - cc) < wlim;
                            }
                            const float pv = in ? ex2f(fmaf(__uint_as_float(sr[c]), sl2, -L)) : 0.f;
                            pp[u] = pv;
                            dd[u] = pv * (__uint_as_float(pr[c]) - D);
                        }
                        split_pair(dd[0], dd[1], dhi[e], dlo[e]);
                        if (KEYS) split_pair(pp[0], pp[1], phi[e], plo[e]);
                    }
                    tmem_st16(lanes + TMC_DP + 32 * h, dhi);
                    tmem_st16(lanes + TMC_DP + 32 * h + 16, dlo);
                    if (KEYS) {
                        tmem_st16(lanes + TMC_S + 32 * h, phi);
                        tmem_st16(lanes + TMC_S + 32 * h + 16, plo);
                    }
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            mbar_arrive_w(ops_ready);
        }
        // epilogue: accumulators -> float32 gradients (and the row statistics)
        if (ok && warp_wait_b(acc_full, 0, abort, p.status, p.wait_ns)) {
            tc_fence_after();
            const size_t row = (size_t)bh * T + orow;
#pragma unroll
            for (int a = 0; a < (KEYS ? 2 : 1); ++a) {
                const float scale = a == 0 ? 0.125f : 1.f;  // 1/sqrt(64) on dq, dk
                float *out = a == 0 ? p.out0 : p.out1;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v[32];
                    tmem_ld32(lanes + (a == 0 ? TMC_ACC0 : TMC_ACC1) + 32 * h, v);
                    tmem_wait_ld();
                    if (orow < T) {
                        float4 *dst = reinterpret_cast<float4 *>(out + row * HDB + 32 * h);
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            dst[c] = make_float4(__uint_as_float(v[4 * c]) * scale,
                                                 __uint_as_float(v[4 * c + 1]) * scale,
                                                 __uint_as_float(v[4 * c + 2]) * scale,
                                                 __uint_as_float(v[4 * c + 3]) * scale);
                    }
                }
            }
            if (!KEYS && orow < p.Tp) {
                p.lse[(size_t)bh * p.Tp + orow] = orow < T ? lse2 : 0.f;
                p.Dt[(size_t)bh * p.Tp + orow] = orow < T ? Drow : 0.f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, TMC_COLS);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [BH][T][64] bf16 -> 3D map, boxes of 64 x rows x 1 with the 128-byte swizzle;
// rows past T read as zero.
bool rows_map(CUtensorMap *m, const void *base, int T, int BH, int rows) {
    EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HDB, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)HDB * 2, (cuuint64_t)T * HDB * 2};
    cuuint32_t box[3] = {HDB, (cuuint32_t)rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH][Tp] float32 -> 2D map, boxes of 64 x 1 (Tp a multiple of 64).
bool stat_map(CUtensorMap *m, const float *base, int Tp, int BH) {
    EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)Tp, (cuuint64_t)BH};
    cuuint64_t strides[1] = {(cuuint64_t)Tp * 4};
    cuuint32_t box[2] = {(cuuint32_t)BX, 1};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool backward_window_tc_supported(const tc_prefill_desc &d) {
    return d.dtype == TC_BF16 && d.dk == HDB && d.dv == HDB && d.T >= 1 && d.T < (int64_t(1) << 30) &&
           d.B * d.H <= 65535 && tensor_map_encoder() != nullptr;
}

int64_t backward_stat_stride(int64_t T) { return (T + BX - 1) / BX * BX; }

cudaError_t launch_backward_window_tc(const tc_prefill_desc &d, const void *q, const void *k,
                                      const void *v, const void *dy, float *dq, float *dk, float *dv,
                                      float *lse, float *Dt, int *status, unsigned long long wait_ns,
                                      cudaStream_t s) {
    const int T = (int)d.T, BH = (int)(d.B * d.H);
    const int Tp = (int)backward_stat_stride(d.T);
    CUtensorMap mq_o, mdy_o, mk_x, mv_x, mk_o, mv_o, mq_x, mdy_x, mlse, mD;
    if (!rows_map(&mq_o, q, T, BH, BO) || !rows_map(&mdy_o, dy, T, BH, BO) ||
        !rows_map(&mk_x, k, T, BH, BX) || !rows_map(&mv_x, v, T, BH, BX) ||
        !rows_map(&mk_o, k, T, BH, BO) || !rows_map(&mv_o, v, T, BH, BO) ||
        !rows_map(&mq_x, q, T, BH, BX) || !rows_map(&mdy_x, dy, T, BH, BX) ||
        !stat_map(&mlse, lse, Tp, BH) || !stat_map(&mD, Dt, Tp, BH))
        return cudaErrorInvalidValue;
    BwdTcParams p{};
    p.lse = lse;
    p.Dt = Dt;
    p.T = T;
    p.Tp = Tp;
    p.W = (int)(d.W < d.T ? d.W : d.T);
    p.status = status;
    p.wait_ns = wait_ns;
    const dim3 grid((unsigned)((T + BO - 1) / BO), (unsigned)BH);
    cudaError_t e = cudaFuncSetAttribute(bwd_window_tc_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BWD_TC);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_window_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BWD_TC);
    if (e != cudaSuccess) return e;
    p.out0 = dq;
    p.out1 = nullptr;
    bwd_window_tc_kernel<false><<<grid, kBwdTcThreads, SMEM_BWD_TC, s>>>(mq_o, mdy_o, mk_x, mv_x, mlse, mD, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    p.out0 = dk;
    p.out1 = dv;
    bwd_window_tc_kernel<true><<<grid, kBwdTcThreads, SMEM_BWD_TC, s>>>(mk_o, mv_o, mq_x, mdy_x, mlse, mD, p);
    return cudaGetLastError();
}

}  // namespace tc
