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
#include <cuda_bf16.h>
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

constexpr uint32_t BLK_O = BO * 128;  // 16 KB: 128 rows x 64 bf16 columns
constexpr uint32_t BLK_X = BX * 128;  // 8 KB: 64 rows x 64 bf16 columns

// Layout of the window kernels for head size D = 64 NB: tiles are NB blocks
// of 64 columns.  TMEM: S (then P hi/lo), dP (then dS hi/lo), two D-column
// accumulators.
template <int NB>
struct BwdCfg {
    static constexpr int D = 64 * NB;
    static constexpr uint32_t OWN = NB * BLK_O, XT = NB * BLK_X;
    static constexpr uint32_t OFF_OWN = 0;                         // own_a, own_b
    static constexpr uint32_t OFF_XS = 2 * OWN;                    // NSX x (x_a, x_b)
    static constexpr uint32_t OFF_ST = OFF_XS + NSX * 2 * XT;      // NSX x (lse[64], D[64]) (keys kernel)
    static constexpr uint32_t OFF_BARS = OFF_ST + NSX * 2 * BX * 4;
    static constexpr uint32_t SMEM = OFF_BARS + 128 + 1024;        // + slack for the 1024-byte alignment
    static constexpr uint32_t TMC_S = 0, TMC_DP = 64, TMC_ACC0 = 128, TMC_ACC1 = 128 + D;
    static constexpr uint32_t COLS = NB == 1 ? 256 : 512;
};

struct BwdTcParams {
    float *out0, *out1;  // rows kernel: dq; keys kernel: dk, dv  ([BH][T][D] float32)
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

template <bool KEYS, int NB>
__global__ void __launch_bounds__(kBwdTcThreads, NB == 1 ? 2 : 1)
    bwd_window_tc_kernel(const __grid_constant__ CUtensorMap t_own_a,
                         const __grid_constant__ CUtensorMap t_own_b,
                         const __grid_constant__ CUtensorMap t_x_a,
                         const __grid_constant__ CUtensorMap t_x_b,
                         const __grid_constant__ CUtensorMap t_lse,
                         const __grid_constant__ CUtensorMap t_D, BwdTcParams p) {
    using Cf = BwdCfg<NB>;
    constexpr int D = Cf::D;
    constexpr uint32_t OWN_TILE = Cf::OWN, X_TILE = Cf::XT, OFF_OWN = Cf::OFF_OWN, OFF_XS = Cf::OFF_XS;
    constexpr uint32_t OFF_ST = Cf::OFF_ST, TMC_S = Cf::TMC_S, TMC_DP = Cf::TMC_DP;
    constexpr uint32_t TMC_ACC0 = Cf::TMC_ACC0, TMC_ACC1 = Cf::TMC_ACC1, TMC_COLS = Cf::COLS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Cf::OFF_BARS);
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
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                tma_load_3d(sm + OFF_OWN + b * BLK_O, &t_own_a, own_full, 64 * b, o0, bh);
                tma_load_3d(sm + OFF_OWN + OWN_TILE + b * BLK_O, &t_own_b, own_full, 64 * b, o0, bh);
            }
            int n = 0;
            for (; n < N; ++n) {
                const int s = n % NSX;
                if (!mbar_wait(&x_empty[s], ((n / NSX) & 1) ^ 1, abort, p.status, p.wait_ns)) break;
                const int x0 = xs + BX * (n % nX);
                uint8_t *dst = sm + OFF_XS + s * 2 * X_TILE;
                mbar_expect_tx(&x_full[s], 2 * X_TILE + (KEYS ? 2 * BX * 4 : 0));
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    tma_load_3d(dst + b * BLK_X, &t_x_a, &x_full[s], 64 * b, x0, bh);
                    tma_load_3d(dst + X_TILE + b * BLK_X, &t_x_b, &x_full[s], 64 * b, x0, bh);
                }
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
        const uint32_t id_g = idesc_bf16(128, D, false, true);  // N = D over NB column blocks
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
                    const uint64_t da = sdesc_sw128(xa, BLK_X, 1024);
                    // acc0 += dS x_a: K step k reads dS columns 16k..16k+15,
                    // hi at 32 (k/2) + 8 (k%2), lo 16 columns further
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t col = TMC_DP + 32 * (k >> 1) + 8 * (k & 1);
                        mma_ts_w(tb + TMC_ACC0, tb + col, da + 128 * k, id_g, (first_grad && k == 0) ? 0u : 1u);
                        mma_ts_w(tb + TMC_ACC0, tb + col + 16, da + 128 * k, id_g, 1u);
                    }
                    if (KEYS) {
                        const uint64_t db = sdesc_sw128(xb, BLK_X, 1024);
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
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const uint64_t oa = sdesc_sw128(own_a + b * BLK_O, 16, 1024), ka = sdesc_sw128(xa + b * BLK_X, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) mma_ss_w(tb + TMC_S, oa + 2 * k, ka + 2 * k, id_s, (b > 0 || k > 0) ? 1u : 0u);
            }
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const uint64_t ob = sdesc_sw128(own_b + b * BLK_O, 16, 1024), kb = sdesc_sw128(xb + b * BLK_X, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) mma_ss_w(tb + TMC_DP, ob + 2 * k, kb + 2 * k, id_s, (b > 0 || k > 0) ? 1u : 0u);
            }
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
        const float sl2 = kLog2eF * rsqrtf((float)D);  // log2(e) / sqrt(D)
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
                const float scale = a == 0 ? rsqrtf((float)D) : 1.f;  // 1/sqrt(D) on dq, dk
                float *out = a == 0 ? p.out0 : p.out1;
#pragma unroll
                for (int h = 0; h < D / 32; ++h) {
                    uint32_t v[32];
                    tmem_ld32(lanes + (a == 0 ? TMC_ACC0 : TMC_ACC1) + 32 * h, v);
                    tmem_wait_ld();
                    if (orow < T) {
                        float4 *dst = reinterpret_cast<float4 *>(out + row * D + 32 * h);
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

// ===========================================================================
// Memory (L2) part, one CTA per chunk of CM = 128 evictions e0 .. e0+L-1
// (local index i or s; the read of eviction e is at t = e + W).  With
// qt_s = q_{e0+W+s}, pw(n) = lam^n, sigma = sigmoid(g), A the chunk's start
// state and H the G passed back from the later chunks:
//   QK[s][j] = qt_s . k_j,  DV[s][j] = dy_s . v_j,
//   Mq[s][j] = pw(s-j) QK[s][j],  Md[s][j] = pw(s-j) DV[s][j]  (j <= s < L),
//   m_s  = pw(s+1) qt_s A + eta (Mq V)_s                     (the read)
//   dq_s = sigma (pw(s+1) dy_s A^T + eta (Md K)_s)
//   dk_i = eta (pw(L-i) H v_i + sigma (Md^T Qt)_i)
//   dv_i = eta (pw(L-i) k_i H + sigma (Mq^T dY)_i)
// and the partials of dlambda, deta, dg (the chunk's steps e of
// <G_e, A_{e-1}>, <G_e, k_e v_e^T> and the gate's sigma (1 - sigma) <dy, m>).
// Every product runs on the tensor cores: QK and DV into TMEM; Mq, Md as
// bf16 hi + lo in shared memory (read K-major for Mq V, Md K and MN-major for
// the transposed Md^T Qt, Mq^T dY); A and H as bf16 hi + lo; eight 64-column
// accumulators (state and in-chunk terms apart, as their row scales differ).
constexpr int CM = 128;
constexpr uint32_t MT_IN = CM * HDB * 2;           // 16 KB: a 128-row input tile
constexpr uint32_t MOFF_K = 0, MOFF_V = MT_IN, MOFF_Q = 2 * MT_IN, MOFF_D = 3 * MT_IN;
constexpr uint32_t MT_ST = HDB * HDB * 2;          // 8 KB: a 64 x 64 bf16 state part
constexpr uint32_t MOFF_AH = 4 * MT_IN;            // A hi, A lo, H hi, H lo
constexpr uint32_t MT_M = CM * CM * 2;             // 32 KB: 128 x 128 bf16 in two 64-column tiles
constexpr uint32_t MOFF_M = MOFF_AH + 4 * MT_ST;   // Mq hi, Mq lo, Md hi, Md lo
constexpr uint32_t MOFF_PW = MOFF_M + 4 * MT_M;    // pw(n), n = 0 .. CM + 1
constexpr uint32_t MOFF_RED = MOFF_PW + 136 * 4;   // 4 warps x 3 partials
constexpr uint32_t MOFF_BAR = MOFF_RED + 64;
constexpr uint32_t SMEM_MEM_TC = MOFF_BAR + 64 + 1024;
// TMEM: QK, DV (then free), the accumulators
constexpr uint32_t TMM_QK = 0, TMM_DV = 128;
constexpr uint32_t TMM_MA = 0, TMM_MI = 64, TMM_QA = 128, TMM_QI = 192, TMM_KH = 256, TMM_KI = 320,
                   TMM_VH = 384, TMM_VI = 448;

struct MemTcParams {
    const float *Ac, *Hc;  // [BH][nC][64][64]
    const float *lam, *eta, *g;
    float *gq, *gk, *gv;   // [BH][T][64], += this part
    float *part;           // [BH][nC][3]
    int T, W, H, E, nC;
    int *status;
    unsigned long long wait_ns;
};

// 8 bf16 pairs (16 values) of one row into a swizzled 128-byte-row tile.
__device__ __forceinline__ void st_row16(uint8_t *tile, int row, int col, const uint32_t *w) {
    *reinterpret_cast<uint4 *>(tile + sw128_offset(row, col)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4 *>(tile + sw128_offset(row, col + 8)) = make_uint4(w[4], w[5], w[6], w[7]);
}
// The 64 bf16 values of one row of a swizzled tile, as float32.
__device__ __forceinline__ void ld_row64(const uint8_t *tile, int row, float (&x)[64]) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint4 w = *reinterpret_cast<const uint4 *>(tile + sw128_offset(row, 8 * u));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[8 * u + 2 * e] = __uint_as_float(ws[e] << 16);
            x[8 * u + 2 * e + 1] = __uint_as_float(ws[e] & 0xffff0000u);
        }
    }
}
// += 64 float32 values into a global row (16-byte aligned).
__device__ __forceinline__ void add_row64(float *dst, const float (&x)[64]) {
    float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        float4 a = d4[u];
        a.x += x[4 * u];
        a.y += x[4 * u + 1];
        a.z += x[4 * u + 2];
        a.w += x[4 * u + 3];
        d4[u] = a;
    }
}
// 64 columns of one accumulator row (two 32-column loads).
__device__ __forceinline__ void ld_acc64(uint32_t taddr, float (&x)[64]) {
    uint32_t r[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        tmem_ld32(taddr + 32 * h, r);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) x[32 * h + c] = __uint_as_float(r[c]);
    }
}

__global__ void __launch_bounds__(kBwdTcThreads, 1)
    l2b_chunk_tc_kernel(const __grid_constant__ CUtensorMap t_k, const __grid_constant__ CUtensorMap t_v,
                        const __grid_constant__ CUtensorMap t_q, const __grid_constant__ CUtensorMap t_dy,
                        MemTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MOFF_BAR);
    uint64_t *in_full = bars, *s_full = bars + 1, *m_ready = bars + 2, *acc_full = bars + 3;
    uint64_t *mma_done = bars + 4;
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(bars + 5);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    float *pw = reinterpret_cast<float *>(sm + MOFF_PW);
    float *red = reinterpret_cast<float *>(sm + MOFF_RED);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int c = blockIdx.x, bh = blockIdx.y, h = bh % p.H;
    const int e0 = c * CM;
    const int L = min(CM, p.E - e0);

    if (tid == 0) {
        mbar_init(in_full, 1);
        mbar_init(s_full, 1);
        mbar_init(m_ready, 128);
        mbar_init(acc_full, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (tid == 0) {
            mbar_expect_tx(in_full, 4 * MT_IN);
            tma_load_3d(sm + MOFF_K, &t_k, in_full, 0, e0, bh);
            tma_load_3d(sm + MOFF_V, &t_v, in_full, 0, e0, bh);
            tma_load_3d(sm + MOFF_Q, &t_q, in_full, 0, e0 + p.W, bh);
            tma_load_3d(sm + MOFF_D, &t_dy, in_full, 0, e0 + p.W, bh);
            mbar_wait_drain(in_full, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t base = smem_u32(sm);
        const uint32_t sK = base + MOFF_K, sV = base + MOFF_V, sQ = base + MOFF_Q, sD = base + MOFF_D;
        const uint32_t sAH = base + MOFF_AH, sM = base + MOFF_M;
        const uint32_t id_n128 = idesc_bf16(128, 128, false, false);
        const uint32_t id_kk = idesc_bf16(128, 64, false, false);
        const uint32_t id_kmn = idesc_bf16(128, 64, false, true);
        const uint32_t id_mnmn = idesc_bf16(128, 64, true, true);
        bool ok = warp_wait_b(in_full, 0, abort, p.status, p.wait_ns);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_ss_w(tb + TMM_QK, sdesc_sw128(sQ, 16, 1024) + 2 * k, sdesc_sw128(sK, 16, 1024) + 2 * k,
                         id_n128, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_ss_w(tb + TMM_DV, sdesc_sw128(sD, 16, 1024) + 2 * k, sdesc_sw128(sV, 16, 1024) + 2 * k,
                         id_n128, k > 0);
            mma_commit_w(s_full);
            ok = warp_wait_b(m_ready, 0, abort, p.status, p.wait_ns);
        }
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t a_st = sAH + part * MT_ST, h_st = sAH + (2 + part) * MT_ST;
                const uint32_t mq = sM + part * MT_M, md = sM + (2 + part) * MT_M;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t acc = (part > 0 || k > 0) ? 1u : 0u;
                    // m (state): Qt A;  dq (state): dY A^T;  dk (state): V H^T;  dv (state): K H
                    mma_ss_w(tb + TMM_MA, sdesc_sw128(sQ, 16, 1024) + 2 * k,
                             sdesc_sw128(a_st, MT_ST, 1024) + 128 * k, id_kmn, acc);
                    mma_ss_w(tb + TMM_QA, sdesc_sw128(sD, 16, 1024) + 2 * k,
                             sdesc_sw128(a_st, 16, 1024) + 2 * k, id_kk, acc);
                    mma_ss_w(tb + TMM_KH, sdesc_sw128(sV, 16, 1024) + 2 * k,
                             sdesc_sw128(h_st, 16, 1024) + 2 * k, id_kk, acc);
                    mma_ss_w(tb + TMM_VH, sdesc_sw128(sK, 16, 1024) + 2 * k,
                             sdesc_sw128(h_st, MT_ST, 1024) + 128 * k, id_kmn, acc);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t acc = (part > 0 || k > 0) ? 1u : 0u;
                    const uint32_t kb = (k >> 2) * (MT_M / 2), kc = 2 * (k & 3);
                    // m (chunk): Mq V;  dq (chunk): Md K
                    mma_ss_w(tb + TMM_MI, sdesc_sw128(mq + kb, 16, 1024) + kc,
                             sdesc_sw128(sV, MT_IN, 1024) + 128 * k, id_kmn, acc);
                    mma_ss_w(tb + TMM_QI, sdesc_sw128(md + kb, 16, 1024) + kc,
                             sdesc_sw128(sK, MT_IN, 1024) + 128 * k, id_kmn, acc);
                    // dk (chunk): Md^T Qt;  dv (chunk): Mq^T dY  (A read MN-major)
                    mma_ss_w(tb + TMM_KI, sdesc_sw128(md, MT_M / 2, 1024) + 128 * k,
                             sdesc_sw128(sQ, MT_IN, 1024) + 128 * k, id_mnmn, acc);
                    mma_ss_w(tb + TMM_VI, sdesc_sw128(mq, MT_M / 2, 1024) + 128 * k,
                             sdesc_sw128(sD, MT_IN, 1024) + 128 * k, id_mnmn, acc);
                }
            }
            mma_commit_w(acc_full);
        }
        mma_commit_w(mma_done);
        mbar_wait_drain(mma_done, 0);
    } else {
        // ------------------------------------------------------------ element-wise side + epilogue
        const int q4 = warp & 3;
        const int x = 32 * q4 + (tid & 31);  // chunk row: s (reads) or i (evictions)
        const uint32_t lanes = tb + ((uint32_t)(32 * q4) << 16);
        const float lam = p.lam[h], eta = p.eta[h];
        const float sg = 1.f / (1.f + expf(-p.g[h]));
        {
            const double l2l = log2((double)lam);
            for (int n = x; n <= CM + 1; n += 128) pw[n] = n == 0 ? 1.f : (float)exp2((double)n * l2l);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        float p_lam = 0.f, p_eta = 0.f, p_g = 0.f;
        // A and H as bf16 hi + lo: thread x takes row x / 2, columns 32 (x % 2) ..
        {
            const int r = x >> 1, c0 = 32 * (x & 1);
            const size_t off = ((size_t)bh * p.nC + c) * HDB * HDB + (size_t)r * HDB + c0;
            const float4 *a4 = reinterpret_cast<const float4 *>(p.Ac + off);
            const float4 *h4 = reinterpret_cast<const float4 *>(p.Hc + off);
            float ah = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {  // 8 columns at a time
                const float4 a0 = a4[2 * u], a1 = a4[2 * u + 1], g0 = h4[2 * u], g1 = h4[2 * u + 1];
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float hv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                uint32_t ahi[4], alo[4], hhi[4], hlo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    split_pair(av[2 * e], av[2 * e + 1], ahi[e], alo[e]);
                    split_pair(hv[2 * e], hv[2 * e + 1], hhi[e], hlo[e]);
                    ah = fmaf(av[2 * e], hv[2 * e], ah);
                    ah = fmaf(av[2 * e + 1], hv[2 * e + 1], ah);
                }
                const int col = c0 + 8 * u;
                *reinterpret_cast<uint4 *>(sm + MOFF_AH + sw128_offset(r, col)) = make_uint4(ahi[0], ahi[1], ahi[2], ahi[3]);
                *reinterpret_cast<uint4 *>(sm + MOFF_AH + MT_ST + sw128_offset(r, col)) = make_uint4(alo[0], alo[1], alo[2], alo[3]);
                *reinterpret_cast<uint4 *>(sm + MOFF_AH + 2 * MT_ST + sw128_offset(r, col)) = make_uint4(hhi[0], hhi[1], hhi[2], hhi[3]);
                *reinterpret_cast<uint4 *>(sm + MOFF_AH + 3 * MT_ST + sw128_offset(r, col)) = make_uint4(hlo[0], hlo[1], hlo[2], hlo[3]);
            }
            p_lam = (float)L * pw[L] * ah;  // <H, A> term
        }
        bool ok = warp_wait_b(s_full, 0, abort, p.status, p.wait_ns);
        if (ok) {
            tc_fence_after();
            // Mq, Md of row s = x, 32 columns j at a time
            const int s = x;
            const bool row_in = s < L;
#pragma unroll 1
            for (int jb = 0; jb < 4; ++jb) {
                uint32_t qk[32], dv[32];
                tmem_ld32(lanes + TMM_QK + 32 * jb, qk);
                tmem_ld32(lanes + TMM_DV + 32 * jb, dv);
                tmem_wait_ld();
                uint32_t mqh[16], mql[16], mdh[16], mdl[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float mqv[2], mdv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int j = 32 * jb + 2 * e + u;
                        const float a = __uint_as_float(qk[2 * e + u]), b = __uint_as_float(dv[2 * e + u]);
                        const bool in = row_in && j <= s;
                        const float w = in ? pw[s - j] : 0.f;
                        mqv[u] = w * a;
                        mdv[u] = w * b;
                        // pair term of dlambda: eta sigma (s-j) pw(s-1-j) QK DV, j < s
                        if (in && j < s) p_lam = fmaf((float)(s - j) * pw[s - 1 - j] * a, b * eta * sg, p_lam);
                    }
                    split_pair(mqv[0], mqv[1], mqh[e], mql[e]);
                    split_pair(mdv[0], mdv[1], mdh[e], mdl[e]);
                }
                uint8_t *blk = sm + MOFF_M + (jb >> 1) * (MT_M / 2);
                const int col = 32 * (jb & 1);
                st_row16(blk, s, col, mqh);
                st_row16(blk, s, col + 16, mqh + 8);
                st_row16(blk + MT_M, s, col, mql);
                st_row16(blk + MT_M, s, col + 16, mql + 8);
                st_row16(blk + 2 * MT_M, s, col, mdh);
                st_row16(blk + 2 * MT_M, s, col + 16, mdh + 8);
                st_row16(blk + 3 * MT_M, s, col, mdl);
                st_row16(blk + 3 * MT_M, s, col + 16, mdl + 8);
            }
        }
        // the A / H parts and Mq, Md go to the tensor cores (every thread
        // arrives, also after a failed wait, so that the MMA side's count holds)
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(m_ready);
        if (ok) ok = warp_wait_b(acc_full, 0, abort, p.status, p.wait_ns);
        if (ok) {
            tc_fence_after();
            const bool valid = x < L;
            float u[64], w[64], row[64];
            // read side, s = x: m (for dg and dlambda) and dq
            ld_row64(sm + MOFF_D, x, row);  // dy_s
            ld_acc64(lanes + TMM_MA, u);
            ld_acc64(lanes + TMM_MI, w);
            {
                float dm = 0.f, da = 0.f;
                const float ps1 = pw[min(x + 1, CM + 1)];
#pragma unroll
                for (int cc = 0; cc < 64; ++cc) {
                    dm = fmaf(row[cc], fmaf(ps1, u[cc], eta * w[cc]), dm);
                    da = fmaf(row[cc], u[cc], da);
                }
                if (valid) {
                    p_g = fmaf(sg, dm, p_g);
                    p_lam = fmaf((float)(x + 1) * pw[x] * sg, da, p_lam);
                }
            }
            ld_acc64(lanes + TMM_QA, u);
            ld_acc64(lanes + TMM_QI, w);
            if (valid) {
                const float ps1 = pw[x + 1];
#pragma unroll
                for (int cc = 0; cc < 64; ++cc) u[cc] = sg * fmaf(ps1, u[cc], eta * w[cc]);
                add_row64(p.gq + ((size_t)bh * p.T + e0 + p.W + x) * HDB, u);
            }
            // eviction side, i = x: dk (and the deta, dlambda terms), dv
            ld_row64(sm + MOFF_K, x, row);  // k_i
            ld_acc64(lanes + TMM_KH, u);
            ld_acc64(lanes + TMM_KI, w);
            if (valid) {
                const float pli = pw[L - x];
                float ke = 0.f, kh = 0.f;
#pragma unroll
                for (int cc = 0; cc < 64; ++cc) {
                    const float dkr = fmaf(pli, u[cc], sg * w[cc]);  // dk_i / eta
                    ke = fmaf(row[cc], dkr, ke);
                    kh = fmaf(row[cc], u[cc], kh);
                    w[cc] = eta * dkr;
                }
                p_eta += ke;
                p_lam = fmaf(eta * (float)(L - 1 - x) * pw[L - 1 - x], kh, p_lam);
                add_row64(p.gk + ((size_t)bh * p.T + e0 + x) * HDB, w);
            }
            ld_acc64(lanes + TMM_VH, u);
            ld_acc64(lanes + TMM_VI, w);
            if (valid) {
                const float pli = pw[L - x];
#pragma unroll
                for (int cc = 0; cc < 64; ++cc) u[cc] = eta * fmaf(pli, u[cc], sg * w[cc]);
                add_row64(p.gv + ((size_t)bh * p.T + e0 + x) * HDB, u);
            }
        }
        // fixed-order sum of the partials over the 128 rows
        p_g *= 1.f - sg;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            p_lam += __shfl_xor_sync(0xffffffffu, p_lam, o);
            p_eta += __shfl_xor_sync(0xffffffffu, p_eta, o);
            p_g += __shfl_xor_sync(0xffffffffu, p_g, o);
        }
        if ((tid & 31) == 0) {
            red[3 * q4] = p_lam;
            red[3 * q4 + 1] = p_eta;
            red[3 * q4 + 2] = p_g;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (x < 3) {
            const float v = ((red[x] + red[3 + x]) + red[6 + x]) + red[9 + x];
            p.part[((size_t)bh * p.nC + c) * 3 + x] = ok ? v : 0.f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, 512);
}

// Per chunk, the two sums the scan over chunks needs: the state increment
// dA_c = eta K^T diag(pw(L-1-i)) V and the summary X_c = sigma Qt^T
// diag(pw(s)) dY.  Both are the diagonal 64 x 64 blocks of one M = 128
// product [K^T; Qt^T] [diag(w1) V | diag(w2) dY] (A read MN-major from the
// K and Qt tiles, B built as bf16 hi + lo by the element-wise warps).
constexpr uint32_t SOFF_KQ = 0;                   // K tile, Qt tile (the A operand's two M blocks)
constexpr uint32_t SOFF_B = 2 * MT_IN;            // B hi (w1 V tile, w2 dY tile), B lo likewise
constexpr uint32_t SOFF_PW = SOFF_B + 4 * MT_IN;  // pw(n), n = 0 .. CM + 1
constexpr uint32_t SOFF_BAR = SOFF_PW + 136 * 4;
constexpr uint32_t SMEM_SUM_TC = SOFF_BAR + 64 + 1024;

struct SumTcParams {
    const __nv_bfloat16 *v, *dy;  // [BH][T][64]
    const float *lam, *eta, *g;
    float *Ac, *Hc;               // [BH][nC][64][64]
    int T, W, H, E, nC;
    int *status;
    unsigned long long wait_ns;
};

// Row `row` of a [BH*T][64] bf16 tensor times w, as bf16 hi + lo pairs into
// row x of two swizzled tiles (zeros when w == 0: the row is not read).
__device__ __forceinline__ void scaled_row_split(const __nv_bfloat16 *src, size_t row, float w, uint8_t *hi_tile,
                                                 uint8_t *lo_tile, int x) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src + row * HDB);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint4 a = w != 0.f ? s4[u] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t ws[4] = {a.x, a.y, a.z, a.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            split_pair(w * __uint_as_float(ws[e] << 16), w * __uint_as_float(ws[e] & 0xffff0000u), hi[e], lo[e]);
        *reinterpret_cast<uint4 *>(hi_tile + sw128_offset(x, 8 * u)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(lo_tile + sw128_offset(x, 8 * u)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

__global__ void __launch_bounds__(kBwdTcThreads, 2)
    l2b_sums_tc_kernel(const __grid_constant__ CUtensorMap t_k, const __grid_constant__ CUtensorMap t_q,
                       SumTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SOFF_BAR);
    uint64_t *in_full = bars, *b_ready = bars + 1, *acc_full = bars + 2, *mma_done = bars + 3;
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(bars + 4);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    float *pw = reinterpret_cast<float *>(sm + SOFF_PW);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int c = blockIdx.x, bh = blockIdx.y, h = bh % p.H;
    const int e0 = c * CM;
    const int L = min(CM, p.E - e0);

    if (tid == 0) {
        mbar_init(in_full, 1);
        mbar_init(b_ready, 128);
        mbar_init(acc_full, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_base;

    if (warp == 0) {
        if (tid == 0) {
            mbar_expect_tx(in_full, 2 * MT_IN);
            tma_load_3d(sm + SOFF_KQ, &t_k, in_full, 0, e0, bh);
            tma_load_3d(sm + SOFF_KQ + MT_IN, &t_q, in_full, 0, e0 + p.W, bh);
            mbar_wait_drain(in_full, 0);
        }
    } else if (warp == 1) {
        const uint32_t sA = smem_u32(sm + SOFF_KQ), sB = smem_u32(sm + SOFF_B);
        const uint32_t id = idesc_bf16(128, 128, true, true);
        bool ok = warp_wait_b(in_full, 0, abort, p.status, p.wait_ns) &&
                  warp_wait_b(b_ready, 0, abort, p.status, p.wait_ns);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ss_w(tb, sdesc_sw128(sA, MT_IN, 1024) + 128 * k,
                             sdesc_sw128(sB + part * 2 * MT_IN, MT_IN, 1024) + 128 * k, id,
                             (part > 0 || k > 0) ? 1u : 0u);
            mma_commit_w(acc_full);
        }
        mma_commit_w(mma_done);
        mbar_wait_drain(mma_done, 0);
    } else {
        const int q4 = warp & 3;
        const int x = 32 * q4 + (tid & 31);
        const uint32_t lanes = tb + ((uint32_t)(32 * q4) << 16);
        const float lam = p.lam[h], eta = p.eta[h];
        const float sg = 1.f / (1.f + expf(-p.g[h]));
        {
            const double l2l = log2((double)lam);
            for (int n = x; n <= CM + 1; n += 128) pw[n] = n == 0 ? 1.f : (float)exp2((double)n * l2l);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // B: row x of w1 V (w1 = pw(L-1-x)) and of w2 dY (w2 = pw(x)), zero past L
        const bool in = x < L;
        const size_t row_v = (size_t)bh * p.T + e0 + x, row_d = row_v + p.W;
        scaled_row_split(p.v, row_v, in ? pw[L - 1 - x] : 0.f, sm + SOFF_B, sm + SOFF_B + 2 * MT_IN, x);
        scaled_row_split(p.dy, row_d, in ? pw[x] : 0.f, sm + SOFF_B + MT_IN, sm + SOFF_B + 3 * MT_IN, x);
        fence_async_smem();
        mbar_arrive(b_ready);
        if (warp_wait_b(acc_full, 0, abort, p.status, p.wait_ns)) {
            tc_fence_after();
            // lanes 0..63: rows of K^T (dA, columns 0..63); 64..127: rows of Qt^T (X, columns 64..127)
            const bool lower = x < 64;
            const int r = lower ? x : x - 64;
            const float scale = lower ? eta : sg;
            float *dst = (lower ? p.Ac : p.Hc) + (((size_t)bh * p.nC + c) * HDB + r) * HDB;
            uint32_t v[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                tmem_ld32(lanes + (lower ? 0u : 64u) + 32 * hh, v);
                tmem_wait_ld();
                float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * hh);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    d4[u] = make_float4(scale * __uint_as_float(v[4 * u]), scale * __uint_as_float(v[4 * u + 1]),
                                        scale * __uint_as_float(v[4 * u + 2]), scale * __uint_as_float(v[4 * u + 3]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, 128);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [BH][T][64] bf16 -> 3D map, boxes of 64 x rows x 1 with the 128-byte swizzle;
// rows past T read as zero.
bool rows_map(CUtensorMap *m, const void *base, int T, int BH, int rows, int D = HDB) {
    EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
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
    return d.dtype == TC_BF16 && d.dk == d.dv && (d.dk == 64 || d.dk == 128) && d.T >= 1 &&
           d.T < (int64_t(1) << 30) && d.B * d.H <= 65535 && tensor_map_encoder() != nullptr;
}

bool backward_memory_tc_supported(const tc_prefill_desc &d) {
    return backward_window_tc_supported(d) && d.dk == HDB;
}

int64_t backward_stat_stride(int64_t T) { return (T + BX - 1) / BX * BX; }

template <int NB>
cudaError_t launch_window_tc_t(const tc_prefill_desc &d, const void *q, const void *k, const void *v,
                               const void *dy, float *dq, float *dk, float *dv, float *lse, float *Dt,
                               int *status, unsigned long long wait_ns, cudaStream_t s) {
    using Cf = BwdCfg<NB>;
    constexpr int D = Cf::D;
    const int T = (int)d.T, BH = (int)(d.B * d.H);
    const int Tp = (int)backward_stat_stride(d.T);
    CUtensorMap mq_o, mdy_o, mk_x, mv_x, mk_o, mv_o, mq_x, mdy_x, mlse, mD;
    if (!rows_map(&mq_o, q, T, BH, BO, D) || !rows_map(&mdy_o, dy, T, BH, BO, D) ||
        !rows_map(&mk_x, k, T, BH, BX, D) || !rows_map(&mv_x, v, T, BH, BX, D) ||
        !rows_map(&mk_o, k, T, BH, BO, D) || !rows_map(&mv_o, v, T, BH, BO, D) ||
        !rows_map(&mq_x, q, T, BH, BX, D) || !rows_map(&mdy_x, dy, T, BH, BX, D) ||
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
    cudaError_t e = cudaFuncSetAttribute(bwd_window_tc_kernel<false, NB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cf::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_window_tc_kernel<true, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Cf::SMEM);
    if (e != cudaSuccess) return e;
    p.out0 = dq;
    p.out1 = nullptr;
    bwd_window_tc_kernel<false, NB><<<grid, kBwdTcThreads, Cf::SMEM, s>>>(mq_o, mdy_o, mk_x, mv_x, mlse, mD, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    p.out0 = dk;
    p.out1 = dv;
    bwd_window_tc_kernel<true, NB><<<grid, kBwdTcThreads, Cf::SMEM, s>>>(mk_o, mv_o, mq_x, mdy_x, mlse, mD, p);
    return cudaGetLastError();
}

cudaError_t launch_backward_window_tc(const tc_prefill_desc &d, const void *q, const void *k,
                                      const void *v, const void *dy, float *dq, float *dk, float *dv,
                                      float *lse, float *Dt, int *status, unsigned long long wait_ns,
                                      cudaStream_t s) {
    return d.dk == 128 ? launch_window_tc_t<2>(d, q, k, v, dy, dq, dk, dv, lse, Dt, status, wait_ns, s)
                       : launch_window_tc_t<1>(d, q, k, v, dy, dq, dk, dv, lse, Dt, status, wait_ns, s);
}

cudaError_t launch_backward_chunks_tc(const tc_prefill_desc &d, const void *q, const void *k,
                                      const void *v, const void *dy, const float *lam,
                                      const float *eta, const float *g, const float *Ac,
                                      const float *Hc, float *dq, float *dk, float *dv, float *part,
                                      int *status, unsigned long long wait_ns, cudaStream_t s) {
    const int T = (int)d.T, BH = (int)(d.B * d.H);
    const int E = d.T > d.W ? (int)(d.T - d.W) : 0;
    const int nC = (E + CM - 1) / CM;
    if (nC == 0) return cudaSuccess;
    CUtensorMap mk, mv, mq, mdy;
    if (!rows_map(&mk, k, T, BH, CM) || !rows_map(&mv, v, T, BH, CM) || !rows_map(&mq, q, T, BH, CM) ||
        !rows_map(&mdy, dy, T, BH, CM))
        return cudaErrorInvalidValue;
    MemTcParams p{};
    p.Ac = Ac;
    p.Hc = Hc;
    p.lam = lam;
    p.eta = eta;
    p.g = g;
    p.gq = dq;
    p.gk = dk;
    p.gv = dv;
    p.part = part;
    p.T = T;
    p.W = (int)d.W;
    p.H = (int)d.H;
    p.E = E;
    p.nC = nC;
    p.status = status;
    p.wait_ns = wait_ns;
    cudaError_t e = cudaFuncSetAttribute(l2b_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_MEM_TC);
    if (e != cudaSuccess) return e;
    l2b_chunk_tc_kernel<<<dim3((unsigned)nC, (unsigned)BH), kBwdTcThreads, SMEM_MEM_TC, s>>>(mk, mv, mq, mdy, p);
    return cudaGetLastError();
}

cudaError_t launch_backward_sums_tc(const tc_prefill_desc &d, const void *q, const void *k, const void *v,
                                    const void *dy, const float *lam, const float *eta, const float *g,
                                    float *Ac, float *Hc, int *status, unsigned long long wait_ns,
                                    cudaStream_t s) {
    const int T = (int)d.T, BH = (int)(d.B * d.H);
    const int E = d.T > d.W ? (int)(d.T - d.W) : 0;
    const int nC = (E + CM - 1) / CM;
    if (nC == 0) return cudaSuccess;
    CUtensorMap mk, mq;
    if (!rows_map(&mk, k, T, BH, CM) || !rows_map(&mq, q, T, BH, CM)) return cudaErrorInvalidValue;
    SumTcParams p{};
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.dy = static_cast<const __nv_bfloat16 *>(dy);
    p.lam = lam;
    p.eta = eta;
    p.g = g;
    p.Ac = Ac;
    p.Hc = Hc;
    p.T = T;
    p.W = (int)d.W;
    p.H = (int)d.H;
    p.E = E;
    p.nC = nC;
    p.status = status;
    p.wait_ns = wait_ns;
    cudaError_t e = cudaFuncSetAttribute(l2b_sums_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_SUM_TC);
    if (e != cudaSuccess) return e;
    l2b_sums_tc_kernel<<<dim3((unsigned)nC, (unsigned)BH), kBwdTcThreads, SMEM_SUM_TC, s>>>(mk, mq, p);
    return cudaGetLastError();
}

}  // namespace tc
