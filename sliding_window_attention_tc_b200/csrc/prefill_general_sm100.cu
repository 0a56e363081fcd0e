// The general tensor-core prefill: bf16 with d_k = d_v = D in {64, 128}, any
// window W >= 1, any T, and continuations with any halo (0 < t0 < W
// included).  It takes every fixed-length call by default (it measured faster
// than the fused prefill_main_kernel at that kernel's shapes too); the fused
// kernel keeps the variable-length calls at its shapes.
//
// "Tensor Cache: Eviction-conditioned Associative Memory for Transformers":
// the window read of §3.1 eq. (1) and the memory of §3.2 / Fig. 2 (write on
// eviction, A <- lam A + eta k v^T; read m = q A; y = y_local + sigma(g) m),
// the memory in the chunked form of the abstract and §2, one chunk per block
// of 128 new rows: the evictions that block's reads take in.  Four kernels,
// all but the copy and the scan on tcgen05:
//   gen_combine_kernel   halo + new keys / values into one sequence (only
//                        when continuing with a halo);
//   gen_sums_kernel      per chunk dA_c = eta K^T diag(lam^(L-1-i)) V, one
//                        M = 128 product (two chunks side by side for D = 64);
//   gen_scan_kernel      A_c = chunk start states from A_init, and A_final;
//   gen_window_kernel    the window softmax in one pass (online rescaling of
//                        the output accumulator in TMEM), the block's reads
//                        m = lam^(i+1) q A_c + the in-chunk terms from the same
//                        scores, and the fusion y = y_local + sigma(g) m.
// Positions are those of the combined sequence (halo first): token tau is a
// new row when tau >= n_halo, evictions are tau = 0 .. n_halo + T - W - 1 and
// A_init holds every eviction before the combined sequence.  float32 values
// that enter the tensor cores (the states, the decayed in-chunk scores) are
// split into bf16 hi + lo pairs; P of the window softmax is bf16, as in the
// fused kernel.

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

constexpr int CG = 128;                  // evictions per chunk, query rows per window CTA
constexpr int GX = 64;                   // key rows per window tile
constexpr int kGThreads = 192;           // warp 0 TMA, warp 1 MMA, warps 2-5 element-wise
constexpr uint32_t BLK128 = 128 * 128;   // a 128-row x 64-column bf16 block (16 KB)
constexpr uint32_t BLK64 = 64 * 128;     // a 64-row x 64-column bf16 block (8 KB)
constexpr float kLog2eG = 1.4426950408889634f;

struct GenParams {
    const __nv_bfloat16 *q, *k, *v;  // q: [BH][T][D] new rows; k, v: the combined sequence
    __nv_bfloat16 *y;
    float *mrow;                     // [BH][T][D] float32 reads (null: none)
    float *dA;                       // [BH][nC][D][D]: per-chunk increments
    __nv_bfloat16 *ab;               // [BH][nC][2][D][D]: chunk start states as bf16 hi, lo
    float *A_final;
    const float *A_init;
    const float *lam, *eta, *g;
    int T, Tc, n_halo, W, H, E, nC;  // new rows, combined rows, halo, window, heads, evictions, chunks
    // variable-length calls: sequence b = packed rows cu[b] .. cu[b+1]-1 of
    // [total][H][D] q, k, v, y (and m rows); T is then the longest length
    // and E, nC the largest eviction and chunk counts.  Null: fixed length.
    const int64_t *cu;
    int total;
    int *status;
    unsigned long long wait_ns;
};

// One (sequence, head) row of work: its row origin and length in the tensors
// (fixed length: rows of [BH][Tc] / [BH][T]; packed: rows of [total][H]).
struct GSeq {
    int bh, h, row0, T, Tc, E, nC;
    bool packed;
};
__device__ __forceinline__ GSeq gseq(const GenParams &p, int bh) {
    GSeq s;
    s.bh = bh;
    s.h = bh % p.H;
    s.packed = p.cu != nullptr;
    if (!s.packed) {
        s.row0 = 0;
        s.T = p.T;
        s.Tc = p.Tc;
    } else {
        const int64_t a = p.cu[bh / p.H], e = p.cu[bh / p.H + 1];
        const bool ok = a >= 0 && e >= a && e <= p.total && e - a <= p.T;
        if (!ok && s.h == 0 && threadIdx.x == 0 && blockIdx.x == 0) report(p.status, 5);
        s.row0 = ok ? (int)a : 0;
        s.T = s.Tc = ok ? (int)(e - a) : 0;
    }
    s.E = s.Tc > p.W ? s.Tc - p.W : 0;
    s.nC = (s.T + CG - 1) / CG;  // one chunk per block of 128 new rows
    return s;
}

// Chunk b holds the evictions that the reads of query block b (new rows
// 128 b .. 128 b + 127, combined positions n_halo + 128 b + r) take in:
// [e_lo, e_hi), possibly empty.  Consecutive chunks are adjacent, and since
// the halo is at most W long the first starts at eviction 0.
__device__ __forceinline__ void chunk_range(const GenParams &p, const GSeq &s, int b, int &e_lo, int &e_hi) {
    const int a = p.n_halo + CG * b - p.W;
    e_lo = max(0, a);
    e_hi = max(e_lo, min(s.E, a + CG));
}
// Element offset of row `row` (of the combined sequence for k and v, else of the
// new rows) of a [.][D] tensor; rows_fixed is the row count of the fixed layout.
__device__ __forceinline__ size_t grow(const GSeq &s, int row, int rows_fixed, int H, int D) {
    return s.packed ? ((size_t)(s.row0 + row) * H + s.h) * D : ((size_t)s.bh * rows_fixed + row) * D;
}

__device__ __forceinline__ bool gwait(uint64_t *bar, uint32_t parity, volatile int *abort, const GenParams &p) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, p.status, p.wait_ns));
}
__device__ __forceinline__ float gex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void gsplit(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16(x0, x1);
    lo = pack_bf16(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xffff0000u));
}
// lam^n, n = 0 .. n_max, by the calling 128 threads (index x)
__device__ __forceinline__ void gpowers(float *pw, int n_max, float lam, int x) {
    const double l2l = log2((double)lam);
    for (int n = x; n <= n_max; n += 128) pw[n] = n == 0 ? 1.f : (float)exp2((double)n * l2l);
}
__device__ __forceinline__ void gbar128() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// lam^n (n >= 0) by binary powering in double, rounded once to float
__device__ __forceinline__ float gpow(float lam, int n) {
    double r = 1.0, b = (double)lam;
    for (; n > 0; n >>= 1) {
        if (n & 1) r *= b;
        b *= b;
    }
    return (float)r;
}

// How the window 0 <= tau - j < W cuts a 64-key tile, for all 32 rows of a
// warp at once: every column inside (no per-column masks), none inside (P =
// 0, no exponentials), or masked column by column.
enum { kTileFull = 0, kTileMasked = 1, kTileNone = 2 };
// O is rescaled only when a row's max grows by more than 2^8 over the max its
// P values are taken against, so P <= 2^8 (exact in bf16's float32 range)
// and most tiles skip the rescale and its wait for the previous P V.
constexpr float kRescaleG = 8.f;
// eta lam^d table for the reads' weights, zero-padded: entry 128 + d holds
// eta lam^d for 0 <= d < 128 and 0 for d < 0 (and for d >= 128, which only
// the columns before the chunk reach, and those are masked)
constexpr int kEpw = 384;

__device__ __forceinline__ int tile_kind(int base, uint32_t wlim) {
    // column c is in the window iff 0 <= base - c < wlim, c in [0, GX)
    if (__all_sync(0xffffffffu, wlim != 0u && base >= GX - 1 && base < (int)wlim)) return kTileFull;
    if (__all_sync(0xffffffffu, wlim == 0u || base < 0 || base - (GX - 1) >= (int)wlim)) return kTileNone;
    return kTileMasked;
}

// Row max of the raw scores over the window columns (-inf if none), as a tree.
template <bool MASK>
__device__ __forceinline__ float tile_max(const float (&s)[GX], int base, uint32_t wlim) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = -INFINITY;
#pragma unroll
    for (int c = 0; c < GX; c += 2) {
        const float a = (!MASK || (uint32_t)(base - c) < wlim) ? s[c] : -INFINITY;
        const float b = (!MASK || (uint32_t)(base - c - 1) < wlim) ? s[c + 1] : -INFINITY;
        m[(c >> 1) & 7] = fmax3(m[(c >> 1) & 7], a, b);
    }
    return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// P = exp2(s sl2 - m) on the window columns (0 elsewhere), bf16 pairs into
// the P columns of the score buffer (keys 32 h .. 32 h + 31 at column 32 h);
// returns the row sum of P.
template <bool MASK>
__device__ __forceinline__ float tile_p(const float (&s)[GX], int base, uint32_t wlim, float sl2, float m,
                                        uint32_t sbuf) {
    uint64_t acc[2] = {0ull, 0ull};  // (0.f, 0.f) pairs
    const uint64_t sl2p = f2pack(sl2, sl2), negm = f2pack(-m, -m);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int c = 32 * h + 2 * e;
            float x0, x1;
            ffma2(x0, x1, s[c], s[c + 1], sl2p, negm);
            if (MASK) {
                x0 = (uint32_t)(base - c) < wlim ? x0 : -INFINITY;
                x1 = (uint32_t)(base - c - 1) < wlim ? x1 : -INFINITY;
            }
            const float p0 = gex2(x0), p1 = gex2(x1);
            fadd2_acc(acc[e & 1], p0, p1);
            pk[e] = pack_bf16(p0, p1);
        }
        tmem_st16(sbuf + 32 * h, pk);
    }
    float a0, a1, b0, b1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc[0]));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(acc[1]));
    return (a0 + b0) + (a1 + b1);
}

// P' = eta lam^(off - c) s for off - c >= 0 (w[-c] from the padded table) and
// c >= cmin, bf16 pairs into the P' columns (keys 32 h .. at column 32 h + 16).
template <bool CMIN>
__device__ __forceinline__ void tile_plin(const float (&s)[GX], const float *w, int cmin, uint32_t sbuf) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int c = 32 * h + 2 * e;
            float w0 = w[-c], w1 = w[-c - 1];
            if (CMIN) {
                w0 = c >= cmin ? w0 : 0.f;
                w1 = c + 1 >= cmin ? w1 : 0.f;
            }
            pk[e] = pack_bf16(w0 * s[c], w1 * s[c + 1]);
        }
        tmem_st16(sbuf + 32 * h + 16, pk);
    }
}

// rows [row, row + rows) of a [.][D] map as NB column blocks of 64: maps
// (D, rows, BH) for fixed lengths, (D, H, total) for packed sequences
template <int NB>
__device__ __forceinline__ void tma_rows_nb(uint8_t *dst, const CUtensorMap *m, uint64_t *bar, int row,
                                            const GSeq &sq, uint32_t blk) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        if (sq.packed)
            tma_load_3d(dst + b * blk, m, bar, 64 * b, sq.h, sq.row0 + row);
        else
            tma_load_3d(dst + b * blk, m, bar, 64 * b, row, sq.bh);
    }
}

// ===========================================================================
// Window part, and with it the memory's reads.  A CTA owns 128 new query rows
// (TMEM lanes, query block b); 64-row key tiles stream through NS stages.
// Scores have two TMEM buffers: S of tile n+1 is issued before P V of tile
// n, so the softmax warpgroup finds the next scores ready when it finishes a
// tile.  Per tile it takes the row max over the band mask 0 <= tau - j < W,
// rescales O in TMEM when the max grew (after waiting for the previous P V,
// which a per-tile commit reports), writes P = exp2(s - m) as bf16 over S,
// and O += P V runs with P as the TMEM operand.
// With the memory (dA set, no m rows): the reads of block b take in chunk b's
// evictions [e_lo, e_hi) (the keys just left of the window) and the start
// state A_b, m_r = lam^(tau-W-e_lo+1) q_r A_b + sum_{e_lo <= j <= tau-W}
// eta lam^(tau-W-j) <q_r, k_j> v_j.  The key tiles then start at e_lo, the
// second term is P' V with P' = eta lam^(tau-W-j) s from the same scores
// (written beside P in the score buffer, accumulated in its own TMEM
// columns), and the first is one more MMA after the last tile, Q A_b with A_b
// as bf16 hi + lo in shared memory.  Score buffer layout (bf16 pairs, 64
// keys): [P keys 0-31 | P' keys 0-31 | P keys 32-63 | P' keys 32-63].
template <int NB>
struct WinCfg {
    static constexpr int D = 64 * NB;
    static constexpr int NS = NB == 1 ? 4 : 3;
    static constexpr uint32_t Q_B = NB * BLK128;
    static constexpr uint32_t X_B = NB * BLK64;   // one K or V tile
    static constexpr uint32_t ST_BLK = D * 128;   // D rows x 64 columns of A_b
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_X = Q_B;         // NS x (K tile, V tile)
    static constexpr uint32_t OFF_A = OFF_X + NS * 2 * X_B;  // A_b hi: NB blocks, lo: NB blocks
    static constexpr uint32_t OFF_PW = OFF_A + 2 * NB * ST_BLK;  // lam^n, n = 0 .. 128
    static constexpr uint32_t OFF_EPW = OFF_PW + 136 * 4;         // padded eta lam^d table
    static constexpr uint32_t OFF_BAR = OFF_EPW + kEpw * 4;
    static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;  // (9 + 2 NS) barriers, TMEM address, abort flag
    // two 64-column score buffers, O, the reads' accumulator (P' V, then + Q A_b
    // lands in the score buffers' columns after the last tile)
    static constexpr uint32_t TM_S = 0, TM_O = 128, TM_MI = 128 + D, COLS = NB == 1 ? 256 : 512;
};

template <int NB>
__global__ void __launch_bounds__(kGThreads, NB == 1 ? 2 : 1)
    gen_window_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tab,
                      GenParams p) {
    using C = WinCfg<NB>;
    constexpr int D = C::D, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *q_full = bars, *x_full = bars + 1, *x_empty = x_full + NS, *s_full = x_empty + NS;
    uint64_t *p_ready = s_full + 2, *o_done = p_ready + 2, *o_full = o_done + 1, *mma_done = o_full + 1;
    uint64_t *a_ready = mma_done + 1;
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(a_ready + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    float *pw = reinterpret_cast<float *>(sm + C::OFF_PW);
    float *epw = reinterpret_cast<float *>(sm + C::OFF_EPW);

    const int tid = threadIdx.x, warp = tid >> 5;
    const GSeq sq = gseq(p, blockIdx.y);
    const int t0 = blockIdx.x * CG;           // first new row
    if (t0 >= sq.T) return;                   // past this sequence (variable-length calls)
    const int tau0 = p.n_halo + t0;           // its combined position
    // the memory's reads of this block: chunk b = blockIdx.x
    const bool mem = p.dA != nullptr && p.mrow == nullptr;
    int e_lo = 0, e_hi = 0;
    if (mem) chunk_range(p, sq, blockIdx.x, e_lo, e_hi);
    const bool reads = mem && e_hi > e_lo;
    const int lo = reads ? e_lo : max(0, tau0 - p.W + 1), hi = min(sq.Tc - 1, tau0 + CG - 1);
    const int xs = lo & ~(GX - 1);
    const int N = (hi - xs) / GX + 1;
    // key tiles holding evictions of the chunk (CTA-uniform)
    auto tile_reads = [&](int n) { return reads && xs + GX * n < e_hi && xs + GX * n + GX > e_lo; };

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_ready[b], 4);
        }
        mbar_init(o_done, 1);
        mbar_init(o_full, 1);
        mbar_init(mma_done, 1);
        mbar_init(a_ready, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base, C::COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_base;

    if (warp == 0) {
        if (tid == 0) {
            mbar_expect_tx(q_full, C::Q_B);
            tma_rows_nb<NB>(sm + C::OFF_Q, &tq, q_full, t0, sq, BLK128);
            int n = 0;
            for (; n < N; ++n) {
                const int s = n % NS;
                if (!mbar_wait(&x_empty[s], ((n / NS) & 1) ^ 1, abort, p.status, p.wait_ns)) break;
                uint8_t *dst = sm + C::OFF_X + s * 2 * C::X_B;
                mbar_expect_tx(&x_full[s], 2 * C::X_B);
                tma_rows_nb<NB>(dst, &tk, &x_full[s], xs + GX * n, sq, BLK64);
                tma_rows_nb<NB>(dst + C::X_B, &tv, &x_full[s], xs + GX * n, sq, BLK64);
            }
            if (reads) {
                // A_b is the scan's output, and this kernel may start while the scan
                // still runs (it is only needed after the last key tile): wait for
                // the scan's grid here, then copy A_b hi, lo (rows (slot * 2 + part)
                // * D of the [.][D] map, NB column blocks)
                griddep_wait();
                const int slot = sq.bh * p.nC + blockIdx.x;
                mbar_expect_tx(a_ready, 2 * NB * C::ST_BLK);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        tma_load_2d(sm + C::OFF_A + (part * NB + b) * C::ST_BLK, &tab, a_ready, 64 * b,
                                    (slot * 2 + part) * D);
            }
            mbar_wait_drain(q_full, 0);
            if (reads) mbar_wait_drain(a_ready, 0);
            for (int st = 0; st < NS; ++st) {
                const int fills = n > st ? (n - 1 - st) / NS + 1 : 0;
                if (fills) mbar_wait_drain(&x_full[st], (fills - 1) & 1);
            }
        }
    } else if (warp == 1) {
        const uint32_t id_s = idesc_bf16(128, 64, false, false);
        const uint32_t id_o = idesc_bf16(128, D, false, true);
        const uint32_t sq_a = smem_u32(sm + C::OFF_Q), sx = smem_u32(sm + C::OFF_X);
        bool ok = gwait(q_full, 0, abort, p);
        // S(n) into score buffer n % 2
        auto issue_s = [&](int n) -> bool {
            const int st = n % NS;
            if (!gwait(&x_full[st], (n / NS) & 1, abort, p)) return false;
            tc_fence_after();
            const uint32_t kx = sx + st * 2 * C::X_B, sb = tb + C::TM_S + 64 * (n & 1);
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ss_w(sb, sdesc_sw128(sq_a + b * BLK128, 16, 1024) + 2 * k,
                             sdesc_sw128(kx + b * BLK64, 16, 1024) + 2 * k, id_s, (b > 0 || k > 0) ? 1u : 0u);
            mma_commit_w(&s_full[n & 1]);
            return true;
        };
        if (ok) ok = issue_s(0);
        bool first_read = true;
        for (int n = 0; ok && n < N; ++n) {
            // the next scores go out before this tile's P V
            if (n + 1 < N && !(ok = issue_s(n + 1))) break;
            if (!(ok = gwait(&p_ready[n & 1], (n >> 1) & 1, abort, p))) break;
            tc_fence_after();
            // O += P V (and M += P' V): K-step k (keys 16 k ..) at columns 32 (k / 2) + 8 (k % 2)
            const uint64_t vd = sdesc_sw128(sx + (n % NS) * 2 * C::X_B + C::X_B, BLK64, 1024);
            const uint32_t pb = tb + C::TM_S + 64 * (n & 1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_ts_w(tb + C::TM_O, pb + 32 * (k >> 1) + 8 * (k & 1), vd + 128 * k, id_o,
                         (n > 0 || k > 0) ? 1u : 0u);
            if (tile_reads(n)) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ts_w(tb + C::TM_MI, pb + 32 * (k >> 1) + 16 + 8 * (k & 1), vd + 128 * k, id_o,
                             (!first_read || k > 0) ? 1u : 0u);
                first_read = false;
            }
            mma_commit_w(&x_empty[n % NS]);
            mma_commit_w(o_done);
        }
        if (ok && reads) {
            // Q A_b (hi + lo) into the score columns, after every P V of the loop
            if ((ok = gwait(a_ready, 0, abort, p))) {
                tc_fence_after();
                const uint32_t sa = smem_u32(sm + C::OFF_A);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int k = 0; k < 4 * NB; ++k)
                        mma_ss_w(tb + C::TM_S, sdesc_sw128(sq_a + (k >> 2) * BLK128, 16, 1024) + 2 * (k & 3),
                                 sdesc_sw128(sa + part * NB * C::ST_BLK, C::ST_BLK, 1024) + 128 * k, id_o,
                                 (part > 0 || k > 0) ? 1u : 0u);
            }
        }
        if (ok) mma_commit_w(o_full);
        mma_commit_w(mma_done);
        mbar_wait_drain(mma_done, 0);
    } else {
        const int q4 = warp & 3;
        const int x = 32 * q4 + (tid & 31);
        const int r = x;
        const uint32_t lanes = tb + ((uint32_t)(32 * q4) << 16);
        const int t = t0 + r, tau = tau0 + r;
        const uint32_t wlim = t < sq.T ? (uint32_t)p.W : 0u;
        const float sl2 = kLog2eG * rsqrtf((float)D);
        if (reads) {
            // lam^n for the reads' weights (A_b arrives by copy), then the
            // padded eta lam^d table
            gpowers(pw, CG, p.lam[sq.h], x);
            const float eta = p.eta[sq.h];
            gbar128();  // pw complete
            for (int i = x; i < kEpw; i += 128) epw[i] = (i >= 128 && i < 128 + CG) ? eta * pw[i - 128] : 0.f;
            gbar128();  // epw complete
        }
        // the reads of row r cover evictions e_lo .. tau - W (none when tau < W or t >= T)
        const int rd_hi = (reads && t < sq.T) ? tau - p.W : -1;
        float m_used = -INFINITY, l_run = 0.f;  // max P is taken against (log2 units), row sum
        bool ok = true;
        for (int n = 0; n < N; ++n) {
            if (!(ok = gwait(&s_full[n & 1], (n >> 1) & 1, abort, p))) break;
            tc_fence_after();
            const uint32_t sbuf = lanes + C::TM_S + 64 * (n & 1);
            const int j0 = xs + GX * n;
            const int base = tau - j0;  // tau - j = base - c
            float s[GX];
            {
                uint32_t ra[32], rb[32];
                tmem_ld32(sbuf, ra);
                tmem_ld32(sbuf + 32, rb);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    s[c] = __uint_as_float(ra[c]);
                    s[32 + c] = __uint_as_float(rb[c]);
                }
            }
            const int kind = tile_kind(base, wlim);
            const float mt = (kind == kTileNone ? -INFINITY
                              : kind == kTileFull ? tile_max<false>(s, base, wlim)
                                                  : tile_max<true>(s, base, wlim)) * sl2;  // sl2 > 0
            const bool raise = mt > m_used + kRescaleG;
            // O holds earlier P V products only once some P was nonzero
            const bool resc = raise && m_used != -INFINITY;
            const float fo = resc ? gex2(m_used - mt) : 1.f;
            // rescale O once the previous P V is complete (its commit is the
            // (n-1)-th completion of o_done; the n-th cannot come before this
            // tile's P, so the parity names it unambiguously)
            if (__any_sync(0xffffffffu, resc)) {
                if (!(ok = gwait(o_done, (n - 1) & 1, abort, p))) break;
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(lanes + C::TM_O + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * fo);
                    tmem_st32(lanes + C::TM_O + c0, o);
                }
            }
            l_run *= fo;
            if (raise) m_used = mt;
            if (kind == kTileNone) {
                uint32_t z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) z[e] = 0u;
                tmem_st16(sbuf, z);
                tmem_st16(sbuf + 32, z);
            } else {
                const float m = m_used == -INFINITY ? 0.f : m_used;
                l_run += kind == kTileFull ? tile_p<false>(s, base, wlim, sl2, m, sbuf)
                                           : tile_p<true>(s, base, wlim, sl2, m, sbuf);
            }
            if (tile_reads(n)) {
                // P' = eta lam^(tau-W-j) s for e_lo <= j <= tau - W: d = rd_hi - j0 - c,
                // clamped so that every table index stays in [1, kEpw)
                const int off = max(rd_hi - j0, -GX);
                const int cmin = e_lo - j0;  // > 0 only in the first tile
                const float *w = epw + 128 + off;
                if (cmin > 0) tile_plin<true>(s, w, cmin, sbuf);
                else tile_plin<false>(s, w, cmin, sbuf);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_w(&p_ready[n & 1]);
        }
        if (ok && gwait(o_full, 0, abort, p)) {
            tc_fence_after();
            const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
            const bool has_m = (p.mrow && tau >= p.W && t < sq.T) || rd_hi >= e_lo;
            const float sg = has_m ? 1.f / (1.f + expf(-p.g[sq.h])) : 0.f;
            const float *mr = (p.mrow && has_m) ? p.mrow + grow(sq, t, p.T, p.H, D) : nullptr;
            // m = lam^(tau-W-e_lo+1) (q A_b) + (P' V) for the in-kernel reads
            const float dec = (reads && rd_hi >= e_lo) ? pw[min(rd_hi - e_lo + 1, CG)] : 0.f;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32], ma[32], mi[32];
                tmem_ld32(lanes + C::TM_O + c0, o);
                if (reads) {
                    tmem_ld32(lanes + C::TM_S + c0, ma);
                    tmem_ld32(lanes + C::TM_MI + c0, mi);
                }
                tmem_wait_ld();
                if (t < sq.T) {
                    float f[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) f[c] = __uint_as_float(o[c]) * inv_l;
                    if (mr) {
#pragma unroll
                        for (int c = 0; c < 32; c += 4) {
                            const float4 mv = *reinterpret_cast<const float4 *>(mr + c0 + c);
                            f[c] = fmaf(sg, mv.x, f[c]);
                            f[c + 1] = fmaf(sg, mv.y, f[c + 1]);
                            f[c + 2] = fmaf(sg, mv.z, f[c + 2]);
                            f[c + 3] = fmaf(sg, mv.w, f[c + 3]);
                        }
                    } else if (reads && has_m) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            f[c] = fmaf(sg, fmaf(dec, __uint_as_float(ma[c]), __uint_as_float(mi[c])), f[c]);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.y + grow(sq, t, p.T, p.H, D) + c0);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(pack_bf16(f[8 * u], f[8 * u + 1]), pack_bf16(f[8 * u + 2], f[8 * u + 3]),
                                            pack_bf16(f[8 * u + 4], f[8 * u + 5]),
                                            pack_bf16(f[8 * u + 6], f[8 * u + 7]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, C::COLS);
}

// ===========================================================================
// Per-chunk increments.  A = two 64-row M blocks (K^T of two chunks for
// D = 64, or the two column halves of one chunk's K^T for D = 128), B = the
// matching two N blocks of diag(w) V as bf16 hi + lo; D's diagonal blocks
// (D = 64) or all of it (D = 128) are the increments.
constexpr uint32_t SUM_OFF_A = 0;                  // 2 blocks (TMA)
constexpr uint32_t SUM_OFF_B = 2 * BLK128;         // hi: 2 blocks, lo: 2 blocks
constexpr uint32_t SUM_OFF_BAR = SUM_OFF_B + 4 * BLK128;
constexpr uint32_t SUM_SMEM = SUM_OFF_BAR + 64 + 1024;

template <int NB>
__global__ void __launch_bounds__(kGThreads, 2)
    gen_sums_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, GenParams p) {
    constexpr int D = 64 * NB;
    constexpr int CPB = NB == 1 ? 2 : 1;  // chunks per CTA
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SUM_OFF_BAR);
    uint64_t *in_full = bars, *b_ready = bars + 1, *acc_full = bars + 2, *mma_done = bars + 3;
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(bars + 4);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    const GSeq sq = gseq(p, blockIdx.y);
    const int bh = sq.bh, c_first = blockIdx.x * CPB;
    const int h = sq.h;
    if (c_first >= sq.nC) return;  // past this sequence's chunks (variable-length calls)
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
            mbar_expect_tx(in_full, 4 * BLK128);
            // K and V of chunks c_first, c_first + 1 (D = 64) or the two column
            // halves of chunk c_first (D = 128), from each chunk's first eviction;
            // rows past the data read zero, rows past a chunk meet zero weights.
            // V lands where B's hi blocks go: each element-wise thread turns its
            // own row into the weighted hi part in place.
            int lo0, hi0, lo1, hi1;
            chunk_range(p, sq, c_first, lo0, hi0);
            chunk_range(p, sq, c_first + 1, lo1, hi1);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const CUtensorMap *m = t == 0 ? &tk : &tv;
                uint8_t *dst = sm + (t == 0 ? SUM_OFF_A : SUM_OFF_B);
                tma_rows_nb<1>(dst, m, in_full, lo0, sq, BLK128);
                if (NB == 1)
                    tma_rows_nb<1>(dst + BLK128, m, in_full, lo1, sq, BLK128);
                else if (sq.packed)
                    tma_load_3d(dst + BLK128, m, in_full, 64, sq.h, sq.row0 + lo0);
                else
                    tma_load_3d(dst + BLK128, m, in_full, 64, lo0, bh);
            }
            mbar_wait_drain(in_full, 0);
        }
    } else if (warp == 1) {
        const uint32_t sa = smem_u32(sm + SUM_OFF_A), sb = smem_u32(sm + SUM_OFF_B);
        const uint32_t id = idesc_bf16(128, 128, true, true);
        bool ok = gwait(in_full, 0, abort, p) && gwait(b_ready, 0, abort, p);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ss_w(tb, sdesc_sw128(sa, BLK128, 1024) + 128 * k,
                             sdesc_sw128(sb + part * 2 * BLK128, BLK128, 1024) + 128 * k, id,
                             (part > 0 || k > 0) ? 1u : 0u);
            mma_commit_w(acc_full);
        }
        mma_commit_w(mma_done);
        mbar_wait_drain(mma_done, 0);
    } else {
        // row x of B is, for each N block b, w * V row of the block's chunk
        // (D = 64) or columns 64 b .. of the chunk's row (D = 128), w = lam^(L-1-x)
        const int x = 32 * (warp & 3) + (tid & 31);
        const uint32_t lanes = tb + ((uint32_t)(32 * (warp & 3)) << 16);
        float wrow[2];
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const int c = NB == 1 ? c_first + b : c_first;
            int e0, e1;
            chunk_range(p, sq, c, e0, e1);
            const int L = c < sq.nC ? e1 - e0 : 0;
            wrow[b] = x < L ? gpow(p.lam[h], L - 1 - x) : 0.f;
        }
        if (gwait(in_full, 0, abort, p)) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const float w = wrow[b];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint8_t *hp = sm + SUM_OFF_B + b * BLK128 + sw128_offset(x, 8 * u);
                    const uint4 a = w != 0.f ? *reinterpret_cast<const uint4 *>(hp) : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t ws[4] = {a.x, a.y, a.z, a.w};
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        gsplit(w * __uint_as_float(ws[e] << 16), w * __uint_as_float(ws[e] & 0xffff0000u), hi[e],
                               lo[e]);
                    *reinterpret_cast<uint4 *>(hp) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(sm + SUM_OFF_B + (2 + b) * BLK128 + sw128_offset(x, 8 * u)) =
                        make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
            }
            fence_async_smem();
            mbar_arrive(b_ready);
        }
        // The result goes out through shared memory (the B region, free once the
        // product is done) so that whole warps write contiguous rows: row x of
        // the staged tile is lane x's TMEM row, eta-scaled, 16-byte chunk u at
        // chunk u ^ (x & 15) of its row.
        constexpr int RW = NB == 1 ? 64 : 128;  // floats per staged row
        constexpr int NCH = RW / 4;             // 16-byte chunks per row
        float *stage = reinterpret_cast<float *>(sm + SUM_OFF_B);
        const bool have = gwait(acc_full, 0, abort, p);
        if (have) {
            tc_fence_after();
            const float eta = p.eta[h];
            // D = 64: lanes 0..63 rows of chunk c_first (columns 0..63), 64..127 of
            // c_first + 1 (columns 64..127); D = 128: every lane a row, all columns
            const uint32_t col0 = NB == 1 ? (uint32_t)(x & 64) : 0u;
#pragma unroll
            for (int c0 = 0; c0 < RW; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(lanes + col0 + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int u = c0 / 4 + q;
                    *reinterpret_cast<float4 *>(stage + x * RW + 4 * (u ^ (x & 15))) =
                        make_float4(eta * __uint_as_float(v[4 * q]), eta * __uint_as_float(v[4 * q + 1]),
                                    eta * __uint_as_float(v[4 * q + 2]), eta * __uint_as_float(v[4 * q + 3]));
                }
            }
        }
        gbar128();  // every element-wise thread, whether or not its wait succeeded
        if (!*abort) {
            // rows 0..127 of the tile are consecutive rows of dA: chunk c_first's
            // 64 (or 128) rows, then (D = 64) chunk c_first + 1's
            float *dst = p.dA + ((size_t)bh * p.nC + c_first) * D * D;
            const int et = tid - 64;  // 0 .. 127
#pragma unroll 4
            for (int i = et; i < 128 * NCH; i += 128) {
                const int row = i / NCH, u = i % NCH;
                const int c = NB == 1 ? c_first + (row >> 6) : c_first;
                if (c < sq.nC)
                    *reinterpret_cast<float4 *>(dst + (size_t)row * RW + 4 * u) =
                        *reinterpret_cast<const float4 *>(stage + row * RW + 4 * (u ^ (row & 15)));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, 128);
}

// ===========================================================================
// Chunk start states A_c (as bf16 hi + lo, for the window kernel's copies)
// and A_final, from the increments of the sums kernel.
constexpr int kMaxScanChunks = 4096;  // chunk decays kept in shared memory (longer rows compute theirs)
constexpr int kScanThreads = 256;
constexpr int kScanVec = 4;            // consecutive state elements per thread

// bf16 hi + lo of four floats, as two 8-byte words
__device__ __forceinline__ void split4(const float4 a, uint2 &hi, uint2 &lo) {
    uint32_t h0, h1, l0, l1;
    gsplit(a.x, a.y, h0, l0);
    gsplit(a.z, a.w, h1, l1);
    hi = make_uint2(h0, h1);
    lo = make_uint2(l0, l1);
}

// Chunk start states A_c (c = 0 .. nC-1) of one row from A_init and the
// increments, A_{c+1} = lam^(L_c) A_c + dA_c, written as bf16 hi + lo for the
// window kernel's copies, and A_final.  Each thread carries kScanVec
// consecutive elements of the D x D state through every chunk.
__global__ void __launch_bounds__(kScanThreads) gen_scan_kernel(GenParams p, int D) {
    extern __shared__ float decay[];  // lam^(length of chunk c), c < min(p.nC, kMaxScanChunks)
    // the window kernel may start now: it reads these states only after
    // waiting for this grid to complete
    griddep_launch_dependents();
    const GSeq sq = gseq(p, blockIdx.y);
    const int bh = sq.bh, nC = sq.nC;
    const float lam = p.lam[sq.h];
    for (int c = threadIdx.x; c < nC && c < kMaxScanChunks; c += blockDim.x) {
        int e0, e1;
        chunk_range(p, sq, c, e0, e1);
        decay[c] = gpow(lam, e1 - e0);
    }
    __syncthreads();
    const int nel = D * D;
    const int x = kScanVec * (blockIdx.x * blockDim.x + threadIdx.x);
    if (x >= nel) return;
    float4 A = p.A_init ? *reinterpret_cast<const float4 *>(p.A_init + (size_t)bh * nel + x)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    const float *dA = p.dA + (size_t)bh * p.nC * nel + x;  // p.nC: chunk slots per row
    constexpr int kB = 8;
    for (int c0 = 0; c0 < nC; c0 += kB) {
        float4 d[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u)
            d[u] = (c0 + u < nC && sq.E > 0) ? *reinterpret_cast<const float4 *>(dA + (size_t)(c0 + u) * nel)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int c = c0 + u;
            if (c < nC) {
                // the start state as bf16 hi + lo, row-major, for the window kernel's copy
                uint2 hi, lo;
                split4(A, hi, lo);
                __nv_bfloat16 *o = p.ab + (((size_t)bh * p.nC + c) * 2) * nel + x;
                *reinterpret_cast<uint2 *>(o) = hi;
                *reinterpret_cast<uint2 *>(o + nel) = lo;
                float dc;
                if (c < kMaxScanChunks) {
                    dc = decay[c];
                } else {
                    int e0, e1;
                    chunk_range(p, sq, c, e0, e1);
                    dc = gpow(lam, e1 - e0);
                }
                A = make_float4(fmaf(dc, A.x, d[u].x), fmaf(dc, A.y, d[u].y), fmaf(dc, A.z, d[u].z),
                                fmaf(dc, A.w, d[u].w));
            }
        }
    }
    if (p.A_final) *reinterpret_cast<float4 *>(p.A_final + (size_t)bh * nel + x) = A;
}

// ===========================================================================
// Halo + new rows of keys and values into one [BH][Tc][D] sequence.
__global__ void gen_combine_kernel(const __nv_bfloat16 *halo, const __nv_bfloat16 *src, __nv_bfloat16 *dst,
                                   int n_halo, int T, int D, int64_t BH) {
    const int64_t per = (int64_t)(n_halo + T) * D / 8;  // 16-byte units per head
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < BH * per; x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bh = x / per, u = x % per;
        const int64_t row = u * 8 / D, col = u * 8 % D;
        const uint4 *s = row < n_halo
                             ? reinterpret_cast<const uint4 *>(halo + (bh * n_halo + row) * D + col)
                             : reinterpret_cast<const uint4 *>(src + (bh * T + row - n_halo) * D + col);
        reinterpret_cast<uint4 *>(dst)[x] = *s;
    }
}

typedef CUresult (*EncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                             const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [BH][rows][D] bf16 -> 3D map (D, rows, BH), boxes of 64 columns x box_rows x 1, 128-byte swizzle
bool gen_map(CUtensorMap *m, const void *base, int rows, int BH, int D, int box_rows) {
    EncodeFn fn = reinterpret_cast<EncodeFn>(tensor_map_encoder());
    if (!fn || rows < 1) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed [total][H][D] bf16 -> 3D map (D, H, total), boxes of 64 columns x 1 x box_rows:
// the same shared-memory tile as gen_map's, box_rows token rows of one head
bool gen_map_packed(CUtensorMap *m, const void *base, int total, int H, int D, int box_rows) {
    EncodeFn fn = reinterpret_cast<EncodeFn>(tensor_map_encoder());
    if (!fn || total < 1) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows][D] bf16 -> 2D map, boxes of 64 columns x D rows, 128-byte swizzle
// (the split chunk start states: D rows per part of each slot)
bool gen_map_rows(CUtensorMap *m, const void *base, int64_t rows, int D) {
    EncodeFn fn = reinterpret_cast<EncodeFn>(tensor_map_encoder());
    if (!fn || rows < 1) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)D};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t gal(size_t x) { return (x + 255) & ~size_t(255); }

struct GenLayout {
    size_t kc, vc, mrow, dA, ab, total;
};
GenLayout gen_layout(const tc_prefill_desc &d, int64_t n_halo) {
    const int64_t BH = d.B * d.H, D = d.dk, Tc = n_halo + d.T;
    const int64_t nC = (d.T + CG - 1) / CG;  // one chunk per block of 128 new rows
    const bool l1 = (d.flags & TC_PREFILL_L1_ONLY) != 0;
    const bool delta = (d.flags & TC_PREFILL_DELTA_RULE) != 0;
    GenLayout L;
    L.kc = 0;
    const size_t comb = n_halo > 0 ? gal((size_t)(BH * Tc * D) * 2) : 0;
    L.vc = L.kc + comb;
    L.mrow = L.vc + comb;  // (unused: the reads happen inside the window kernel)
    L.dA = L.mrow;
    const size_t dA = (!l1 && !delta) ? gal((size_t)(BH * nC * D * D) * sizeof(float)) : 0;
    L.ab = L.dA + dA;  // the split start states: the same bytes again
    L.total = L.ab + dA;
    return L;
}

template <int NB>
cudaError_t launch_general_t(const PrefillParams &pp, const float *mrow_in, cudaStream_t s) {
    constexpr int D = 64 * NB;
    tc_prefill_desc d{};
    d.B = pp.B;
    d.H = pp.H;
    d.T = pp.T;
    d.dk = pp.dk;
    d.dv = pp.dv;
    d.W = pp.W;
    d.C = pp.C;
    d.dtype = TC_BF16;
    d.flags = (pp.l1_only ? TC_PREFILL_L1_ONLY : 0u) | (pp.state_only ? TC_PREFILL_STATE_ONLY : 0u) |
              (pp.delta_rule ? TC_PREFILL_DELTA_RULE : 0u);
    const GenLayout Lo = gen_layout(d, pp.n_halo);
    char *ws = static_cast<char *>(pp.workspace);
    const int BH = (int)(pp.B * pp.H);
    GenParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(pp.q);
    p.k = static_cast<const __nv_bfloat16 *>(pp.k);
    p.v = static_cast<const __nv_bfloat16 *>(pp.v);
    p.y = static_cast<__nv_bfloat16 *>(pp.y);
    p.T = (int)pp.T;
    p.n_halo = (int)pp.n_halo;
    p.Tc = p.T + p.n_halo;
    p.W = (int)(pp.W < p.Tc + 1 ? pp.W : p.Tc + 1);  // a window past the sequence changes nothing
    p.H = (int)pp.H;
    p.E = p.Tc > p.W ? p.Tc - p.W : 0;
    p.nC = (p.T + CG - 1) / CG;  // chunk slots per row: one per block of 128 new rows
    p.lam = pp.lam;
    p.eta = pp.eta;
    p.g = pp.g;
    p.A_init = pp.A_init;
    p.A_final = pp.A_final;
    p.status = pp.status;
    p.wait_ns = pp.wait_ns;
    p.cu = pp.cu_seqlens;  // variable-length: T is the longest length, no halo
    p.total = (int)pp.total;
    const bool packed = p.cu != nullptr;
    cudaError_t e;
    if (p.n_halo > 0) {  // one sequence of keys and values, halo first
        __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(ws + Lo.kc);
        __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(ws + Lo.vc);
        gen_combine_kernel<<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(pp.halo_k), p.k, kc, p.n_halo,
                                                p.T, D, BH);
        gen_combine_kernel<<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(pp.halo_v), p.v, vc, p.n_halo,
                                                p.T, D, BH);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        p.k = kc;
        p.v = vc;
    }
    const bool l2 = !pp.l1_only && !pp.delta_rule;
    p.dA = l2 ? reinterpret_cast<float *>(ws + Lo.dA) : nullptr;
    p.ab = l2 ? reinterpret_cast<__nv_bfloat16 *>(ws + Lo.ab) : nullptr;
    p.mrow = pp.delta_rule ? const_cast<float *>(mrow_in) : nullptr;
    const bool queries = !pp.state_only && p.T > 0;
    CUtensorMap mk128, mv128, mq128, mk64, mv64;
    auto map = [&](CUtensorMap *m, const void *base, int rows, int box) {
        return packed ? gen_map_packed(m, base, p.total, p.H, D, box) : gen_map(m, base, rows, BH, D, box);
    };
    if ((queries || (l2 && p.E > 0)) &&
        (!map(&mk128, p.k, p.Tc, 128) || !map(&mv128, p.v, p.Tc, 128) || !map(&mk64, p.k, p.Tc, 64) ||
         !map(&mv64, p.v, p.Tc, 64)))
        return cudaErrorInvalidValue;
    if (queries && !map(&mq128, p.q, p.T, 128)) return cudaErrorInvalidValue;
    CUtensorMap mab = mq128;  // any valid map when the memory is off (not read then)
    if (queries && l2 && p.nC > 0 && !gen_map_rows(&mab, p.ab, (int64_t)BH * p.nC * 2 * D, D))
        return cudaErrorInvalidValue;
    if (l2) {
        if (p.E > 0) {
            e = cudaFuncSetAttribute(gen_sums_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SUM_SMEM);
            if (e != cudaSuccess) return e;
            const int cpb = NB == 1 ? 2 : 1;
            gen_sums_kernel<NB><<<dim3((unsigned)((p.nC + cpb - 1) / cpb), (unsigned)BH), kGThreads, SUM_SMEM, s>>>(
                mk128, mv128, p);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        const int per_cta = kScanThreads * kScanVec;
        const size_t decay_bytes = (size_t)(p.nC < kMaxScanChunks ? p.nC : kMaxScanChunks) * sizeof(float);
        gen_scan_kernel<<<dim3((unsigned)((D * D + per_cta - 1) / per_cta), (unsigned)BH), kScanThreads,
                          decay_bytes, s>>>(p, D);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (queries) {
        using WC = WinCfg<NB>;
        e = cudaFuncSetAttribute(gen_window_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)WC::SMEM);
        if (e != cudaSuccess) return e;
        // After the scan, the window kernel may start early (programmatic stream
        // serialization): it reads the scan's states only after griddep_wait,
        // and everything else it reads was complete before the sums kernel
        // (launched in plain stream order) started.
        cudaLaunchAttribute early[1];
        early[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        early[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t wc = {};
        wc.gridDim = dim3((unsigned)((p.T + CG - 1) / CG), (unsigned)BH);
        wc.blockDim = dim3(kGThreads);
        wc.dynamicSmemBytes = WC::SMEM;
        wc.stream = s;
        wc.attrs = early;
        wc.numAttrs = l2 ? 1 : 0;
        e = cudaLaunchKernelEx(&wc, gen_window_kernel<NB>, mq128, mk64, mv64, mab, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

bool general_varlen_supported(const tc_prefill_desc &d) {
    tc_prefill_desc c = d;
    if (c.T < 1) c.T = 1;
    return !(d.flags & ~TC_PREFILL_L1_ONLY) && general_supported(c, 0);
}

bool general_supported(const tc_prefill_desc &d, int64_t n_halo) {
    if (d.dtype != TC_BF16 || d.dk != d.dv || (d.dk != 64 && d.dk != 128)) return false;
    if (d.flags & TC_PREFILL_CHUNK_MEAN) return false;
    if ((d.flags & TC_PREFILL_DELTA_RULE) && (n_halo != 0 || (d.flags & (TC_PREFILL_STATE_ONLY | TC_PREFILL_L1_ONLY))))
        return false;
    // shapes only: a call without a device gets TC_ERR_NO_DEVICE, not UNSUPPORTED;
    // the split start states are addressed by 32-bit copy coordinates
    const int64_t slots = d.B * d.H * ((d.T + CG - 1) / CG);
    return d.T + n_halo < (int64_t(1) << 30) && d.B * d.H <= 65535 && slots * 2 * d.dk < (int64_t(1) << 31);
}

size_t general_workspace_bytes(const tc_prefill_desc &d, int64_t n_halo) { return gen_layout(d, n_halo).total; }

int general_launch_count(const tc_prefill_desc &d, int64_t n_halo) {
    const int64_t Tc = n_halo + d.T, W = d.W < Tc + 1 ? d.W : Tc + 1, E = Tc > W ? Tc - W : 0;
    const bool l1 = (d.flags & TC_PREFILL_L1_ONLY) != 0, state = (d.flags & TC_PREFILL_STATE_ONLY) != 0;
    const bool delta = (d.flags & TC_PREFILL_DELTA_RULE) != 0;
    const bool queries = !state && d.T > 0;
    int n = n_halo > 0 ? 2 : 0;
    if (!l1 && !delta) n += (E > 0 ? 1 : 0) + 1;  // sums, scan
    return n + (queries ? 1 : 0);                  // window (with the reads)
}

cudaError_t launch_prefill_general(const PrefillParams &p, const float *mrow, cudaStream_t s) {
    return p.dk == 64 ? launch_general_t<1>(p, mrow, s) : launch_general_t<2>(p, mrow, s);
}

}  // namespace tc
