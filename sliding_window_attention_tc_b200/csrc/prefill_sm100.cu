// Tensor-core prefill of the Tensor Cache layer for B200 (tcgen05 + TMA),
// bf16 inputs with d_k = d_v = 64 and W a multiple of 128.
//
// "Tensor Cache: Eviction-conditioned Associative Memory for Transformers":
// L1 is exact softmax attention over the window (§3.1 eq. (1)); L2 is the
// matrix A written by evicted pairs A <- lambda A + eta k v^T and read as
// m = q A (§3.2, Fig. 2 steps (3) and (5)); y = y_local + sigmoid(g) m.  The
// training form computes A with the parallel weighted-sum chunk scan
// (abstract; §1; §2), here with chunks of 128 evictions = one query tile.
//
// Tiling.  Query tile = 128 rows t0..t0+127 of one (b,h).  Its keys are
// 128-row key tiles:
//   LEAD  [t0-W, t0-W+128)  (when t0 >= W): column c <= row r is eviction
//         e = t0-W+c <= t-W, i.e. already in A -> decay-weighted linear read
//         eta lam^(r-c) <q,k> v (intra-chunk part of m); c > r is in the
//         window -> softmax.  One Q K^T product serves both paths.
//   FULL  tiles fully inside every row's window -> softmax.
//   DIAG  [t0, t0+128): causal mask c <= r.
// The inter-chunk read lam^(r+1) q S(n0) uses the state S(n0) = A after the
// first n0 = t0-W evictions, and the state advances per tile as
//   S(n0+128) = lam^128 S(n0) + K_lead^T diag(eta lam^(127-c)) V_lead,
// a tensor-core contraction whose scaled keys are split into bf16 hi + lo
// parts (stacked as the M = 128 rows of one MMA) so that A keeps float32
// accuracy.
//
// Work split.  Each head's query tiles are cut into n_s contiguous spans; a
// persistent CTA (one per SM) runs spans.  A span that starts after other
// evictions of its head needs S at its start.  Two small pre-pass kernels
// provide it: span_summary_kernel computes, in parts spread over CTAs, the
// state dA_u that the evictions of span u add (decayed to the span's end),
// and span_prefix_kernel folds the parts and the predecessors into one start
// state per span.  The prefix and main kernels are launched as programmatic
// dependents of the kernel before them: each may start as its predecessor's
// CTAs finish, and waits for the predecessor's results (griddep_wait) only
// where it reads them.
//
// Roles in the main kernel (512 threads):
//   warp 0        TMA producer: Q tile, then K/V tiles through an NS-stage ring
//   warp 1        MMA issuer: S = Q K^T into TMEM (two buffers), O += P V
//                 with P read from TMEM, the L2 MMAs; owns TMEM
//   warps 2-3     idle
//   warps 4-11    softmax + epilogue, two column halves: warps 4-7 take score
//                 columns 0-63, warps 8-11 columns 64-127; one thread per
//                 query row / TMEM lane in each half; the halves exchange
//                 their row maxima once per key tile
//   warps 12-15   state: keeps S (float32, registers), stages it as bf16 for
//                 the inter read, builds the scaled hi/lo keys
// All waits are bounded (mbar_wait); on timeout every role drains and the
// kernel returns with TC_ERR_DEVICE_TIMEOUT in the status word.

#include <cuda.h>

#include "sm100_ptx.cuh"
#include "tc_internal.cuh"

namespace tc {
namespace {

using namespace sm100;

constexpr int BM = 128;                  // query / key rows per tile, eviction chunk
constexpr int HD = 64;                   // head dimension handled here
constexpr int NS = 4;                    // K/V stages (main kernel)
constexpr uint32_t TILE_B = BM * HD * 2; // 16 KB bf16 tile
constexpr int kMainThreads = 512;
constexpr int kMaxSpans = 64;           // spans per head at most (choose_spans)

// main-kernel shared memory (offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;                          // 2 Q tiles
constexpr uint32_t OFF_KV = OFF_Q + 2 * TILE_B;        // NS x (K, V)
constexpr uint32_t OFF_KT = OFF_KV + NS * 2 * TILE_B;  // scaled keys hi | lo
constexpr uint32_t OFF_SB = OFF_KT + 2 * TILE_B;       // state bf16 [64 k][64 n]
constexpr uint32_t OFF_DS = OFF_SB + 8192;             // float32 64x64 scratch
constexpr uint32_t OFF_EPW = OFF_DS + 16384;           // [256]: eta lam^(i-128), 0 for i < 128
constexpr uint32_t OFF_XM = OFF_EPW + 1024;            // [2 parity][2 halves][128] row maxima
constexpr uint32_t OFF_XL = OFF_XM + 2048;             // [2 halves][128] row sums
constexpr uint32_t OFF_STT = OFF_XL + 1024;            // state tables: eta lam^k, lam^k
constexpr uint32_t OFF_BAR = OFF_STT + 1536;
constexpr uint32_t SMEM_MAIN = OFF_BAR + 256 + 1024;

// TMEM columns (512 allocated)
constexpr uint32_t TM_S = 0;    // two 128-column score buffers (P / P' alias them)
constexpr uint32_t TM_O = 256;  // O accumulator, 64 columns
constexpr uint32_t TM_MI = 320; // intra-chunk memory read
constexpr uint32_t TM_MX = 384; // inter-chunk memory read q S(n0)
constexpr uint32_t TM_DS = 448; // state increment: rows 0-63 hi part, 64-127 lo part

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;  // rescale O only when the running max grows by > 2^8

// Variable-length calls: sequence b of the batch is tokens cu[b] .. cu[b+1]-1
// of packed [total][H][64] tensors; cu == null for fixed-length calls.
struct Varlen {
    const int64_t *cu;   // device [n_seq + 1]
    int total, max_len;
};

struct PrefixParams {
    float *dA;            // [BH * (n_s - 1) * n_parts][64][64]: partial summaries in,
                          // span start states out (over part 0 of the previous span)
    const float *lam;
    int T, W, H, nT, n_s, n_parts, q_off;
    Varlen vl;
    int *status;
};

// Token coordinates.  The kernels run over a combined sequence of T tokens:
// the first q_off are a halo (the keys and values of the tokens just before
// a continued sequence, read through their own tensor maps), the rest are the
// new tokens, whose queries and outputs are rows 0.. of q and y.  Query tiles
// start at i_begin = q_off / 128; q_off is 0 or W, a multiple of 128.
struct MainParams {
    void *y;
    float *A_final;
    const float *lam, *eta, *g;
    const float *S_pre;   // state at the start of span js >= 1: matrix (bh (n_s-1) + js-1) n_parts
    const float *A_init;  // [BH][64][64] state before the first eviction, or null
    int T, W, H, BH, nT, n_s, n_parts, l1_only, q_off;
    int *status;
    unsigned long long wait_ns;  // limit of every bounded wait
    Varlen vl;
    const int *order;     // rows (bh) in the order their spans are dealt out, or null
};

struct SumParams {
    float *dA;            // [BH * (n_s - 1) * n_parts][64][64] partial span summaries
    const float *lam, *eta;
    int T, W, H, BH, nT, n_s, n_parts, q_off;
    int *status;
    unsigned long long wait_ns;  // limit of every bounded wait
    Varlen vl;
};

// Query tiles [i0, i1) of span j: the tiles i_begin .. nT-1 cut into n_s parts.
__device__ __forceinline__ void span_range(int j, int nT, int n_s, int i_begin, int &i0, int &i1) {
    const int n = nT - i_begin;
    i0 = i_begin + (int)((long long)j * n / n_s);
    i1 = i_begin + (int)((long long)(j + 1) * n / n_s);
}

// The k-th span of this CTA.  Spans are dealt to the persistent CTAs in
// snake order (round k left to right when k is even, right to left when
// odd) over the rows in `order` (null: index order), so that with rows
// sorted longest first the CTAs get nearly equal work.  Returns false past
// the last span.
struct Span {
    int bh, js;
};
__device__ __forceinline__ bool cta_span(int k, int n_spans, int n_s, const int *order, Span &sp) {
    const int G = gridDim.x, c = blockIdx.x;
    const long long pos = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
    if (pos >= n_spans) return false;
    const int row = (int)(pos / n_s);
    sp.bh = order ? order[row] : row;
    sp.js = (int)(pos % n_s);
    return true;
}

// The sequence of row bh (one head of one sequence).  Fixed-length calls: T
// tokens (halo included) in the row's own [T][64] slab.  Variable-length
// calls: sequence b = bh / H, tokens cu[b] .. cu[b+1]-1 of the packed
// [total][H][64] tensors, head z = bh % H.  Offsets that are inconsistent
// (decreasing, past total, or longer than max_len) are reported as
// TC_ERR_DEVICE_BOUNDS and the row is treated as empty, so nothing outside
// the tensors is read or written.
struct SeqView {
    int T, nT, row0, z;
};
__device__ __forceinline__ SeqView seq_view(const Varlen &vl, int bh, int H, int T_fixed,
                                            int *status) {
    SeqView v;
    if (!vl.cu) {
        v.T = T_fixed;
        v.row0 = 0;
        v.z = bh;
    } else {
        const int b = bh / H;
        const int64_t a = vl.cu[b], e = vl.cu[b + 1];
        if (a < 0 || e < a || e > vl.total || e - a > vl.max_len) {
            report(status, 5);
            v.T = 0;
            v.row0 = 0;
        } else {
            v.T = (int)(e - a);
            v.row0 = (int)a;
        }
        v.z = bh % H;
    }
    v.nT = (v.T + BM - 1) / BM;
    return v;
}

// 128 rows starting at sequence row `row` of a [.][64] tensor map: (0, row, z)
// for fixed-length maps, (0, z, row0 + row) for the packed (d, H, total) maps.
__device__ __forceinline__ void tma_rows(void *dst, const CUtensorMap *m, uint64_t *bar, int row,
                                         const SeqView &v, bool varlen) {
    if (varlen)
        tma_load_3d(dst, m, bar, 0, v.z, v.row0 + row);
    else
        tma_load_3d(dst, m, bar, 0, row, v.z);
}

// Key / value tile u of the combined sequence: halo maps for u < q_off/128.
__device__ __forceinline__ void load_kv_tile(uint8_t *dst, const CUtensorMap *tk,
                                             const CUtensorMap *tv, const CUtensorMap *tkh,
                                             const CUtensorMap *tvh, uint64_t *bar, int u,
                                             int q_off, const SeqView &v, bool varlen) {
    const int row = u * 128;
    if (row < q_off) {
        tma_load_3d(dst, tkh, bar, 0, row, v.z);
        tma_load_3d(dst + 128 * 64 * 2, tvh, bar, 0, row, v.z);
    } else {
        tma_rows(dst, tk, bar, row - q_off, v, varlen);
        tma_rows(dst + 128 * 64 * 2, tv, bar, row - q_off, v, varlen);
    }
}

// Named barrier over n threads that also ORs pred over them; returns true if
// any passed true.  A hardware barrier has no time limit, so a role group
// that syncs with it follows one rule: a bounded wait that gives up only sets
// a flag, the thread still reaches the group's next barrier with it, and all
// threads leave their loops together right after a barrier that reported
// one.  Every thread of the group then passes the same sequence of barriers.
// (Per query key tile it costs a few tens of cycles, against a few hundred
// for an mbarrier that 256 threads arrive on and poll.)
__device__ __forceinline__ bool bar_any(int id, int n, bool pred) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return res != 0;
}

// mbar_wait with one answer for the whole warp, so that warps which go on to
// warp-collective tcgen05.ld / st never diverge on a failed wait.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          int *status, uint64_t limit = kWaitTimeoutNs) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status, limit));
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Per-tile schedule shared by every role.
struct TileInfo {
    int t0, nk, kt0;
    bool lead, l2;
};
__device__ __forceinline__ TileInfo tile_info(int i, int W, bool l1_only) {
    TileInfo ti;
    ti.t0 = i * BM;
    ti.lead = ti.t0 >= W;
    ti.l2 = ti.lead && !l1_only;
    if (ti.lead) {
        ti.nk = W / BM + 1;
        ti.kt0 = (ti.t0 - W) / BM;
    } else {
        ti.nk = i + 1;
        ti.kt0 = 0;
    }
    return ti;
}

// Kinds of key tile seen by one query row r (column c of the tile):
//   FULL     every column is in the window            -> softmax
//   DIAG     c <= r in the window (causal diagonal)   -> softmax, c > r masked
//   LEAD     c > r in the window, c <= r evicted      -> softmax on c > r, and
//   LEAD_L2  ... plus the linear read eta lam^(r-c) <q,k> for c <= r (P')
enum { KIND_FULL = 0, KIND_DIAG = 1, KIND_LEAD = 2, KIND_LEAD_L2 = 3 };

// rc = r - cb: the row index relative to this half's first column cb, so a
// local column c is global column cb + c.  One instance of each kind serves
// both halves, and DIAG and LEAD share one masked instance: column c is in
// the window iff rcx - sgn * c >= 0, with (rcx, sgn) = (rc, 1) for DIAG
// (c <= rc) and (-rc - 1, -1) for LEAD (c > rc).  The kernel's code exceeds
// the SM instruction cache, so smaller code is faster.
template <int KIND>
__device__ __forceinline__ bool in_window(int c, int rcx, int sgn) {
    return KIND == KIND_FULL ? true : rcx - sgn * c >= 0;
}

// x on window columns, -inf elsewhere, without predicate registers: the sign
// of (rc - c) or (c - rc - 1) selects the bits of x or of -inf (one LOP3).
template <int KIND>
__device__ __forceinline__ float mask_window(float x, int c, int rcx, int sgn) {
    if (KIND == KIND_FULL) return x;
    const int d = rcx - sgn * c;
    const int m = d >> 31;  // 0 in the window, -1 outside
    return __int_as_float((__float_as_int(x) & ~m) | (int(0xff800000u) & m));
}

// Row maximum of the raw scores over this half's window columns (-inf if none).
template <int KIND>
__device__ __forceinline__ float window_max(const float (&s)[64], int rc, int sgn) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 64; c += 2)
        m[(c >> 1) & 7] = fmax3(m[(c >> 1) & 7], in_window<KIND>(c, rc, sgn) ? s[c] : -INFINITY,
                                in_window<KIND>(c + 1, rc, sgn) ? s[c + 1] : -INFINITY);
    return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// P = exp2(s * sl2 - m) on window columns (0 elsewhere) as bf16 pairs into 32
// TMEM columns starting at taddr; returns this half's row sum of P.
template <int KIND>
__device__ __forceinline__ float write_p(const float (&s)[64], int rc, int sgn, float sl2,
                                      float m, uint32_t taddr) {
    uint64_t acc[2] = {0ull, 0ull};  // (0.f, 0.f) pairs
    const uint64_t sl2p = f2pack(sl2, sl2), negm = f2pack(-m, -m);
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int c = c0 + 2 * e;
            float x0, x1;
            ffma2(x0, x1, s[c], s[c + 1], sl2p, negm);
            x0 = mask_window<KIND>(x0, c, rc, sgn);
            x1 = mask_window<KIND>(x1, c + 1, rc, sgn);
            const float p0 = ex2(x0), p1 = ex2(x1);
            fadd2_acc(acc[e & 1], p0, p1);
            pk[e] = pack_bf16(p0, p1);
        }
        tmem_st16(taddr + c0 / 2, pk);
    }
    float a0, a1, b0, b1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc[0]));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(acc[1]));
    return (a0 + b0) + (a1 + b1);
}

// P' = eta lam^(r-c) s for c <= r (the zero-padded table gives 0 for c > r)
// as bf16 pairs into 32 TMEM columns starting at taddr.
__device__ __forceinline__ void write_plin(const float (&s)[64], int rc, const float *epw_pad,
                                        uint32_t taddr) {
    const float *w = epw_pad + 128 + rc;  // w[-c] = eta lam^(rc-c), or 0 when c > rc
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int c = c0 + 2 * e;
            pk[e] = pack_bf16(s[c] * w[-c], s[c + 1] * w[-c - 1]);
        }
        tmem_st16(taddr + c0 / 2, pk);
    }
}

// A masked kind reduces to FULL (every column inside) or to nothing (every
// column outside) for the whole warp when all its rows agree; such warps skip
// the per-column masks, and fully masked ones skip the exponentials.
enum { SLICE_NONE = -1 };
__device__ __forceinline__ int slice_kind(int kind, int rc) {
    if (kind == KIND_FULL) return KIND_FULL;
    const bool lead = kind != KIND_DIAG;
    const bool all_in = lead ? (rc < 0) : (rc >= 63);
    const bool all_out = lead ? (rc >= 63) : (rc < 0);
    if (__all_sync(0xffffffffu, all_in)) return KIND_FULL;
    if (__all_sync(0xffffffffu, all_out)) return SLICE_NONE;
    return lead ? KIND_LEAD : KIND_DIAG;
}

__device__ __forceinline__ float half_max(int kind, const float (&s)[64], int rc) {
    switch (kind) {
        case SLICE_NONE: return -INFINITY;
        case KIND_FULL: return window_max<KIND_FULL>(s, rc, 1);
        case KIND_DIAG: return window_max<KIND_DIAG>(s, rc, 1);
        default: return window_max<KIND_DIAG>(s, -rc - 1, -1);
    }
}
__device__ __forceinline__ float half_p(int kind, const float (&s)[64], int rc, float sl2, float m,
                                        uint32_t taddr) {
    switch (kind) {
        case SLICE_NONE: {
            uint32_t z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) z[e] = 0u;
            tmem_st16(taddr, z);
            tmem_st16(taddr + 16, z);
            return 0.f;
        }
        case KIND_FULL: return write_p<KIND_FULL>(s, rc, 1, sl2, m, taddr);
        case KIND_DIAG: return write_p<KIND_DIAG>(s, rc, 1, sl2, m, taddr);
        default: return write_p<KIND_DIAG>(s, -rc - 1, -1, sl2, m, taddr);
    }
}

// Scaled key row for the state MMA: row u of the key tile times w, split into
// bf16 hi and lo = bf16(x - hi), written to two SWIZZLE_128B tiles.
__device__ __forceinline__ void build_scaled_key_row(const uint8_t *ktile, uint8_t *hi_tile,
                                                     uint8_t *lo_tile, int u, float w) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint32_t off = sw128_offset(u, ch * 8);
        const uint4 raw = *reinterpret_cast<const uint4 *>(ktile + off);
        float f[8];
        Vec16<__nv_bfloat16>::unpack(raw, f);
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = f[2 * e] * w, x1 = f[2 * e + 1] * w;
            const uint32_t hp = pack_bf16(x0, x1);
            const float h0 = __uint_as_float(hp << 16), h1 = __uint_as_float(hp & 0xffff0000u);
            h[e] = hp;
            l[e] = pack_bf16(x0 - h0, x1 - h1);
        }
        *reinterpret_cast<uint4 *>(hi_tile + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4 *>(lo_tile + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// The same for half a row: 16-byte chunks [4 half, 4 half + 4) of row u.
__device__ __forceinline__ void build_scaled_key_half(const uint8_t *ktile, uint8_t *hi_tile,
                                                      uint8_t *lo_tile, int u, int half, float w) {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        const uint32_t off = sw128_offset(u, (4 * half + cc) * 8);
        const uint4 raw = *reinterpret_cast<const uint4 *>(ktile + off);
        float f[8];
        Vec16<__nv_bfloat16>::unpack(raw, f);
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = f[2 * e] * w, x1 = f[2 * e + 1] * w;
            const uint32_t hp = pack_bf16(x0, x1);
            const float h0 = __uint_as_float(hp << 16), h1 = __uint_as_float(hp & 0xffff0000u);
            h[e] = hp;
            l[e] = pack_bf16(x0 - h0, x1 - h1);
        }
        *reinterpret_cast<uint4 *>(hi_tile + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4 *>(lo_tile + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// ============================================================================
// Span start states: S_pre(js) = sum over the spans u < js of
//   lam^(n_start(js) - e_end(u)) dA_u,  dA_u = sum of its parts,
// as the recurrence S_pre(js) = lam^(n_start(js) - n_start(js-1)) S_pre(js-1)
//                               + lam^(n_start(js) - e_end(js-1)) dA_(js-1).
// One thread per (b,h, element); spans in order, parts in index order.  The
// start state of span js is written over part 0 of span js-1 (the same thread
// has read that element already).
// ============================================================================
__global__ void __launch_bounds__(256) span_prefix_kernel(PrefixParams p) {
    griddep_launch_dependents();
    // decay coefficients per span, once per block: c1 for the previous start
    // state, c2 for the previous span's summary (lam^0 = 1 also for lam = 0)
    __shared__ float c1s[kMaxSpans], c2s[kMaxSpans];
    const int bh = blockIdx.y;
    const int h = bh % p.H;
    const int per_head = p.n_s - 1;
    if (threadIdx.x >= 1 && (int)threadIdx.x < p.n_s) {
        const int js = threadIdx.x;
        const SeqView sv = seq_view(p.vl, bh, p.H, p.T, js == 1 ? p.status : nullptr);
        const double l2l = log2((double)p.lam[h]);
        const int E = sv.T > p.W ? sv.T - p.W : 0;
        int a0, a1, b0, b1, z0, z1;
        span_range(js - 1, sv.nT, p.n_s, p.q_off / BM, a0, a1);
        span_range(js, sv.nT, p.n_s, p.q_off / BM, b0, b1);
        const int n_start = max(0, b0 * BM - p.W);
        const int e_end = max(0, min(E, a1 * BM - p.W));
        int n_prev = 0;
        if (js > 1) {
            span_range(js - 1, sv.nT, p.n_s, p.q_off / BM, z0, z1);
            n_prev = max(0, z0 * BM - p.W);
        }
        const int n1 = n_start - n_prev, n2 = n_start - e_end;
        c1s[js] = n1 == 0 ? 1.f : (float)exp2((double)n1 * l2l);
        c2s[js] = n2 == 0 ? 1.f : (float)exp2((double)n2 * l2l);
    }
    __syncthreads();
    const int x = blockIdx.x * blockDim.x + threadIdx.x;  // element of the 64 x 64 state
    if (x >= HD * HD) return;
    griddep_wait();  // the span summaries
    float acc = 0.f;
#pragma unroll 4
    for (int js = 1; js < p.n_s; ++js) {
        float *src = p.dA + ((size_t)(bh * per_head + js - 1) * p.n_parts) * HD * HD + x;
        float d = 0.f;
        for (int q = 0; q < p.n_parts; ++q) d += src[(size_t)q * HD * HD];
        acc = c1s[js] * acc + c2s[js] * d;
        src[0] = acc;
    }
}

// ============================================================================
// Pre-pass: dA_u = sum over the evictions e of span u of
//           eta lam^(e_end - 1 - e) k_e v_e^T     (e_end = end of span u)
// ============================================================================
constexpr int NS_SUM = 4;            // K/V stages of the summary kernel
constexpr int kSumTilesPerPart = 3;  // eviction tiles per span-summary part
constexpr int kSumThreads = 448;     // producer, MMA, 8 builder and 4 epilogue warps
constexpr uint32_t SOFF_KV = 0;
constexpr uint32_t SOFF_KT = SOFF_KV + NS_SUM * 2 * TILE_B;  // two buffers (hi, lo)
constexpr uint32_t SOFF_DS = SOFF_KT + 2 * 2 * TILE_B;       // float32 64x64 exchange
constexpr uint32_t SOFF_BAR = SOFF_DS + 16384;
constexpr uint32_t SMEM_SUM = SOFF_BAR + 256 + 1024;         // ~210 KB: one CTA per SM

// Where the evictions of one summary part lie: span js of row bh, part
// `part` of its n_parts; ev_first / ne its eviction tiles, e_end the end of
// the span's evictions (every part decays to it, so the parts add up to the
// span's summary).
struct SumSlot {
    SeqView sv;
    int bh, ev_first, ne, e_end;
};
__device__ __forceinline__ SumSlot sum_slot(const SumParams &p, int slot, int *status) {
    SumSlot q;
    const int per_head = p.n_s - 1;
    const int part = slot % p.n_parts;
    const int js = (slot / p.n_parts) % per_head;
    q.bh = slot / (per_head * p.n_parts);
    q.sv = seq_view(p.vl, q.bh, p.H, p.T, status);
    int i0, i1;
    span_range(js, q.sv.nT, p.n_s, p.q_off / BM, i0, i1);
    const int E = q.sv.T > p.W ? q.sv.T - p.W : 0;
    const int ev_span = i0 > p.W / BM ? i0 : p.W / BM;  // first tile of the span with evictions
    const int ne_span = i1 > ev_span ? i1 - ev_span : 0;
    q.ev_first = ev_span + (int)((long long)ne_span * part / p.n_parts);
    q.ne = ev_span + (int)((long long)ne_span * (part + 1) / p.n_parts) - q.ev_first;
    q.e_end = ne_span > 0 ? min(E, i1 * BM - p.W) : 0;
    return q;
}

// Persistent CTAs, one per SM, each taking parts blockIdx.x, + gridDim.x, ...
// Roles: warp 0 loads K/V tiles through an NS_SUM-stage ring; warps 2-9
// build the scaled hi/lo keys (half a row per thread, two warps per SM
// sub-partition to hide the build's latency) into two alternating buffers;
// warp 1 accumulates a part's tiles into one of two TMEM accumulators;
// warps 10-13 read a finished accumulator, add its hi and lo rows and store
// the part.  So the loads, builds, MMAs and stores of consecutive tiles and
// parts overlap.
__global__ void __launch_bounds__(kSumThreads, 1)
    span_summary_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                        const __grid_constant__ CUtensorMap tkh,
                        const __grid_constant__ CUtensorMap tvh, SumParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-aligned base by pointer arithmetic on the shared array itself, so
    // that the compiler keeps the shared address space (ld/st.shared) for
    // every access derived from it
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SOFF_BAR);
    uint64_t *kv_full = bars, *kv_empty = bars + NS_SUM;
    uint64_t *kt_full = bars + 2 * NS_SUM, *kt_empty = kt_full + 2;
    uint64_t *acc_full = kt_empty + 2, *acc_empty = acc_full + 2, *done = acc_empty + 2;
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(done + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    float *sDS = reinterpret_cast<float *>(sm + SOFF_DS);

    griddep_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5;
    const int n_slots = p.BH * (p.n_s - 1) * p.n_parts;
    const bool varlen = p.vl.cu != nullptr;

    if (tid == 0) {
        for (int s = 0; s < NS_SUM; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&kt_full[b], 256);
            mbar_init(&kt_empty[b], 1);
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        mbar_init(done, 1);
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
        // ------------------------------------------------------------ producer
        if (tid == 0) {
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            uint32_t g = 0;
            bool ok = true;
            for (int slot = blockIdx.x; slot < n_slots && ok; slot += gridDim.x) {
                const SumSlot q = sum_slot(p, slot, nullptr);
                for (int e = 0; e < q.ne; ++e, ++g) {
                    const int s = g % NS_SUM;
                    if (!(ok = mbar_wait(&kv_empty[s], ((g / NS_SUM) & 1) ^ 1, abort, p.status, p.wait_ns))) break;
                    const int n0 = (q.ev_first + e) * BM - p.W;
                    mbar_expect_tx(&kv_full[s], 2 * TILE_B);
                    load_kv_tile(sm + SOFF_KV + s * 2 * TILE_B, &tk, &tv, &tkh, &tvh, &kv_full[s],
                                 n0 / BM, p.q_off, q.sv, varlen);
                }
            }
            // every issued copy lands before the CTA exits
            for (uint32_t st = 0; st < NS_SUM; ++st) {
                const uint32_t fills = g > st ? (g - 1 - st) / NS_SUM + 1 : 0;
                if (fills) mbar_wait_drain(&kv_full[st], (fills - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t id_ds = idesc_bf16(128, 64, true, true);
        uint32_t g = 0, nz = 0;
        bool ok = true;
        for (int slot = blockIdx.x; slot < n_slots && ok; slot += gridDim.x) {
            const SumSlot q = sum_slot(p, slot, nullptr);
            if (q.ne == 0) continue;
            const uint32_t acc = tb + 64 * (nz & 1);
            for (int e = 0; e < q.ne; ++e, ++g) {
                const int s = g % NS_SUM, b = g & 1;
                if (!(ok = warp_wait(&kt_full[b], (g >> 1) & 1, abort, p.status, p.wait_ns))) break;
                if (e == 0 && !(ok = warp_wait(&acc_empty[nz & 1], ((nz >> 1) & 1) ^ 1, abort, p.status, p.wait_ns))) break;
                tc_fence_after();
                const uint64_t ktd = sdesc_sw128(smem_u32(sm + SOFF_KT + b * 2 * TILE_B), TILE_B, 1024);
                const uint64_t vd = sdesc_sw128(smem_u32(sm + SOFF_KV + s * 2 * TILE_B + TILE_B), TILE_B, 1024);
                mma_ss_w(acc, ktd, vd, id_ds, e > 0);
#pragma unroll
                for (int k = 1; k < 8; ++k) mma_ss_w(acc, ktd + 128 * k, vd + 128 * k, id_ds, 1);
                mma_commit_w(&kt_empty[b]);
                mma_commit_w(&kv_empty[s]);
                if (e == q.ne - 1) mma_commit_w(&acc_full[nz & 1]);
            }
            ++nz;
        }
        // nothing may still run on the tensor cores when TMEM is released
        mma_commit_w(done);
        mbar_wait_drain(done, 0);
    } else if (warp >= 2 && warp < 10) {
        // ------------------------------------------------------------ key builders
        const int u = (tid - 64) & 127, half = (tid - 64) >> 7;  // key row, half of it
        uint32_t g = 0;
        bool ok = true;
        for (int slot = blockIdx.x; slot < n_slots && ok; slot += gridDim.x) {
            const SumSlot q = sum_slot(p, slot, tid == 64 ? p.status : nullptr);
            if (q.ne == 0) continue;
            const int h = q.bh % p.H;
            const float l2l = (float)log2((double)p.lam[h]);
            const float eta = p.eta[h];
            for (int e = 0; e < q.ne; ++e, ++g) {
                const int s = g % NS_SUM, b = g & 1;
                if (!(ok = mbar_wait(&kv_full[s], (g / NS_SUM) & 1, abort, p.status, p.wait_ns))) break;
                if (!(ok = mbar_wait(&kt_empty[b], ((g >> 1) & 1) ^ 1, abort, p.status, p.wait_ns))) break;
                const int ev = (q.ev_first + e) * BM - p.W + u;
                // float exp2: relative error ~1e-7 for the weights that matter (the
                // exponent error grows with the decay, and decayed terms are small)
                const float w = ev < q.e_end ? eta * exp2f((float)(q.e_end - 1 - ev) * l2l) : 0.f;
                uint8_t *kt = sm + SOFF_KT + b * 2 * TILE_B;
                build_scaled_key_half(sm + SOFF_KV + s * 2 * TILE_B, kt, kt + TILE_B, u, half, w);
                fence_async_smem();
                mbar_arrive(&kt_full[b]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // TMEM lane L = row of the accumulator: L < 64 the hi part of state row
        // L, L >= 64 the lo part of state row L - 64.  A wait that gives up sets
        // `failed`; the next barrier (named barrier 1, these 128 threads) tells
        // all, and all leave together.
        const int L = 32 * (warp & 3) + (tid & 31);
        uint32_t nz = 0;
        bool failed = false;
        for (int slot = blockIdx.x; slot < n_slots; slot += gridDim.x) {
            const SumSlot q = sum_slot(p, slot, nullptr);
            float *out = p.dA + (size_t)slot * HD * HD;
            if (q.ne == 0) {
                if (L < 64) {
                    float4 *dst = reinterpret_cast<float4 *>(out + L * HD);
#pragma unroll
                    for (int c = 0; c < 16; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                continue;
            }
            if (!failed && !warp_wait(&acc_full[nz & 1], (nz >> 1) & 1, abort, p.status, p.wait_ns))
                failed = true;
            tc_fence_after();
            float v[64];
            if (!failed) {
                uint32_t r[32];
                const uint32_t acc = tb + 64 * (nz & 1);
                tmem_ld32(tmem_addr(acc, 32 * (warp & 3), 0), r);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) v[c] = __uint_as_float(r[c]);
                tmem_ld32(tmem_addr(acc, 32 * (warp & 3), 32), r);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) v[32 + c] = __uint_as_float(r[c]);
            }
            // the previous part's readers of sDS are done
            if (bar_any(1, 128, failed)) break;
            if (L >= 64) {
#pragma unroll
                for (int c = 0; c < 64; ++c) sDS[c * 64 + (L - 64)] = v[c];
            }
            // the accumulator is read: the MMA issuer may start the part after next in it
            tc_fence_before();
            mbar_arrive(&acc_empty[nz & 1]);
            if (bar_any(1, 128, false)) break;
            if (L < 64) {
                float4 *dst = reinterpret_cast<float4 *>(out + L * HD);
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    dst[c] = make_float4(v[4 * c] + sDS[(4 * c) * 64 + L], v[4 * c + 1] + sDS[(4 * c + 1) * 64 + L],
                                         v[4 * c + 2] + sDS[(4 * c + 2) * 64 + L],
                                         v[4 * c + 3] + sDS[(4 * c + 3) * 64 + L]);
            }
            ++nz;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, 128);
}

// ============================================================================
// Main kernel
// ============================================================================
__global__ void __launch_bounds__(kMainThreads, 1)
    prefill_main_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tkh,
                        const __grid_constant__ CUtensorMap tvh, MainParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-aligned base by pointer arithmetic on the shared array itself, so
    // that the compiler keeps the shared address space (ld/st.shared) for
    // every access derived from it
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *q_full = bars, *q_empty = bars + 2;
    uint64_t *kv_full = bars + 4, *kv_empty = kv_full + NS;
    uint64_t *s_full = kv_empty + NS, *p_full = s_full + 2;
    uint64_t *o_prog = p_full + 2, *o_full = o_prog + 1, *o_empty = o_full + 1;
    uint64_t *sst_full = o_empty + 1, *kt_full = sst_full + 1, *ds_full = kt_full + 1;
    uint64_t *lead_ready = ds_full + 1, *mma_done = lead_ready + 1;
    uint32_t *tmem_base = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_base + 1);
    float *epw = reinterpret_cast<float *>(sm + OFF_EPW);
    float *sDS = reinterpret_cast<float *>(sm + OFF_DS);

    const int tid = threadIdx.x, warp = tid >> 5;
    const bool l1_only = p.l1_only != 0;
    const int n_spans = p.BH * p.n_s;
    const bool varlen = p.vl.cu != nullptr;

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], 1);
            mbar_init(&q_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 256);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(o_prog, 1);
        mbar_init(o_full, 1);
        mbar_init(o_empty, 256);
        mbar_init(sst_full, 128);
        mbar_init(kt_full, 128);
        mbar_init(ds_full, 1);
        mbar_init(lead_ready, 1);
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
        // ------------------------------------------------------------ producer
        if (tid == 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            if (p.q_off > 0) {
                tma_prefetch_desc(&tkh);
                tma_prefetch_desc(&tvh);
            }
            uint32_t tile = 0, kc = 0;
            bool ok = true;
            Span spn;
            for (int ks = 0; ok && cta_span(ks, n_spans, p.n_s, p.order, spn); ++ks) {
                const int bh = spn.bh;
                const SeqView sv = seq_view(p.vl, bh, p.H, p.T, nullptr);
                int i0, i1;
                span_range(spn.js, sv.nT, p.n_s, p.q_off / BM, i0, i1);
                for (int i = i0; i < i1 && ok; ++i, ++tile) {
                    const TileInfo ti = tile_info(i, p.W, l1_only);
                    const int qb = tile & 1;
                    if (!(ok = mbar_wait(&q_empty[qb], ((tile >> 1) & 1) ^ 1, abort, p.status, p.wait_ns))) break;
                    mbar_expect_tx(&q_full[qb], TILE_B);
                    tma_rows(sm + OFF_Q + qb * TILE_B, &tq, &q_full[qb], ti.t0 - p.q_off, sv, varlen);
                    for (int j = 0; j < ti.nk; ++j, ++kc) {
                        const int s = kc % NS;
                        if (!(ok = mbar_wait(&kv_empty[s], ((kc / NS) & 1) ^ 1, abort, p.status, p.wait_ns))) break;
                        uint8_t *dst = sm + OFF_KV + s * 2 * TILE_B;
                        mbar_expect_tx(&kv_full[s], 2 * TILE_B);
                        load_kv_tile(dst, &tk, &tv, &tkh, &tvh, &kv_full[s], ti.kt0 + j, p.q_off, sv, varlen);
                    }
                }
            }
            // every issued copy must land before the CTA exits (normally the
            // MMA side has already waited for all of them)
            for (uint32_t st = 0; st < NS; ++st) {
                const uint32_t fills = kc > st ? (kc - 1 - st) / NS + 1 : 0;
                if (fills) mbar_wait_drain(&kv_full[st], (fills - 1) & 1);
            }
            for (uint32_t b = 0; b < 2; ++b) {
                const uint32_t fills = tile > b ? (tile - 1 - b) / 2 + 1 : 0;
                if (fills) mbar_wait_drain(&q_full[b], (fills - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // One flat stream over the CTA's key tiles: Q K^T of key tile g is
        // issued before P V of key tile g-1, also across query tiles, so the
        // next tile's first scores are ready when the softmax side finishes
        // the current tile.  Q K^T of tile g+1 overwrites the score buffer
        // whose P (and P') the P V (and P'V) of tile g-1 reads; it is issued
        // right after them without waiting for their completion, because the
        // tensor core runs one thread's MMAs in issue order.
        {
            const uint32_t id_qk = idesc_bf16(128, 128, false, false);
            const uint32_t id_pv = idesc_bf16(128, 64, false, true);
            const uint32_t id_qs = idesc_bf16(128, 64, false, true);
            const uint32_t id_ds = idesc_bf16(128, 64, true, true);
            const uint32_t sb_addr = smem_u32(sm + OFF_SB);
            const uint32_t kt_addr = smem_u32(sm + OFF_KT);
            const uint32_t q_base = smem_u32(sm + OFF_Q), kv_base = smem_u32(sm + OFF_KV);
            uint32_t tile = 0, g = 0, lc = 0;
            bool ok = true;
            // the key tile whose P V is still to be issued
            struct Pending {
                bool valid, first, last, l2;
                uint32_t g, tile;
            } pend = {false, false, false, false, 0, 0};
            auto pv_step = [&](const Pending &pv) -> bool {
                const int sb = pv.g & 1, s = pv.g % NS;
                if (!warp_wait(&p_full[sb], (pv.g >> 1) & 1, abort, p.status, p.wait_ns)) return false;
                if (pv.first && !warp_wait(o_empty, (pv.tile & 1) ^ 1, abort, p.status, p.wait_ns)) return false;
                tc_fence_after();
                const uint32_t v_addr = kv_base + s * 2 * TILE_B + TILE_B;
                const uint32_t s_col = tb + TM_S + sb * 128;
                // Issue loops are unrolled with the descriptors stepped by
                // constants (+2048 bytes of a K/V tile = +128 in the address
                // field): a rolled loop that rebuilds each descriptor takes more
                // than twice as long to issue the same MMAs.
                const uint64_t vd = sdesc_sw128(v_addr, TILE_B, 1024);
                mma_ts_w(tb + TM_O, s_col, vd, id_pv, !pv.first);
#pragma unroll
                for (int k = 1; k < 8; ++k) mma_ts_w(tb + TM_O, s_col + 8 * k, vd + 128 * k, id_pv, 1);
                if (pv.first && pv.l2) {
                    const uint32_t q_addr = q_base + (pv.tile & 1) * TILE_B;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_ts_w(tb + TM_MI, s_col + 64 + 8 * k, vd + 128 * k, id_pv, k > 0);
                    if (!warp_wait(sst_full, lc & 1, abort, p.status, p.wait_ns)) return false;
                    tc_fence_after();
                    const uint64_t qd = sdesc_sw128(q_addr, 16, 1024), sd = sdesc_sw128(sb_addr, 8192, 1024);
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma_ss_w(tb + TM_MX, qd + 2 * k, sd + 128 * k, id_qs, k > 0);
                    if (!warp_wait(kt_full, lc & 1, abort, p.status, p.wait_ns)) return false;
                    tc_fence_after();
                    const uint64_t ktd = sdesc_sw128(kt_addr, TILE_B, 1024);
#pragma unroll
                    for (int k = 0; k < 8; ++k) mma_ss_w(tb + TM_DS, ktd + 128 * k, vd + 128 * k, id_ds, k > 0);
                    mma_commit_w(ds_full);
                    ++lc;
                }
                mma_commit_w(o_prog);
                mma_commit_w(&kv_empty[s]);
                if (pv.last) {
                    mma_commit_w(&q_empty[pv.tile & 1]);
                    mma_commit_w(o_full);
                }
                return true;
            };
            Span spn;
            for (int ks = 0; ok && cta_span(ks, n_spans, p.n_s, p.order, spn); ++ks) {
                const SeqView sv = seq_view(p.vl, spn.bh, p.H, p.T, nullptr);
                int i0, i1;
                span_range(spn.js, sv.nT, p.n_s, p.q_off / BM, i0, i1);
                for (int i = i0; i < i1 && ok; ++i, ++tile) {
                    const TileInfo ti = tile_info(i, p.W, l1_only);
                    const int qb = tile & 1;
                    const uint32_t q_addr = q_base + qb * TILE_B;
                    if (!(ok = warp_wait(&q_full[qb], (tile >> 1) & 1, abort, p.status, p.wait_ns))) break;
                    for (int j = 0; j < ti.nk && ok; ++j, ++g) {
                        const int s = g % NS, sb = g & 1;
                        if (!(ok = warp_wait(&kv_full[s], (g / NS) & 1, abort, p.status, p.wait_ns))) break;
                        // the state warps read the leading key tile: hand it on
                        if (j == 0 && ti.l2) mbar_arrive_w(lead_ready);
                        tc_fence_after();
                        const uint32_t k_addr = kv_base + s * 2 * TILE_B;
                        const uint64_t qd = sdesc_sw128(q_addr, 16, 1024), kd = sdesc_sw128(k_addr, 16, 1024);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_ss_w(tb + TM_S + sb * 128, qd + 2 * k, kd + 2 * k, id_qk, k > 0);
                        mma_commit_w(&s_full[sb]);
                        if (pend.valid && !(ok = pv_step(pend))) break;
                        pend = {true, j == 0, j == ti.nk - 1, ti.l2, g, tile};
                    }
                }
            }
            if (ok && pend.valid) ok = pv_step(pend);
            // nothing may still run on the tensor cores when TMEM is released
            mma_commit_w(mma_done);
            mbar_wait_drain(mma_done, 0);
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------------------ softmax + epilogue
        // two warpgroups; half h = 0 (warps 4-7) / 1 (warps 8-11) owns score
        // columns 64h.., output columns 32h..; both see every row r (TMEM lane)
        const int half = (warp - 4) >> 2;
        const int r = tid - 128 - 128 * half;
        const int lane_base = 32 * (warp & 3);
        const float sl2 = kLog2e * rsqrtf((float)HD);
        float *xm = reinterpret_cast<float *>(sm + OFF_XM);
        float *xl = reinterpret_cast<float *>(sm + OFF_XL);
        uint32_t tile = 0, kc = 0;
        bool ok = true;
        // The epilogue of a tile runs after the first key tile of the next one,
        // so the wait for the tile's last P V product overlaps useful work.
        struct Epi {
            bool valid, l2;
            int t0, bh, T, row0;  // T, row0: the row's sequence (SeqView)
            float gate, pw_r1, l;
            uint32_t tile;
        } pe = {false, false, 0, 0, 0, 0, 0.f, 0.f, 0.f, 0};
        // A bounded wait that gives up sets `failed`; the thread carries on to
        // the next softmax barrier, which tells every softmax thread, and all
        // 256 leave their loops right after that barrier.  So every one of them
        // passes the same sequence of barriers.
        bool failed = false;
        auto epilogue = [&](const Epi &e) -> bool {  // false: all softmax threads stop
            // y = O / l + sigmoid(g) (m_intra + lam^(r+1) m_inter)
            // (between two epilogues every thread passes a key-tile barrier, so
            // one xl buffer suffices)
            xl[half * 128 + r] = e.l;
            if (bar_any(1, 256, failed)) return false;
            const float inv_l = 1.0f / (e.l + xl[(1 - half) * 128 + r]);
            if (!warp_wait(o_full, e.tile & 1, abort, p.status, p.wait_ns)) {
                failed = true;
                return true;
            }
            tc_fence_after();
            float yv[32];
            uint32_t rr[32];
            tmem_ld32(tmem_addr(tb, lane_base, TM_O + 32 * half), rr);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) yv[c] = __uint_as_float(rr[c]) * inv_l;
            if (e.l2) {
                uint32_t rx[32];
                tmem_ld32(tmem_addr(tb, lane_base, TM_MI + 32 * half), rr);
                tmem_ld32(tmem_addr(tb, lane_base, TM_MX + 32 * half), rx);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    yv[c] += e.gate * (__uint_as_float(rr[c]) + e.pw_r1 * __uint_as_float(rx[c]));
            }
            tc_fence_before();
            mbar_arrive(o_empty);
            const int t = e.t0 + r;
            if (t < e.T) {
                // fixed length: [BH][T_new][64]; variable length: [total][H][64]
                const size_t row = varlen ? ((size_t)(e.row0 + t) * p.H + e.bh % p.H)
                                          : ((size_t)e.bh * (size_t)(p.T - p.q_off) + (t - p.q_off));
                uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.y) +
                                                       row * HD + 32 * half);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    dst[c] = make_uint4(pack_bf16(yv[8 * c], yv[8 * c + 1]),
                                        pack_bf16(yv[8 * c + 2], yv[8 * c + 3]),
                                        pack_bf16(yv[8 * c + 4], yv[8 * c + 5]),
                                        pack_bf16(yv[8 * c + 6], yv[8 * c + 7]));
            }
            return true;
        };
        Span spn;
        for (int ks = 0; ok && cta_span(ks, n_spans, p.n_s, p.order, spn); ++ks) {
            const int bh = spn.bh, h = bh % p.H;
            const SeqView sv = seq_view(p.vl, bh, p.H, p.T, nullptr);
            int i0, i1;
            span_range(spn.js, sv.nT, p.n_s, p.q_off / BM, i0, i1);
            const double lam = p.lam[h];
            const float gate = 1.0f / (1.0f + expf(-p.g[h]));
            const float pw_r1 = (float)pow(lam, (double)(r + 1));
            // previous span done with epw, then publish this head's table
            if (bar_any(1, 256, failed)) {
                ok = false;
                break;
            }
            if (half == 0)
                epw[128 + r] = (float)((double)p.eta[h] * pow(lam, (double)r));
            else
                epw[r] = 0.f;
            if (bar_any(1, 256, failed)) {
                ok = false;
                break;
            }
            for (int i = i0; i < i1 && ok; ++i, ++tile) {
                const TileInfo ti = tile_info(i, p.W, l1_only);
                float m_used = -INFINITY, l = 0.f;
                for (int j = 0; j < ti.nk && ok; ++j, ++kc) {
                    const int sb = kc & 1;
                    // (on a timeout the scores read below are stale, and unused)
                    if (!warp_wait(&s_full[sb], (kc >> 1) & 1, abort, p.status, p.wait_ns)) failed = true;
                    tc_fence_after();
                    const uint32_t s_col = TM_S + sb * 128;
                    float s[64];
                    {
                        uint32_t ra[32], rb[32];
                        tmem_ld32(tmem_addr(tb, lane_base, s_col + 64 * half), ra);
                        tmem_ld32(tmem_addr(tb, lane_base, s_col + 64 * half + 32), rb);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            s[c] = __uint_as_float(ra[c]);
                            s[32 + c] = __uint_as_float(rb[c]);
                        }
                    }
                    const int kind = (j == 0 && ti.lead) ? (ti.l2 ? KIND_LEAD_L2 : KIND_LEAD)
                                                         : (j == ti.nk - 1 ? KIND_DIAG : KIND_FULL);
                    const int skind = slice_kind(kind, r - 64 * half);
                    const float mh = half_max(skind, s, r - 64 * half);
                    float *xmk = xm + (kc & 1) * 256;
                    xmk[half * 128 + r] = mh;
                    if (bar_any(1, 256, failed)) {
                        ok = false;
                        break;
                    }
                    const float mt = fmaxf(mh, xmk[(1 - half) * 128 + r]) * sl2;  // sl2 > 0
                    // Raise the row's reference max only when it grew by more than
                    // 2^kRescale; rows whose O already holds earlier P V products
                    // are rescaled in TMEM (each half its 32 columns of O).  TMEM
                    // access is warp-collective, so the warp rescales together.
                    const bool raise = mt > m_used + kRescale;
                    const bool resc = raise && m_used != -INFINITY && j > 0;
                    const float fo = resc ? ex2(m_used - mt) : 1.0f;
                    if (__any_sync(0xffffffffu, resc)) {
                        if (warp_wait(o_prog, (kc - 1) & 1, abort, p.status, p.wait_ns)) {
                            tc_fence_after();
                            uint32_t rr[32];
                            tmem_ld32(tmem_addr(tb, lane_base, TM_O + 32 * half), rr);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                rr[c] = __float_as_uint(__uint_as_float(rr[c]) * fo);
                            tmem_st32(tmem_addr(tb, lane_base, TM_O + 32 * half), rr);
                        } else {
                            failed = true;  // skip the P work, still reach every barrier
                        }
                    }
                    if (!failed) {
                        l *= fo;
                        if (raise) m_used = mt;
                        const uint32_t p_addr = tmem_addr(tb, lane_base, s_col + 32 * half);
                        l += half_p(skind, s, r - 64 * half, sl2, m_used, p_addr);
                        if (kind == KIND_LEAD_L2) write_plin(s, r - 64 * half, epw, p_addr + 64);
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&p_full[sb]);
                    }
                    if (j == 0 && pe.valid) {
                        pe.valid = false;
                        if (!(ok = epilogue(pe))) break;
                    }
                }
                if (!ok) break;
                pe = {true, ti.l2, ti.t0, bh, sv.T, sv.row0, gate, pw_r1, l, tile};
            }
        }
        if (pe.valid) epilogue(pe);  // every softmax thread: pe.valid is the same for all

    } else if (warp >= 12) {
        // ------------------------------------------------------------ state
        const int u = tid - 384;  // TMEM lane; u < 64 owns row u of S
        uint32_t kc = 0, lc = 0;
        bool ok = true;
        // as in the softmax warps: a wait that gives up sets `failed`, the next
        // state barrier (named barrier 2, 128 threads) tells all, and all leave
        // right after it
        bool failed = false;
        uint8_t *sb_tile = sm + OFF_SB;
        uint8_t *kt_hi = sm + OFF_KT, *kt_lo = sm + OFF_KT + TILE_B;
        float S[64];
        Span spn;
        for (int ks = 0; ok && cta_span(ks, n_spans, p.n_s, p.order, spn); ++ks) {
            const int bh = spn.bh, h = bh % p.H, js = spn.js;
            // the state warps report rows with inconsistent offsets (once per span)
            const SeqView sv = seq_view(p.vl, bh, p.H, p.T, u == 0 ? p.status : nullptr);
            const int E = sv.T > p.W ? sv.T - p.W : 0;
            int i0, i1;
            span_range(js, sv.nT, p.n_s, p.q_off / BM, i0, i1);
            const double lam = p.lam[h];
            const double l2l = log2(lam);
            // per-span tables (float math in the tile loop only): ew[k] = eta lam^k,
            // lp[k] = lam^k; the previous span is done with them after its last consume
            float *ew = reinterpret_cast<float *>(sm + OFF_STT), *lp = ew + 128;
            ew[u] = (float)((double)p.eta[h] * exp2((double)u * l2l));
            lp[u] = (float)exp2((double)u * l2l);
            if (u == 0) lp[128] = (float)exp2(128.0 * l2l);
            if (bar_any(2, 128, failed)) {
                ok = false;
                break;
            }
            // state at the span start from the predecessors' summaries
            const int n_start = max(0, i0 * BM - p.W);
#pragma unroll
            for (int c = 0; c < 64; ++c) S[c] = 0.f;
            if (!l1_only && u < 64 && p.A_init) {
                // the given state before the first eviction, decayed to the span start
                const float coef = (float)exp2((double)n_start * l2l);
                const float *src = p.A_init + ((size_t)bh * HD + u) * HD;
#pragma unroll
                for (int c = 0; c < 64; ++c) S[c] = coef * src[c];
            }
            if (!l1_only && u < 64 && js > 0) {
                // the predecessors' evictions, from span_prefix_kernel
                griddep_wait();
                const float *src =
                    p.S_pre + (((size_t)(bh * (p.n_s - 1) + js - 1) * p.n_parts) * HD + u) * HD;
#pragma unroll
                for (int c = 0; c < 64; ++c) S[c] += src[c];
            }
            bool have_prev = false;
            int c_prev = 0;
            auto consume = [&](int c_eff) -> bool {  // false: all state threads stop
                // rows 64..127 of the increment (lo parts) go through shared
                // memory to the owners of rows 0..63 (hi parts)
                if (!warp_wait(ds_full, (lc - 1) & 1, abort, p.status, p.wait_ns)) failed = true;
                tc_fence_after();
                uint32_t rr[32];
                if (u >= 64 && !failed) {
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                        tmem_ld32(tmem_addr(tb, 32 * (warp & 3), TM_DS + c0), rr);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) sDS[(c0 + c) * 64 + (u - 64)] = __uint_as_float(rr[c]);
                    }
                }
                if (bar_any(2, 128, failed)) return false;
                if (u < 64) {
                    const float dec = lp[c_eff];
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                        tmem_ld32(tmem_addr(tb, 32 * (warp & 3), TM_DS + c0), rr);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            S[c0 + c] = fmaf(dec, S[c0 + c],
                                             __uint_as_float(rr[c]) + sDS[(c0 + c) * 64 + u]);
                    }
                }
                return !bar_any(2, 128, false);
            };
            for (int i = i0; i < i1 && ok; ++i) {
                const TileInfo ti = tile_info(i, p.W, l1_only);
                if (ti.l2) {
                    if (have_prev && !(ok = consume(c_prev))) break;
                    // stage S(n0) as bf16 for the inter read (row k = u, 64 columns n)
                    if (u < 64) {
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            *reinterpret_cast<uint4 *>(sb_tile + sw128_offset(u, ch * 8)) =
                                make_uint4(pack_bf16(S[8 * ch], S[8 * ch + 1]),
                                           pack_bf16(S[8 * ch + 2], S[8 * ch + 3]),
                                           pack_bf16(S[8 * ch + 4], S[8 * ch + 5]),
                                           pack_bf16(S[8 * ch + 6], S[8 * ch + 7]));
                    }
                    fence_async_smem();
                    mbar_arrive(sst_full);
                    // scaled keys of the leading tile for the state MMA
                    const int s = kc % NS;
                    if (!warp_wait(lead_ready, lc & 1, abort, p.status, p.wait_ns)) failed = true;
                    const int n0 = ti.t0 - p.W;
                    const int c_eff = min(BM, E - n0);
                    if (!failed) {
                        const float w = u < c_eff ? ew[c_eff - 1 - u] : 0.f;
                        build_scaled_key_row(sm + OFF_KV + s * 2 * TILE_B, kt_hi, kt_lo, u, w);
                        fence_async_smem();
                        mbar_arrive(kt_full);
                    }
                    have_prev = true;
                    c_prev = c_eff;
                    ++lc;
                }
                kc += ti.nk;
            }
            if (!ok) break;
            if (have_prev && !(ok = consume(c_prev))) break;
            if (!l1_only && js == p.n_s - 1 && u < 64 && p.A_final) {
                float4 *dst = reinterpret_cast<float4 *>(p.A_final + ((size_t)bh * HD + u) * HD);
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, 512);
}

// ============================================================================
// Row order of a variable-length call: the sequences by decreasing length
// (ties by index), the H heads of each together, so that the main kernel
// deals the longest spans out first.  One block; for more than kOrderMax
// sequences the rows keep their index order.
// ============================================================================
constexpr int kOrderMax = 4096;
__global__ void __launch_bounds__(1024) varlen_order_kernel(Varlen vl, int B, int H, int *order) {
    __shared__ unsigned long long key[kOrderMax];
    const int tid = threadIdx.x;
    if (B > kOrderMax) {
        for (int x = tid; x < B * H; x += blockDim.x) order[x] = x;
        return;
    }
    int n = 1;
    while (n < B) n <<= 1;
    for (int b = tid; b < n; b += blockDim.x) {
        unsigned long long k = ~0ull;  // padding sorts last
        if (b < B) {
            const int64_t a = vl.cu[b], e = vl.cu[b + 1];
            const bool okb = a >= 0 && e >= a && e <= vl.total && e - a <= vl.max_len;
            const unsigned len = okb ? (unsigned)(e - a) : 0u;
            k = ((unsigned long long)(0x7fffffffu - len) << 32) | (unsigned)b;
        }
        key[b] = k;
    }
    __syncthreads();
    // bitonic sort, ascending keys = descending lengths
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < n; i += blockDim.x) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool up = (i & size) == 0;
                    const unsigned long long x = key[i], y = key[j];
                    if ((x > y) == up) {
                        key[i] = y;
                        key[j] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int x = tid; x < B * H; x += blockDim.x)
        order[x] = (int)(key[x / H] & 0xffffffffu) * H + x % H;
}

// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() { return reinterpret_cast<EncodeTiledFn>(tensor_map_encoder()); }

// [BH][T][64] bf16 -> 3D map with 64 x 128 x 1 boxes, 128-byte swizzle;
// rows past T read as zero.
bool make_map(CUtensorMap *m, const void *base, int T, int BH) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)T * HD * 2};
    cuuint32_t box[3] = {HD, BM, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Packed [total][H][64] bf16 (variable-length calls) -> 3D map over
// (column, head, token) with 64 x 1 x 128 boxes: the same shared-memory tile
// as make_map's, 128 token rows of one head; rows past total read as zero.
bool make_map_packed(CUtensorMap *m, const void *base, int64_t total, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)H, (cuuint64_t)total};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)H * HD * 2};
    cuuint32_t box[3] = {HD, 1, BM};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Spans per head: minimise the work of the busiest CTA, counting each span as
// its tiles plus a fixed start-up cost (pipeline fill, the pre-pass summary it
// needs and the combine of its predecessors' summaries); ties go to fewer spans.
constexpr int kSpanOverheadTiles = 2;
int choose_spans(int64_t BH, int nT, int num_sms) {
    int best = 1;
    int64_t best_cost = INT64_MAX;
    for (int ns = 1; ns <= nT && ns <= kMaxSpans; ++ns) {
        const int64_t spans = BH * ns;
        const int64_t G = spans < num_sms ? spans : num_sms;
        const int64_t per_cta = (spans + G - 1) / G;
        const int64_t cost = per_cta * ((nT + ns - 1) / ns + kSpanOverheadTiles);
        if (cost < best_cost) {
            best_cost = cost;
            best = ns;
        }
    }
    return best;
}

}  // namespace

void *tensor_map_encoder() {
    static void *fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = ptr;
    }
    return fn;
}

bool sm100_supported(const tc_prefill_desc &d, int64_t n_halo) {
    return d.dtype == TC_BF16 && d.dk == HD && d.dv == HD && d.W >= BM && d.W % BM == 0 &&
           d.T >= 1 && d.T + n_halo <= (int64_t(1) << 30) && d.B * d.H <= 65535 &&
           (n_halo == 0 || n_halo == d.W) &&
           !(d.flags & (TC_PREFILL_STATE_ONLY | TC_PREFILL_DELTA_RULE));
}

// Spans are cut over the new query tiles only (the halo has no queries).
static int spans_for(const tc_prefill_desc &d, int num_sms) {
    const int nT_new = (int)((d.T + BM - 1) / BM);
    return choose_spans(d.B * d.H, nT_new, num_sms);
}

// Parts per span summary: about kSumTilesPerPart eviction tiles per CTA, and
// at most about 4 CTAs per SM in all (which also bounds the workspace).
static int parts_for(int nT_new, int ns, int64_t BH, int num_sms) {
    const int tiles = (nT_new + ns - 1) / ns;
    int parts = (tiles + kSumTilesPerPart - 1) / kSumTilesPerPart;
    const int64_t cap = (int64_t)4 * num_sms / (BH * (ns - 1));
    if (parts > cap) parts = (int)cap;
    return parts < 1 ? 1 : (parts > 16 ? 16 : parts);
}

// Summary parts; for a variable-length call the row order follows them.
static size_t summary_bytes(const tc_prefill_desc &d, int num_sms) {
    if (d.flags & TC_PREFILL_L1_ONLY) return 0;
    const int ns = spans_for(d, num_sms);
    if (ns <= 1) return 0;
    const int nT_new = (int)((d.T + BM - 1) / BM);
    const int64_t BH = d.B * d.H;
    const size_t mats = (size_t)BH * (ns - 1) * parts_for(nT_new, ns, BH, num_sms);
    return mats * HD * HD * sizeof(float);
}

size_t sm100_workspace_bytes(const tc_prefill_desc &d, int num_sms, bool varlen) {
    const size_t sum = summary_bytes(d, num_sms);
    if (!varlen) return sum;
    return (sum + 255) / 256 * 256 + (size_t)(d.B * d.H) * sizeof(int);
}

int sm100_launch_count(const tc_prefill_desc &d) {
    const bool l1 = (d.flags & TC_PREFILL_L1_ONLY) != 0;
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    else
        cudaGetLastError();
    return 1 + ((!l1 && spans_for(d, sms) > 1) ? 2 : 0);
}

cudaError_t launch_prefill_sm100(const PrefillParams &p, int num_sms, cudaStream_t s) {
    const int64_t BH = p.B * p.H;
    const int q_off = (int)p.n_halo;
    const int T_all = (int)(p.T + p.n_halo);  // combined sequence
    const int nT = (T_all + BM - 1) / BM;
    const int ns = choose_spans(BH, nT - q_off / BM, num_sms);
    // variable length: B sequences of at most T tokens packed in [total][H][64],
    // one row bh = (sequence, head) per B * H, spans cut over the longest
    const bool varlen = p.cu_seqlens != nullptr;
    const Varlen vl{p.cu_seqlens, (int)p.total, (int)p.T};
    CUtensorMap tq, tk, tv, tkh, tvh;
    if (varlen) {
        if (!make_map_packed(&tq, p.q, p.total, (int)p.H) ||
            !make_map_packed(&tk, p.k, p.total, (int)p.H) ||
            !make_map_packed(&tv, p.v, p.total, (int)p.H))
            return cudaErrorInvalidValue;
    } else if (!make_map(&tq, p.q, (int)p.T, (int)BH) || !make_map(&tk, p.k, (int)p.T, (int)BH) ||
               !make_map(&tv, p.v, (int)p.T, (int)BH)) {
        return cudaErrorInvalidValue;
    }
    if (q_off > 0) {
        if (!make_map(&tkh, p.halo_k, q_off, (int)BH) || !make_map(&tvh, p.halo_v, q_off, (int)BH))
            return cudaErrorInvalidValue;
    } else {
        tkh = tk;  // never read
        tvh = tv;
    }
    cudaError_t e = cudaFuncSetAttribute(prefill_main_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_MAIN);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(span_summary_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_SUM);
    if (e != cudaSuccess) return e;
    const int n_parts = ns > 1 ? parts_for(nT - q_off / BM, ns, BH, num_sms) : 1;
    float *dA = reinterpret_cast<float *>(p.workspace);
    int *order = nullptr;
    if (varlen) {
        tc_prefill_desc d{};
        d.B = p.B;
        d.H = p.H;
        d.T = p.T;
        d.flags = p.l1_only ? TC_PREFILL_L1_ONLY : 0u;
        const size_t sum = summary_bytes(d, num_sms);
        order = reinterpret_cast<int *>(static_cast<char *>(p.workspace) + (sum + 255) / 256 * 256);
        varlen_order_kernel<<<1, 1024, 0, s>>>(vl, (int)p.B, (int)p.H, order);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // The summary kernel waits for all earlier work of the stream, as usual.
    // The prefix and main kernels after it may start early (programmatic
    // stream serialization); they read their predecessor's results only
    // after griddep_wait, and everything else they read was complete before
    // the summary kernel started.
    cudaLaunchAttribute early[1];
    early[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    early[0].val.programmaticStreamSerializationAllowed = 1;
    const bool summaries = !p.l1_only && ns > 1;
    if (summaries) {
        SumParams sp{dA, p.lam, p.eta, T_all, (int)p.W, (int)p.H, (int)BH, nT, ns, n_parts, q_off,
                     p.status, p.wait_ns, vl};
        const int64_t n_slots = BH * (ns - 1) * n_parts;  // persistent: one CTA per SM at most
        span_summary_kernel<<<(unsigned)(n_slots < num_sms ? n_slots : num_sms), kSumThreads, SMEM_SUM,
                              s>>>(tk, tv, tkh, tvh, sp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        PrefixParams pp{dA, p.lam, T_all, (int)p.W, (int)p.H, nT, ns, n_parts, q_off, vl, p.status};
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3(HD * HD / 256, (unsigned)BH);
        pc.blockDim = dim3(256);
        pc.stream = s;
        pc.attrs = early;
        pc.numAttrs = 1;
        e = cudaLaunchKernelEx(&pc, span_prefix_kernel, pp);
        if (e != cudaSuccess) return e;
    }
    MainParams mp{p.y,      p.A_final, p.lam, p.eta, p.g,  dA, p.A_init, T_all, (int)p.W, (int)p.H,
                  (int)BH, nT,        ns,    n_parts,         p.l1_only ? 1 : 0, q_off, p.status,
                  p.wait_ns,  vl, order};
    const int64_t spans = BH * ns;
    cudaLaunchConfig_t mc = {};
    mc.gridDim = dim3((unsigned)(spans < num_sms ? spans : num_sms));
    mc.blockDim = dim3(kMainThreads);
    mc.dynamicSmemBytes = SMEM_MAIN;
    mc.stream = s;
    mc.attrs = early;
    mc.numAttrs = summaries ? 1 : 0;
    return cudaLaunchKernelEx(&mc, prefill_main_kernel, tq, tk, tv, tkh, tvh, mp);
}

}  // namespace tc
