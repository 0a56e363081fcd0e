// Internal declarations shared by the libtc translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tc.h"

namespace tc {

// ---- element access -------------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Two floats -> a bf16 pair (round to nearest even), a in the low half.
__device__ __forceinline__ uint32_t pack_bf16_rn(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Unpack 16 bytes holding VEC elements of T into floats.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4 &r, float *f) {
        f[0] = __uint_as_float(r.x);
        f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z);
        f[3] = __uint_as_float(r.w);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4 &r, float *f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// One 4 x 4 block of out[m][n] = sum_k a(m, k) b(k, n) in registers (m0, n0
// its corner; a and b return 0 outside the ranges they cover).  Each operand
// loaded from shared memory serves four products (float32 SIMT products of
// the small per-chunk matrices).
template <class FA, class FB>
__device__ __forceinline__ void tile44(int K, int m0, int n0, FA a, FB b, float (&acc)[4][4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = 0.f;
    for (int k = 0; k < K; ++k) {
        float av[4], bv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) av[u] = a(m0 + u, k);
#pragma unroll
        for (int w = 0; w < 4; ++w) bv[w] = b(k, n0 + w);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
    }
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float sigmoidf_acc(float g) { return 1.0f / (1.0f + expf(-g)); }

// ---- device status word ---------------------------------------------------

__device__ __forceinline__ void report(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ---- launch parameter blocks ---------------------------------------------

struct DecodeParams {
    const void *q, *k, *v;
    void *y;
    void *ring_k, *ring_v;
    float *A;
    const float *lam, *eta, *g;
    int64_t H, W, t;
    const int64_t *t_rows;  // per batch row clocks (device), or null: every row at t
    int write_rule;         // TC_WRITE_OUTER or TC_WRITE_DELTA
    int dk, dv;
    int *status;
};

// T new tokens (q, k, v, y rows), continuing after n_halo earlier tokens whose
// keys and values are halo_k / halo_v ([BH][n_halo][d], oldest first), with
// the state A_init ([BH][dk][dv] float32, null = zero) holding every eviction
// before the first one of the combined halo + new sequence.  A plain prefill
// has n_halo = 0 and A_init = null.
struct PrefillParams {
    const void *q, *k, *v;
    void *y;
    float *A_final;
    const float *lam, *eta, *g;
    int64_t B, H, T, W, C;
    int dk, dv;
    bool l1_only;
    bool state_only;  // A_final only (the chunk scan); q and y unused
    bool delta_rule;  // write of Fig. 2 step (3): delta rule instead of the outer product
    bool chunk_mean;  // ablation: the chunk-mean shortcut instead of the weighted sum
    const void *halo_k, *halo_v;
    int64_t n_halo;
    const float *A_init;
    void *workspace;
    size_t workspace_bytes;
    int *status;
    unsigned long long wait_ns;  // limit of the tensor-core kernels' bounded waits
    // variable-length calls (tc_prefill_varlen): B sequences packed along the
    // token axis, sequence b = tokens cu_seqlens[b] .. cu_seqlens[b+1]-1 of
    // [total][H][d] q, k, v, y; T is the longest length.  Null: fixed length.
    const int64_t *cu_seqlens;
    int64_t total;
};

// decode.cu
cudaError_t launch_decode(const DecodeParams &p, tc_dtype dtype, int64_t BH, cudaStream_t s);
// t_rows[b] += 1 for every active row (t_rows[b] >= 0), after a ragged step.
cudaError_t launch_advance_clocks(int64_t *t_rows, int64_t B, cudaStream_t s);
bool decode_supported(int dk, int dv, tc_dtype dtype);

// delta_chunked.cu: the delta-rule write in chunks (no halo), float32 SIMT.
// Workspace: m_t rows ([BH][T][dv] float32, at offset 0, unless state-only)
// and the chunk buffers.  Writes A_final; with add_y it adds sigma(g) m_t into
// y (which holds the window part), else it leaves m_t in the workspace rows.
size_t delta_chunked_workspace_bytes(const tc_prefill_desc &d);
int delta_chunked_launch_count(const tc_prefill_desc &d);
cudaError_t launch_delta_chunked(const PrefillParams &p, tc_dtype dtype, bool add_y, cudaStream_t s);

// prefill_portable.cu: any shape in the supported range, SIMT float32 math.
size_t portable_workspace_bytes(const tc_prefill_desc &d, int64_t n_halo);
cudaError_t launch_prefill_portable(const PrefillParams &p, tc_dtype dtype, cudaStream_t s);

// backward.cu: gradients of the layer (outer-product write); the window part
// on the tensor cores where backward_sm100.cu takes the shape, else float32
// SIMT; the memory part as a float32 chunk scan.
size_t backward_workspace_bytes(const tc_prefill_desc &d);
cudaError_t launch_backward(const tc_prefill_desc &d, const void *q, const void *k, const void *v,
                            const float *lam, const float *eta, const float *g, const void *dy,
                            float *dq, float *dk, float *dv, float *dlam, float *deta, float *dg,
                            void *workspace, int *status, unsigned long long wait_ns,
                            cudaStream_t s);
// Kernels of one backward call.
int backward_launch_count(const tc_prefill_desc &d);

// backward_sm100.cu: window part of the backward, tcgen05 / TMA (bf16, d = 64).
// dq, dk, dv are written (not accumulated); lse and Dt ([BH][Tp] float32,
// Tp = backward_stat_stride(T)) receive the per-query statistics.
bool backward_window_tc_supported(const tc_prefill_desc &d);
int64_t backward_stat_stride(int64_t T);
cudaError_t launch_backward_window_tc(const tc_prefill_desc &d, const void *q, const void *k,
                                      const void *v, const void *dy, float *dq, float *dk, float *dv,
                                      float *lse, float *Dt, int *status, unsigned long long wait_ns,
                                      cudaStream_t s);

// Memory part of the backward, per chunk of 128 evictions on the tensor cores
// (bf16, d = 64).  launch_backward_sums_tc writes each chunk's state
// increment and gradient summary into Ac, Hc ([BH][nC][64][64] float32); after
// the scan over chunks these hold each chunk's start state A_c and the G
// passed back from the later chunks H_c, from which launch_backward_chunks_tc
// adds the chunk's contributions to dq, dk, dv and writes its partials of
// dlambda, deta, dg into part [BH][nC][3].
bool backward_memory_tc_supported(const tc_prefill_desc &d);
cudaError_t launch_backward_sums_tc(const tc_prefill_desc &d, const void *q, const void *k, const void *v,
                                    const void *dy, const float *lam, const float *eta, const float *g,
                                    float *Ac, float *Hc, int *status, unsigned long long wait_ns,
                                    cudaStream_t s);
cudaError_t launch_backward_chunks_tc(const tc_prefill_desc &d, const void *q, const void *k,
                                      const void *v, const void *dy, const float *lam,
                                      const float *eta, const float *g, const float *Ac,
                                      const float *Hc, float *dq, float *dk, float *dv, float *part,
                                      int *status, unsigned long long wait_ns, cudaStream_t s);

// prefill_general_sm100.cu: tensor-core prefill for bf16, d_k = d_v in {64,
// 128}, any W and halo (what prefill_main_kernel does not take).  With the
// delta rule (no halo) the memory's reads come from mrow ([BH][T][d] float32,
// written by launch_delta_chunked); otherwise mrow is null.
bool general_supported(const tc_prefill_desc &d, int64_t n_halo);
// Variable-length calls (PrefillParams::cu_seqlens set) on the general path:
// bf16, d_k = d_v in {64, 128}, any W, flags 0 or L1-only.  Workspace as
// general_workspace_bytes(d, 0) with d.T the longest length.
bool general_varlen_supported(const tc_prefill_desc &d);
size_t general_workspace_bytes(const tc_prefill_desc &d, int64_t n_halo);
int general_launch_count(const tc_prefill_desc &d, int64_t n_halo);
cudaError_t launch_prefill_general(const PrefillParams &p, const float *mrow, cudaStream_t s);

// cuTensorMapEncodeTiled from the driver (null if unavailable).
void *tensor_map_encoder();

// prefill_sm100.cu: tcgen05 / TMA path for bf16, d_k = d_v = 64.
bool sm100_supported(const tc_prefill_desc &d, int64_t n_halo);
size_t sm100_workspace_bytes(const tc_prefill_desc &d, int num_sms, bool varlen = false);
cudaError_t launch_prefill_sm100(const PrefillParams &p, int num_sms, cudaStream_t s);
int sm100_launch_count(const tc_prefill_desc &d);

// tc_api.cu: a per-thread override of tc_set_prefill_path (TC_PATH_*, or -1
// for none) for the calls this thread makes while the object lives.
struct ScopedPrefillPath {
    int prev;
    explicit ScopedPrefillPath(int path);
    ~ScopedPrefillPath();
};

}  // namespace tc
