// tc_state_fold: the exclusive prefix of L2 states across consecutive pieces
// of one sequence.
//
// "Tensor Cache: Eviction-conditioned Associative Memory for Transformers",
// §3.2 / Fig. 2 step (3): every eviction does A <- lambda A + eta k v^T.  If a
// sequence is cut into consecutive pieces s = 0, 1, ... and piece s alone
// (from A = 0) leaves dA_s after its E_s evictions, then the state before
// piece p is the recurrence A_0 = 0, A_{s+1} = lambda^{E_s} A_s + dA_s taken
// up to s = p - 1 -- the same weighted sum the chunk scan uses, with pieces
// as chunks.

#include <cuda_runtime.h>

#include <cstdint>

#include "tc.h"

namespace {

__global__ void state_fold_kernel(int64_t BH, int64_t H, int64_t nel, int64_t n_parts,
                                  const float *dA, const int64_t *E, const float *lam,
                                  float *A_out) {
    const int64_t total = BH * nel;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = (x / nel) % H;
        const double l2l = log2((double)lam[h]);
        float a = 0.f;
        for (int64_t s = 0; s < n_parts; ++s) {
            const float dec = (float)exp2((double)E[s] * l2l);
            a = fmaf(dec, a, dA[s * total + x]);
        }
        A_out[x] = a;
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool device_ptr(const void *p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

}  // namespace

extern "C" tc_status tc_state_fold(int64_t B, int64_t H, int64_t dk, int64_t dv, int64_t n_parts,
                                   const float *dA, const int64_t *E, const float *lambda,
                                   float *A_out, tc_stream_t stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1 || n_parts < 0 || dk > 128 || dv > 128)
        return TC_ERR_INVALID_ARG;
    if (!A_out || !lambda || (n_parts > 0 && (!dA || !E))) return TC_ERR_INVALID_ARG;
    if (!aligned16(A_out) || !aligned16(dA)) return TC_ERR_INVALID_ARG;
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count == 0) {
        cudaGetLastError();
        return TC_ERR_NO_DEVICE;
    }
    if (!device_ptr(A_out) || !device_ptr(lambda) || (n_parts > 0 && (!device_ptr(dA) || !device_ptr(E))))
        return TC_ERR_INVALID_ARG;
    const int64_t total = B * H * dk * dv;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    state_fold_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), threads, 0,
                        reinterpret_cast<cudaStream_t>(stream)>>>(B * H, H, dk * dv, n_parts, dA,
                                                                  E, lambda, A_out);
    return cudaGetLastError() == cudaSuccess ? TC_OK : TC_ERR_CUDA;
}
