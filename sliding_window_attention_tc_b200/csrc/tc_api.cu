// C-ABI entry points of libtc: argument validation, path selection and the
// host-buffer variants.  Everything numeric happens in the kernels of
// decode.cu, prefill_portable.cu and prefill_sm100.cu.

#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "tc.h"
#include "tc_internal.cuh"

// Per-device status word written by kernels that detect an error on the
// device (never by a trap).
__device__ int tc_device_status_word;

namespace {

constexpr int64_t kMaxDim = 128;
constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(tc_dtype d) { return d == TC_BF16 ? 2 : 4; }

bool valid_dtype(tc_dtype d) { return d == TC_F32 || d == TC_BF16; }

// Host-side checks of a prefill description (no CUDA calls).
tc_status check_desc(const tc_prefill_desc *d) {
    if (!d) return TC_ERR_INVALID_ARG;
    if (d->B < 1 || d->H < 1 || d->T < 0 || d->dk < 1 || d->dv < 1 || d->W < 1 || d->C < 1)
        return TC_ERR_INVALID_ARG;
    if (!valid_dtype(d->dtype)) return TC_ERR_INVALID_ARG;
    if (d->flags & ~(TC_PREFILL_L1_ONLY | TC_PREFILL_STATE_ONLY | TC_PREFILL_DELTA_RULE |
                     TC_PREFILL_CHUNK_MEAN))
        return TC_ERR_INVALID_ARG;
    if ((d->flags & TC_PREFILL_CHUNK_MEAN) &&
        (!(d->flags & TC_PREFILL_STATE_ONLY) || (d->flags & TC_PREFILL_DELTA_RULE)))
        return TC_ERR_INVALID_ARG;
    if ((d->flags & TC_PREFILL_L1_ONLY) && (d->flags & TC_PREFILL_STATE_ONLY))
        return TC_ERR_INVALID_ARG;
    if (d->dk > kMaxDim || d->dv > kMaxDim) return TC_ERR_UNSUPPORTED;
    // grid limits of the portable path and 32-bit-safe element counts
    if (d->B * d->H > 65535) return TC_ERR_UNSUPPORTED;
    if (d->T > (int64_t(1) << 31) || d->W > (int64_t(1) << 31)) return TC_ERR_UNSUPPORTED;
    if (d->B * d->H * d->T * (d->dk > d->dv ? d->dk : d->dv) > (int64_t(1) << 40))
        return TC_ERR_UNSUPPORTED;
    return TC_OK;
}

// Current device, required to be sm_100 (B200).
tc_status current_device(int *dev, int *num_sms) {
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count == 0) {
        cudaGetLastError();
        return TC_ERR_NO_DEVICE;
    }
    if (cudaGetDevice(dev) != cudaSuccess) return TC_ERR_NO_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess)
        return TC_ERR_CUDA;
    if (major != 10) return TC_ERR_NO_DEVICE;
    if (num_sms &&
        cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
        return TC_ERR_CUDA;
    return TC_OK;
}

// A pointer the current device dev can dereference: managed memory, or
// device memory allocated on dev itself.  Memory of another GPU is refused:
// a kernel on dev would otherwise read it over the peer link, or fault when
// peer access is off.
bool is_device_ptr(const void *p, int dev) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeManaged || (a.type == cudaMemoryTypeDevice && a.device == dev);
}

// Limit of the bounded waits inside the tensor-core kernels (0 = default).
unsigned long long g_wait_limit_ns = 0;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s
unsigned long long wait_limit_ns() { return g_wait_limit_ns ? g_wait_limit_ns : kDefaultWaitNs; }

int *status_ptr() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, tc_device_status_word) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return static_cast<int *>(p);
}

// Halo length of a call that continues at global position t0.
int64_t halo_len(const tc_prefill_desc &d, int64_t t0) { return t0 < d.W ? t0 : d.W; }

// tc_set_prefill_path: which tensor-core prefill takes a call both can run
// (and a per-thread override, for tc_prefill_no_alloc).
int g_prefill_path = TC_PATH_AUTO;
thread_local int t_path_override = -1;

// The automatic choice between the two tensor-core paths for a call both
// take (bf16, d = 64, W a multiple of 128), from B200 measurements: the
// general path for fixed-length calls (faster at the LM and long-context
// shapes with and without the memory, for continuations and for the delta
// rule's window part: by 15 % on the LM prefill, 25 % L1-only), the fused
// kernel for variable-length calls (3 % faster on a 15-sequence batch of
// 55..8192 tokens, whose spans it balances across the SMs).
bool general_preferred(bool varlen) {
    switch (t_path_override >= 0 ? t_path_override : g_prefill_path) {
        case TC_PATH_FUSED: return false;
        case TC_PATH_GENERAL: return true;
        default: return !varlen;
    }
}

// The fused kernel takes the call: it supports the shape, and the general
// path does not or is not the one chosen.
bool use_sm100(const tc_prefill_desc &d, int64_t n_halo, bool varlen = false) {
    if (!tc::sm100_supported(d, n_halo)) return false;
    return !(general_preferred(varlen) && tc::general_supported(d, n_halo));
}

// A delta-rule call with queries and no halo whose window part the
// tensor-core kernel takes (its L1-only form): window part there, memory in
// chunks (which then adds sigma(g) m into y).
bool delta_window_on_sm100(const tc_prefill_desc &d, int64_t n_halo) {
    if (!(d.flags & TC_PREFILL_DELTA_RULE) || (d.flags & (TC_PREFILL_L1_ONLY | TC_PREFILL_STATE_ONLY)) ||
        n_halo != 0 || d.T < 1)
        return false;
    tc_prefill_desc l1 = d;
    l1.flags = TC_PREFILL_L1_ONLY;
    return use_sm100(l1, 0);
}

// Shapes the fused kernel does not take but the general tensor-core path does
// (bf16, d_k = d_v in {64, 128}: any W, any halo).
bool use_general(const tc_prefill_desc &d, int64_t n_halo) {
    return !use_sm100(d, n_halo) && tc::general_supported(d, n_halo);
}

size_t prefill_ws(const tc_prefill_desc &d, int64_t n_halo, int num_sms) {
    if (use_sm100(d, n_halo)) return tc::sm100_workspace_bytes(d, num_sms);
    if (use_general(d, n_halo))
        return (d.flags & TC_PREFILL_DELTA_RULE) ? tc::delta_chunked_workspace_bytes(d)
                                                 : tc::general_workspace_bytes(d, n_halo);
    return tc::portable_workspace_bytes(d, n_halo);
}

// Variable-length calls run on the tensor-core path only (any longest
// length, 0 included), without the state-only, delta-rule and chunk-mean
// variants.
bool varlen_supported(const tc_prefill_desc &d) {
    tc_prefill_desc c = d;
    if (c.T < 1) c.T = 1;
    return use_sm100(c, 0, true) && !(d.flags & ~TC_PREFILL_L1_ONLY);
}

// Workspace of a variable-length call on the general path (at least 256
// bytes, so that the call always has a device workspace to check).
size_t varlen_general_ws(const tc_prefill_desc &d) {
    tc_prefill_desc c = d;
    if (c.T < 1) c.T = 1;
    const size_t n = tc::general_workspace_bytes(c, 0);
    return n < 256 ? 256 : n;
}

int sm_count_or_default() {
    int dev = 0, sms = 0;
    if (current_device(&dev, &sms) != TC_OK) return 148;
    return sms;
}

tc_status check_decode_state(const tc_decode_state *s) {
    if (!s) return TC_ERR_INVALID_ARG;
    if (s->B < 1 || s->H < 1 || s->dk < 1 || s->dv < 1 || s->W < 1 || s->t < 0)
        return TC_ERR_INVALID_ARG;
    if (!valid_dtype(s->kv_dtype)) return TC_ERR_INVALID_ARG;
    if (s->write_rule != TC_WRITE_OUTER && s->write_rule != TC_WRITE_DELTA) return TC_ERR_INVALID_ARG;
    if (!s->ring_k || !s->ring_v || !s->A || !s->lambda || !s->eta || !s->g)
        return TC_ERR_INVALID_ARG;
    if (!aligned16(s->ring_k) || !aligned16(s->ring_v) || !aligned16(s->A))
        return TC_ERR_INVALID_ARG;
    if (!tc::decode_supported((int)s->dk, (int)s->dv, s->kv_dtype)) return TC_ERR_UNSUPPORTED;
    if (s->B * s->H > (int64_t(1) << 31)) return TC_ERR_UNSUPPORTED;
    return TC_OK;
}

}  // namespace

namespace tc {
ScopedPrefillPath::ScopedPrefillPath(int path) : prev(t_path_override) { t_path_override = path; }
ScopedPrefillPath::~ScopedPrefillPath() { t_path_override = prev; }
}  // namespace tc

extern "C" {

const char *tc_version(void) { return "0.1.0"; }

void tc_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }

tc_status tc_set_prefill_path(int path) {
    if (path != TC_PATH_AUTO && path != TC_PATH_FUSED && path != TC_PATH_GENERAL) return TC_ERR_INVALID_ARG;
    g_prefill_path = path;
    return TC_OK;
}

int tc_get_prefill_path(void) { return g_prefill_path; }

int tc_prefill_path_for(const tc_prefill_desc *d, int64_t t0) {
    if (check_desc(d) != TC_OK || t0 < 0) return -1;
    const int64_t n_halo = halo_len(*d, t0);
    if (use_sm100(*d, n_halo) || delta_window_on_sm100(*d, n_halo)) return TC_PATH_FUSED;
    if (use_general(*d, n_halo)) return TC_PATH_GENERAL;
    return -1;
}

const char *tc_status_string(tc_status s) {
    switch (s) {
        case TC_OK: return "ok";
        case TC_ERR_INVALID_ARG: return "invalid argument";
        case TC_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case TC_ERR_NO_DEVICE: return "no sm_100 CUDA device";
        case TC_ERR_CUDA: return "CUDA runtime or launch error";
        case TC_ERR_DEVICE_BOUNDS: return "device-side bounds check failed";
        case TC_ERR_DEVICE_TIMEOUT: return "device-side bounded wait timed out";
        case TC_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

size_t tc_prefill_workspace_size(const tc_prefill_desc *d) {
    if (check_desc(d) != TC_OK) return (size_t)-1;
    return prefill_ws(*d, 0, sm_count_or_default());
}

size_t tc_prefill_from_state_workspace_size(const tc_prefill_desc *d, int64_t t0) {
    if (check_desc(d) != TC_OK || t0 < 0) return (size_t)-1;
    return prefill_ws(*d, halo_len(*d, t0), sm_count_or_default());
}

}  // extern "C"

namespace {

// Shared body of tc_prefill (t0 = 0) and tc_prefill_from_state.
tc_status prefill_impl(const tc_prefill_desc *d, int64_t t0, const void *halo_k,
                       const void *halo_v, const float *A_init, const void *q, const void *k,
                       const void *v, const float *lambda, const float *eta, const float *g,
                       void *y, float *A_final, void *workspace, size_t workspace_bytes,
                       tc_stream_t stream) {
    tc_status st = check_desc(d);
    if (st != TC_OK) return st;
    if (t0 < 0 || t0 > (int64_t(1) << 31)) return TC_ERR_INVALID_ARG;
    const bool l1_only = (d->flags & TC_PREFILL_L1_ONLY) != 0;
    const bool state_only = (d->flags & TC_PREFILL_STATE_ONLY) != 0;
    const int64_t n_halo = halo_len(*d, t0);
    // With T = 0 the token tensors are empty and may be NULL; a state-only
    // call reads no queries and writes no outputs.
    const bool empty = d->T == 0;
    const bool need_q = !empty && !state_only;
    if ((need_q && (!q || !y)) || (!empty && (!k || !v)) || !lambda || !eta || !g ||
        (!l1_only && !A_final) || (n_halo > 0 && (!halo_k || !halo_v)))
        return TC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) ||
        (A_final && !aligned16(A_final)) || (workspace && !aligned16(workspace)) ||
        !aligned16(halo_k) || !aligned16(halo_v) || !aligned16(A_init))
        return TC_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = current_device(&dev, &sms);
    if (st != TC_OK) return st;
    const size_t need = prefill_ws(*d, n_halo, sms);
    if (need > 0 && (!workspace || workspace_bytes < need)) return TC_ERR_WORKSPACE;
    const void *ptrs[] = {q, y, k, v, lambda, eta, g};
    for (int i = 0; i < 7; ++i) {
        const bool may_be_null = (i < 2 && !need_q) || (i < 4 && empty);
        if (!(may_be_null && !ptrs[i]) && !is_device_ptr(ptrs[i], dev)) return TC_ERR_INVALID_ARG;
    }
    if (A_final && !is_device_ptr(A_final, dev)) return TC_ERR_INVALID_ARG;
    if (A_init && !is_device_ptr(A_init, dev)) return TC_ERR_INVALID_ARG;
    if (n_halo > 0 && (!is_device_ptr(halo_k, dev) || !is_device_ptr(halo_v, dev))) return TC_ERR_INVALID_ARG;
    if (need > 0 && !is_device_ptr(workspace, dev)) return TC_ERR_INVALID_ARG;

    tc::PrefillParams p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.y = y;
    p.A_final = l1_only ? nullptr : A_final;
    p.lam = lambda;
    p.eta = eta;
    p.g = g;
    p.B = d->B;
    p.H = d->H;
    p.T = d->T;
    p.W = d->W;
    p.C = d->C;
    p.dk = (int)d->dk;
    p.dv = (int)d->dv;
    p.l1_only = l1_only;
    p.state_only = state_only;
    p.delta_rule = (d->flags & TC_PREFILL_DELTA_RULE) != 0;
    p.chunk_mean = (d->flags & TC_PREFILL_CHUNK_MEAN) != 0;
    p.halo_k = n_halo > 0 ? halo_k : nullptr;
    p.halo_v = n_halo > 0 ? halo_v : nullptr;
    p.n_halo = n_halo;
    p.A_init = l1_only ? nullptr : A_init;
    p.workspace = workspace;
    p.workspace_bytes = workspace_bytes;
    p.status = status_ptr();
    p.wait_ns = wait_limit_ns();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (delta_window_on_sm100(*d, n_halo)) {
        tc::PrefillParams w = p;
        w.l1_only = true;
        w.delta_rule = false;
        w.A_final = nullptr;
        w.A_init = nullptr;
        w.workspace = nullptr;
        w.workspace_bytes = 0;
        cudaError_t e = tc::launch_prefill_sm100(w, sms, s);
        if (e == cudaSuccess) e = tc::launch_delta_chunked(p, d->dtype, true, s);
        return e == cudaSuccess ? TC_OK : TC_ERR_CUDA;
    }
    if (use_general(*d, n_halo)) {
        cudaError_t e = cudaSuccess;
        const float *mrow = nullptr;
        if (p.delta_rule) {  // chunked delta memory into the workspace rows, then the window part
            e = tc::launch_delta_chunked(p, d->dtype, false, s);
            mrow = reinterpret_cast<const float *>(workspace);
        }
        if (e == cudaSuccess) e = tc::launch_prefill_general(p, mrow, s);
        return e == cudaSuccess ? TC_OK : TC_ERR_CUDA;
    }
    cudaError_t e = use_sm100(*d, n_halo) ? tc::launch_prefill_sm100(p, sms, s)
                                          : tc::launch_prefill_portable(p, d->dtype, s);
    return e == cudaSuccess ? TC_OK : TC_ERR_CUDA;
}

}  // namespace

extern "C" {

tc_status tc_prefill(const tc_prefill_desc *d, const void *q, const void *k, const void *v,
                     const float *lambda, const float *eta, const float *g, void *y,
                     float *A_final, void *workspace, size_t workspace_bytes,
                     tc_stream_t stream) {
    return prefill_impl(d, 0, nullptr, nullptr, nullptr, q, k, v, lambda, eta, g, y, A_final,
                        workspace, workspace_bytes, stream);
}

tc_status tc_prefill_from_state(const tc_prefill_desc *d, int64_t t0, const void *halo_k,
                                const void *halo_v, const float *A_init, const void *q,
                                const void *k, const void *v, const float *lambda,
                                const float *eta, const float *g, void *y, float *A_final,
                                void *workspace, size_t workspace_bytes, tc_stream_t stream) {
    return prefill_impl(d, t0, halo_k, halo_v, A_init, q, k, v, lambda, eta, g, y, A_final,
                        workspace, workspace_bytes, stream);
}

size_t tc_prefill_varlen_workspace_size(const tc_prefill_desc *d) {
    if (check_desc(d) != TC_OK) return (size_t)-1;
    if (varlen_supported(*d)) return tc::sm100_workspace_bytes(*d, sm_count_or_default(), true);
    if (tc::general_varlen_supported(*d)) return varlen_general_ws(*d);
    return (size_t)-1;
}

tc_status tc_prefill_varlen(const tc_prefill_desc *d, const int64_t *cu_seqlens, int64_t total,
                            const void *q, const void *k, const void *v, const float *lambda,
                            const float *eta, const float *g, void *y, float *A_final,
                            void *workspace, size_t workspace_bytes, tc_stream_t stream) {
    tc_status st = check_desc(d);
    if (st != TC_OK) return st;
    const bool l1_only = (d->flags & TC_PREFILL_L1_ONLY) != 0;
    if (total < 0 || total > (int64_t(1) << 30) || !cu_seqlens ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 7u))
        return TC_ERR_INVALID_ARG;
    if ((total > 0 && (!q || !k || !v || !y)) || !lambda || !eta || !g || (!l1_only && !A_final))
        return TC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) ||
        (A_final && !aligned16(A_final)) || (workspace && !aligned16(workspace)))
        return TC_ERR_INVALID_ARG;
    // tensor-core paths only (the fused kernel, else the general path: bf16,
    // d_k = d_v in {64, 128}), without the state-only, delta-rule or chunk-mean
    // variants
    const bool fused = varlen_supported(*d);
    if (!fused && !tc::general_varlen_supported(*d)) return TC_ERR_UNSUPPORTED;
    if (d->H * total > (int64_t(1) << 31)) return TC_ERR_UNSUPPORTED;
    int dev = 0, sms = 0;
    st = current_device(&dev, &sms);
    if (st != TC_OK) return st;
    const size_t need = fused ? tc::sm100_workspace_bytes(*d, sms, true) : varlen_general_ws(*d);
    if (!workspace || workspace_bytes < need) return TC_ERR_WORKSPACE;
    const void *ptrs[] = {q, k, v, y};
    for (const void *x : ptrs)
        if (total > 0 && !is_device_ptr(x, dev)) return TC_ERR_INVALID_ARG;
    const void *hd[] = {lambda, eta, g, cu_seqlens};
    for (const void *x : hd)
        if (!is_device_ptr(x, dev)) return TC_ERR_INVALID_ARG;
    if (A_final && !l1_only && !is_device_ptr(A_final, dev)) return TC_ERR_INVALID_ARG;
    if (!is_device_ptr(workspace, dev)) return TC_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (total == 0) {
        // every sequence is empty: no tokens to read, A_final = 0
        if (l1_only) return TC_OK;
        const size_t na = (size_t)(d->B * d->H * d->dk * d->dv) * sizeof(float);
        return cudaMemsetAsync(A_final, 0, na, s) == cudaSuccess ? TC_OK : TC_ERR_CUDA;
    }
    tc::PrefillParams p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.y = y;
    p.A_final = l1_only ? nullptr : A_final;
    p.lam = lambda;
    p.eta = eta;
    p.g = g;
    p.B = d->B;
    p.H = d->H;
    p.T = d->T;
    p.W = d->W;
    p.C = d->C;
    p.dk = (int)d->dk;
    p.dv = (int)d->dv;
    p.l1_only = l1_only;
    p.workspace = workspace;
    p.workspace_bytes = workspace_bytes;
    p.status = status_ptr();
    p.wait_ns = wait_limit_ns();
    p.cu_seqlens = cu_seqlens;
    p.total = total;
    const cudaError_t e = fused ? tc::launch_prefill_sm100(p, sms, s) : tc::launch_prefill_general(p, nullptr, s);
    return e == cudaSuccess ? TC_OK : TC_ERR_CUDA;
}

size_t tc_backward_workspace_size(const tc_prefill_desc *d) {
    if (check_desc(d) != TC_OK || d->flags != 0) return (size_t)-1;
    return tc::backward_workspace_bytes(*d);
}

tc_status tc_backward(const tc_prefill_desc *d, const void *q, const void *k, const void *v,
                      const float *lambda, const float *eta, const float *g, const void *dy,
                      float *dq, float *dk, float *dv, float *dlambda, float *deta, float *dg,
                      void *workspace, size_t workspace_bytes, tc_stream_t stream) {
    tc_status st = check_desc(d);
    if (st != TC_OK) return st;
    if (d->flags != 0) return TC_ERR_UNSUPPORTED;
    const bool empty = d->T == 0;
    const void *tok[] = {q, k, v, dy, dq, dk, dv};
    const void *hd[] = {lambda, eta, g, dlambda, deta, dg};
    for (const void *x : tok)
        if ((!x && !empty) || !aligned16(x)) return TC_ERR_INVALID_ARG;
    for (const void *x : hd)
        if (!x) return TC_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return TC_ERR_INVALID_ARG;
    int dev = 0;
    st = current_device(&dev, nullptr);
    if (st != TC_OK) return st;
    const size_t need = tc::backward_workspace_bytes(*d);
    if (need > 0 && (!workspace || workspace_bytes < need)) return TC_ERR_WORKSPACE;
    for (const void *x : tok)
        if (x && !is_device_ptr(x, dev)) return TC_ERR_INVALID_ARG;
    for (const void *x : hd)
        if (!is_device_ptr(x, dev)) return TC_ERR_INVALID_ARG;
    if (need > 0 && !is_device_ptr(workspace, dev)) return TC_ERR_INVALID_ARG;
    cudaError_t e = tc::launch_backward(*d, q, k, v, lambda, eta, g, dy, dq, dk, dv, dlambda, deta,
                                        dg, workspace, status_ptr(), wait_limit_ns(),
                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TC_OK : TC_ERR_CUDA;
}

int tc_backward_launch_count(const tc_prefill_desc *d, int *tensor_cores) {
    if (check_desc(d) != TC_OK || d->flags != 0) return -1;
    if (tensor_cores) *tensor_cores = tc::backward_window_tc_supported(*d) ? 1 : 0;
    return tc::backward_launch_count(*d);
}

int tc_prefill_launch_count(const tc_prefill_desc *d) {
    if (check_desc(d) != TC_OK) return -1;
    if (use_sm100(*d, 0)) return tc::sm100_launch_count(*d);
    const bool l1_only = (d->flags & TC_PREFILL_L1_ONLY) != 0;
    const bool state_only = (d->flags & TC_PREFILL_STATE_ONLY) != 0;
    if (use_general(*d, 0))
        return ((d->flags & TC_PREFILL_DELTA_RULE) ? tc::delta_chunked_launch_count(*d) : 0) +
               tc::general_launch_count(*d, 0);
    if ((d->flags & TC_PREFILL_DELTA_RULE) && !l1_only)  // chunked memory + the window part
        return tc::delta_chunked_launch_count(*d) + (d->T > 0 && !state_only ? 1 : 0);
    return (l1_only ? 0 : 1) + (d->T > 0 && !state_only ? 1 : 0);
}

size_t tc_prefill_host_workspace_size(const tc_prefill_desc *d) {
    if (check_desc(d) != TC_OK) return (size_t)-1;
    const size_t es = elem_size(d->dtype);
    const size_t nq = (size_t)(d->B * d->H * d->T * d->dk) * es;
    const size_t nv = (size_t)(d->B * d->H * d->T * d->dv) * es;
    const size_t na = (size_t)(d->B * d->H * d->dk * d->dv) * sizeof(float);
    const size_t np = (size_t)d->H * sizeof(float);
    return round_up(prefill_ws(*d, 0, sm_count_or_default())) + 2 * round_up(nq) + 2 * round_up(nv) +
           3 * round_up(np) + round_up(na);
}

tc_status tc_prefill_host(const tc_prefill_desc *d, const void *q, const void *k, const void *v,
                          const float *lambda, const float *eta, const float *g, void *y,
                          float *A_final, void *workspace, size_t workspace_bytes,
                          tc_stream_t stream) {
    tc_status st = check_desc(d);
    if (st != TC_OK) return st;
    const bool l1_only = (d->flags & TC_PREFILL_L1_ONLY) != 0;
    if ((d->T > 0 && (!q || !k || !v || !y)) || !lambda || !eta || !g) return TC_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = current_device(&dev, &sms);
    if (st != TC_OK) return st;
    const size_t need = tc_prefill_host_workspace_size(d);
    if (!workspace || workspace_bytes < need) return TC_ERR_WORKSPACE;
    if (!aligned16(workspace) || !is_device_ptr(workspace, dev)) return TC_ERR_INVALID_ARG;

    const size_t es = elem_size(d->dtype);
    const size_t nq = (size_t)(d->B * d->H * d->T * d->dk) * es;
    const size_t nv = (size_t)(d->B * d->H * d->T * d->dv) * es;
    const size_t na = (size_t)(d->B * d->H * d->dk * d->dv) * sizeof(float);
    const size_t np = (size_t)d->H * sizeof(float);
    char *base = static_cast<char *>(workspace);
    const size_t ws = round_up(prefill_ws(*d, 0, sms));
    char *dq = base + ws;
    char *dk_ = dq + round_up(nq);
    char *dv_ = dk_ + round_up(nq);
    char *dy = dv_ + round_up(nv);
    char *dl = dy + round_up(nv);
    char *de = dl + round_up(np);
    char *dg = de + round_up(np);
    char *da = dg + round_up(np);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice, d2h = cudaMemcpyDeviceToHost;
    if (cudaMemcpyAsync(dq, q, nq, h2d, s) != cudaSuccess ||
        cudaMemcpyAsync(dk_, k, nq, h2d, s) != cudaSuccess ||
        cudaMemcpyAsync(dv_, v, nv, h2d, s) != cudaSuccess ||
        cudaMemcpyAsync(dl, lambda, np, h2d, s) != cudaSuccess ||
        cudaMemcpyAsync(de, eta, np, h2d, s) != cudaSuccess ||
        cudaMemcpyAsync(dg, g, np, h2d, s) != cudaSuccess)
        return TC_ERR_CUDA;
    st = tc_prefill(d, dq, dk_, dv_, reinterpret_cast<float *>(dl), reinterpret_cast<float *>(de),
                    reinterpret_cast<float *>(dg), dy, l1_only ? nullptr : reinterpret_cast<float *>(da),
                    ws ? base : nullptr, ws, stream);
    if (st != TC_OK) return st;
    if (cudaMemcpyAsync(y, dy, nv, d2h, s) != cudaSuccess) return TC_ERR_CUDA;
    if (A_final && !l1_only && cudaMemcpyAsync(A_final, da, na, d2h, s) != cudaSuccess)
        return TC_ERR_CUDA;
    return TC_OK;
}

}  // extern "C"

namespace {

// Shared body of tc_decode_step (one clock, s->t) and tc_decode_step_ragged
// (a device clock per batch row).
tc_status decode_impl(tc_decode_state *s, int64_t *t_rows, const void *q_t, const void *k_t,
                      const void *v_t, void *y_t, tc_stream_t stream) {
    tc_status st = check_decode_state(s);
    if (st != TC_OK) return st;
    if (!q_t || !k_t || !v_t || !y_t) return TC_ERR_INVALID_ARG;
    if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) || !aligned16(y_t) ||
        (t_rows && (reinterpret_cast<uintptr_t>(t_rows) & 7u)))
        return TC_ERR_INVALID_ARG;
    int dev = 0;
    st = current_device(&dev, nullptr);
    if (st != TC_OK) return st;
    const void *ptrs[] = {q_t, k_t, v_t, y_t, s->ring_k, s->ring_v, s->A, s->lambda, s->eta, s->g};
    for (const void *p : ptrs)
        if (!is_device_ptr(p, dev)) return TC_ERR_INVALID_ARG;
    if (t_rows && !is_device_ptr(t_rows, dev)) return TC_ERR_INVALID_ARG;
    tc::DecodeParams p{};
    p.q = q_t;
    p.k = k_t;
    p.v = v_t;
    p.y = y_t;
    p.ring_k = s->ring_k;
    p.ring_v = s->ring_v;
    p.A = s->A;
    p.lam = s->lambda;
    p.eta = s->eta;
    p.g = s->g;
    p.H = s->H;
    p.W = s->W;
    p.t = s->t;
    p.t_rows = t_rows;
    p.write_rule = (int)s->write_rule;
    p.dk = (int)s->dk;
    p.dv = (int)s->dv;
    p.status = status_ptr();
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = tc::launch_decode(p, s->kv_dtype, s->B * s->H, cs);
    if (e != cudaSuccess) return TC_ERR_CUDA;
    if (t_rows) {
        if (tc::launch_advance_clocks(t_rows, s->B, cs) != cudaSuccess) return TC_ERR_CUDA;
    } else {
        s->t += 1;
    }
    return TC_OK;
}

}  // namespace

extern "C" {

tc_status tc_decode_step(tc_decode_state *s, const void *q_t, const void *k_t, const void *v_t,
                         void *y_t, tc_stream_t stream) {
    return decode_impl(s, nullptr, q_t, k_t, v_t, y_t, stream);
}

tc_status tc_decode_step_ragged(tc_decode_state *s, int64_t *t_rows, const void *q_t,
                                const void *k_t, const void *v_t, void *y_t, tc_stream_t stream) {
    if (!t_rows) return TC_ERR_INVALID_ARG;
    return decode_impl(s, t_rows, q_t, k_t, v_t, y_t, stream);
}

size_t tc_decode_step_host_workspace_size(const tc_decode_state *s) {
    if (check_decode_state(s) != TC_OK) return (size_t)-1;
    const size_t es = elem_size(s->kv_dtype);
    return 2 * round_up((size_t)(s->B * s->H * s->dk) * es) +
           2 * round_up((size_t)(s->B * s->H * s->dv) * es);
}

tc_status tc_decode_step_host(tc_decode_state *s, const void *q_t, const void *k_t,
                              const void *v_t, void *y_t, void *workspace,
                              size_t workspace_bytes, tc_stream_t stream) {
    tc_status st = check_decode_state(s);
    if (st != TC_OK) return st;
    if (!q_t || !k_t || !v_t || !y_t) return TC_ERR_INVALID_ARG;
    int dev = 0;
    st = current_device(&dev, nullptr);
    if (st != TC_OK) return st;
    const size_t need = tc_decode_step_host_workspace_size(s);
    if (!workspace || workspace_bytes < need) return TC_ERR_WORKSPACE;
    if (!aligned16(workspace) || !is_device_ptr(workspace, dev)) return TC_ERR_INVALID_ARG;
    const size_t es = elem_size(s->kv_dtype);
    const size_t nk = (size_t)(s->B * s->H * s->dk) * es, nv = (size_t)(s->B * s->H * s->dv) * es;
    char *dq = static_cast<char *>(workspace);
    char *dk_ = dq + round_up(nk);
    char *dv_ = dk_ + round_up(nk);
    char *dy = dv_ + round_up(nv);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(dq, q_t, nk, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(dk_, k_t, nk, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(dv_, v_t, nv, cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return TC_ERR_CUDA;
    st = tc_decode_step(s, dq, dk_, dv_, dy, stream);
    if (st != TC_OK) return st;
    if (cudaMemcpyAsync(y_t, dy, nv, cudaMemcpyDeviceToHost, cs) != cudaSuccess) return TC_ERR_CUDA;
    return TC_OK;
}

tc_status tc_get_device_status(tc_stream_t stream) {
    int dev = 0;
    tc_status st = current_device(&dev, nullptr);
    if (st != TC_OK) return st;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return TC_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, tc_device_status_word, sizeof(int)) != cudaSuccess)
        return TC_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(tc_device_status_word, &zero, sizeof(int)) != cudaSuccess)
        return TC_ERR_CUDA;
    return v == 0 ? TC_OK : static_cast<tc_status>(v);
}

}  // extern "C"
