// Tensor-core prefill path (tcgen05 + TMA); filled in below the portable path.
#include "tc_internal.cuh"

namespace tc {

bool sm100_supported(const tc_prefill_desc &d) {
    (void)d;
    return false;
}

size_t sm100_workspace_bytes(const tc_prefill_desc &d, int num_sms) {
    (void)d;
    (void)num_sms;
    return 0;
}

int sm100_launch_count(const tc_prefill_desc &d) {
    (void)d;
    return 0;
}

cudaError_t launch_prefill_sm100(const PrefillParams &p, int num_sms, cudaStream_t s) {
    (void)p;
    (void)num_sms;
    (void)s;
    return cudaErrorNotSupported;
}

}  // namespace tc
