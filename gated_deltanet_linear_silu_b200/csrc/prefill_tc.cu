// Tensor-core (tcgen05) chunked prefill for bf16, d_k = d_v = 128, chunk 64.
// Not built yet: the CUDA-core kernel serves every shape until it lands.
#include "launch.h"

namespace gdn {

bool prefill_tc_supported(const PrefillArgs& a) {
    (void)a;
    return false;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
    (void)a;
    (void)s;
    return cudaErrorNotSupported;
}

}  // namespace gdn
