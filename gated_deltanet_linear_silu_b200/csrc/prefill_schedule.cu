// Work schedule for the persistent prefill kernels: sequences ordered longest
// first (so the long tail of a variable-length batch starts early), the work
// counter reset to zero, and cu_seqlens checked on the device.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kMaxSortN = 8192;  // above this the identity order is used

__global__ void __launch_bounds__(1024) prefill_schedule_kernel(const int32_t* cu, int N,
                                                                int64_t T_tot, int32_t* order,
                                                                int32_t* counter, int* status) {
    extern __shared__ int32_t len[];
    const bool sort = N <= kMaxSortN;
    if (threadIdx.x == 0) {
        *counter = 0;
        if (cu[0] != 0 || cu[N] != T_tot) set_status(status, kStatusBadSeqlens);
    }
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        const int32_t l = cu[i + 1] - cu[i];
        if (l < 0) set_status(status, kStatusBadSeqlens);
        if (sort) len[i] = l;
        else order[i] = i;
    }
    if (!sort) return;
    __syncthreads();
    // Rank sort: position = number of sequences that go before this one
    // (longer, or equally long with a smaller index). Stable and unique.
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        const int32_t li = len[i];
        int rank = 0;
        for (int j = 0; j < N; ++j) {
            const int32_t lj = len[j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
}

}  // namespace

WorkspaceLayout prefill_workspace_layout(int N) {
    WorkspaceLayout l;
    l.counter_off = 0;
    l.order_off = 256;
    const size_t order_bytes = sizeof(int32_t) * (size_t)(N > 0 ? N : 1);
    l.total = l.order_off + ((order_bytes + 255) / 256) * 256;
    return l;
}

cudaError_t launch_prefill_schedule(const PrefillArgs& a, cudaStream_t s) {
    const size_t smem = a.N <= kMaxSortN ? sizeof(int32_t) * (size_t)a.N : 0;
    prefill_schedule_kernel<<<1, 1024, smem, s>>>(a.cu, a.N, a.T_tot, a.order, a.counter, a.status);
    return cudaGetLastError();
}

}  // namespace gdn
