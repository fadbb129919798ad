// Work schedule for the persistent prefill kernels: sequences ordered longest
// first (so the long tail of a variable-length batch starts early), empty
// ones last, their count after the work counter; the work counter reset to
// zero, and cu_seqlens checked on the device.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kMaxSortN = 8192;  // above this: index order (work first)

// A sequence with tokens and sane bounds is work for the chunk kernels; the
// others (empty, or a bad cu_seqlens entry) go after all of them.
__device__ __forceinline__ bool is_work(const int32_t* cu, int i, int64_t T_tot) {
    return cu[i] >= 0 && cu[i + 1] > cu[i] && cu[i + 1] <= T_tot;
}

// `copies` counter pairs (work counter, number of work sequences), 2 ints
// apart, for launches that share one schedule.
__global__ void __launch_bounds__(1024) prefill_schedule_kernel(const int32_t* cu, int N,
                                                                int64_t T_tot, int32_t* order,
                                                                int32_t* counter, int copies, int* status) {
    extern __shared__ int32_t len[];
    __shared__ int32_t s_work, s_warp[32];
    pdl_launch_dependents();  // dependent launch (the sequence split): the chunk kernel may
    pdl_wait_previous();      // start launching; no-ops for an ordinary launch
    const bool sort = N <= kMaxSortN;
    if (threadIdx.x == 0) {
        for (int c = 0; c < copies; ++c) counter[2 * c] = 0;
        s_work = 0;
        if (cu[0] != 0 || cu[N] != T_tot) set_status(status, kStatusBadSeqlens);
    }
    __syncthreads();
    int mine = 0;
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        const int32_t l = cu[i + 1] - cu[i];
        if (l < 0) set_status(status, kStatusBadSeqlens);
        const bool w = is_work(cu, i, T_tot);
        mine += w;
        if (sort) len[i] = w ? l : -1;
    }
    atomicAdd(&s_work, mine);
    __syncthreads();
    const int n_work = s_work;
    if (threadIdx.x == 0)
        for (int c = 0; c < copies; ++c) counter[2 * c + 1] = n_work;
    if (sort) {
        // Rank sort: position = number of sequences that go before this one
        // (longer, or equally long with a smaller index); non-work (-1) last.
        for (int i = threadIdx.x; i < N; i += blockDim.x) {
            const int32_t li = len[i];
            int rank = 0;
            for (int j = 0; j < N; ++j) {
                const int32_t lj = len[j];
                rank += (lj > li) || (lj == li && j < i);
            }
            order[rank] = i;
        }
        return;
    }
    // Above kMaxSortN: index order, work first (a stable partition).
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int done_work = 0, done_rest = 0;
    for (int base = 0; base < N; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const bool w = i < N && is_work(cu, i, T_tot);
        const bool rest = i < N && !w;
        const unsigned bw = __ballot_sync(0xffffffffu, w), br = __ballot_sync(0xffffffffu, rest);
        if (lane == 0) s_warp[wid] = (__popc(br) << 16) | __popc(bw);
        __syncthreads();
        int pw = 0, pr = 0, tw = 0, tr = 0;
        for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
            const int v = s_warp[k];
            if (k < wid) { pw += v & 0xFFFF; pr += v >> 16; }
            tw += v & 0xFFFF;
            tr += v >> 16;
        }
        const unsigned below = (1u << lane) - 1u;
        if (w) order[done_work + pw + __popc(bw & below)] = i;
        if (rest) order[n_work + done_rest + pr + __popc(br & below)] = i;
        done_work += tw;
        done_rest += tr;
        __syncthreads();
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

cudaError_t launch_prefill_schedule(const PrefillArgs& a, cudaStream_t s, int copies, bool pdl) {
    const size_t smem = a.N <= kMaxSortN ? sizeof(int32_t) * (size_t)a.N : 0;
    if (pdl)
        return launch_pdl(prefill_schedule_kernel, dim3(1), dim3(1024), smem, s, a.cu, a.N, a.T_tot, a.order,
                          a.counter, copies, a.status);
    prefill_schedule_kernel<<<1, 1024, smem, s>>>(a.cu, a.N, a.T_tot, a.order, a.counter, copies, a.status);
    return cudaGetLastError();
}

}  // namespace gdn
