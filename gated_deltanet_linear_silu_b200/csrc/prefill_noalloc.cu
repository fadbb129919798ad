// gdn_prefill_noalloc: gdn_prefill for callers that cannot hand the library
// a workspace buffer.
//
// Some callers have no way to allocate device memory at the point where they
// run the mixer: an inference runtime whose memory planner reserved the whole
// device arena at start-up and hands out no extra buffers, or a serving loop
// that must not call cudaMalloc/cudaFree (which can synchronise the device)
// once it is running. For them the scratch that gdn_prefill keeps in the
// caller's workspace (the longest-first schedule and the work counter) lives
// here instead, in one fixed array in device global memory that every GPU
// loading this library holds until the process exits.
//
// The array is shared by every call on a device and keeps the contents of the
// last call; the schedule kernel rewrites the schedule and resets the counter
// at the start of each call. Two calls whose kernels overlap on the GPU (on
// different streams without ordering between them) race on the array: order
// such calls on one stream, or use gdn_prefill with separate workspaces.
#include <mutex>

#include "../../include/gdn.h"

namespace {

// Limit of the shared scratch array: 64 KiB, enough for the schedule of
// (65536 - 256) / 4 = 16320 sequences per call.
constexpr size_t kNoallocScratchBytes = 64 * 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device. In host code the
// name g_noalloc_scratch is only a host-side handle, so the address is looked
// up with cudaGetSymbolAddress once per device (with that device current) and
// cached.
void* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

size_t gdn_prefill_noalloc_max_scratch(void) { return kNoallocScratchBytes; }

gdn_status_t gdn_prefill_noalloc(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                                 const float* g, const float* beta, const int32_t* cu_seqlens,
                                 const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H,
                                 int Hk, int dk, int dv, int64_t ld_q, int64_t ld_k, int64_t ld_v,
                                 float scale, int qk_l2norm, float eps, int undecayed, int chunk,
                                 const float* h0, float* hT, void* o, gdn_algo_t algo,
                                 void* stream) {
    // The fixed array stands in for the caller's workspace: gdn_prefill checks
    // every argument first and returns GDN_ERR_WORKSPACE only for a valid
    // problem whose schedule does not fit (more than 16320 sequences).
    void* scratch = nullptr;
    if (N > 0) {
        scratch = scratch_on_current_device();
        if (!scratch) return GDN_ERR_CUDA;
    }
    return gdn_prefill(q, k, v, dtype, g, beta, cu_seqlens, cu_seqlens_host, N, T_tot, H, Hk, dk, dv,
                       ld_q, ld_k, ld_v, scale, qk_l2norm, eps, undecayed, chunk, h0, hT, o, scratch,
                       kNoallocScratchBytes, algo, stream);
}

}  // extern "C"
