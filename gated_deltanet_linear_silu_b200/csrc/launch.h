// Internal launcher declarations of libgdn (host side). Arguments are
// validated by the C-ABI layer (api.cu) before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream finishes; it must call pdl_wait_previous()
// before reading what that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

struct ConvArgs {
    const void* x;
    int is_bf16;
    const void* w;
    const int32_t* cu;
    int N;
    int64_t T_tot;
    int C, K;
    const void* state_in;
    void* state_out;
    int qk_l2norm, n_qk, head_dim;
    float eps;
    void* y;
    int* status;
};
cudaError_t launch_conv_silu(const ConvArgs& a, cudaStream_t s);
// The conv-state update alone (state_out from the last K-1 inputs of each sequence).
cudaError_t launch_conv_state(const ConvArgs& a, cudaStream_t s);

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    int is_bf16;
    const float* g;
    const float* beta;
    float* state;
    int N, H, Hk, dk, dv;  // H value heads; q, k have Hk heads, head h reads h / (H / Hk)
    float scale;
    int qk_l2norm;
    float eps;
    int undecayed;  // 1: the memory is read from the state before the decay
    void* o;
    // whole-mixer step (x != nullptr): q, k, v come from the conv update of x
    const void* x;        // [N, C] fused projections, C = 2*Hk*dk + H*dv
    const void* conv_w;   // [C, K]
    void* conv_state;     // [N, C, K-1], updated in place
    int K;
    // gated RMSNorm output (z != nullptr)
    const void* z;        // [N, H, dv]
    const float* norm_w;  // [dv]
    float norm_eps;
    int* status;      // device status word (GDN_ERR_TIMEOUT when a wait runs out)
    uint64_t wait_ns;  // bound on each wait of the streaming kernel
};
cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s);
// Persistent streaming form of the whole-mixer step: two CTAs per SM, each
// taking whole q/k groups of value heads and prefetching its next unit's state
// and conv inputs into a shared-memory slot by bulk copies.
bool decode_stream_supported(const DecodeArgs& a);
cudaError_t launch_decode_stream(const DecodeArgs& a, cudaStream_t s);

// Backward of the recurrence (fp32, one CTA per (sequence, value head)).
constexpr int kCk = 16;  // tokens between state checkpoints
struct BackwardArgs {
    const void* q;
    const void* k;
    const void* v;
    int is_bf16;
    const float* g;
    const float* beta;
    const int32_t* cu;
    int N;
    int64_t T_tot;
    int H, Hk, dk, dv;
    float scale;
    int qk_l2norm;
    float eps;
    const float* h0;    // [N, H, dk, dv] or null
    const float* dO;    // [T, H, dv]
    const float* dhT;   // [N, H, dk, dv] or null
    float* dq_out;      // [T, Hk, dk]
    float* dk_out;      // [T, Hk, dk]
    float* dv_out;      // [T, H, dv]
    float* dg;          // [T, H]
    float* dbeta;       // [T, H]
    float* dh0;         // [N, H, dk, dv] or null
    float* ws_ckpt;     // ck_slots x H checkpoints of dk x dv
    float* ws_buf;      // N x H x ck states of dk x dv (ck > 1)
    int64_t ck_slots;
    int* status;
    int ck;             // tokens between checkpoints: kCk, or 1 (every state kept, no recompute)
};
size_t backward_workspace_floats(int N, int64_t T_tot, int H, int dk, int dv, int ck);
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s);

struct GatedNormArgs {
    const void* y;
    const void* z;
    const float* w;
    int is_bf16;
    int64_t rows;
    int dv;
    float eps;
    void* out;
};
cudaError_t launch_gated_rmsnorm(const GatedNormArgs& a, cudaStream_t s);

struct PrefillArgs {
    const void* q;
    const void* k;
    const void* v;
    int is_bf16;
    const float* g;
    const float* beta;
    const int32_t* cu;
    int N;
    int64_t T_tot;
    int H, Hk, dk, dv;         // H value heads; q, k have Hk heads, head h reads h / (H / Hk)
    int64_t ld_q, ld_k, ld_v;  // elements between consecutive tokens of q, k, v
    float scale;
    int qk_l2norm;
    float eps;
    int undecayed;  // 1: each token reads the state before its own decay (gamma_{r-1} row decay)
    int chunk;
    const float* h0;
    float* hT;
    void* o;
    // Workspace carve-up (see prefill_workspace_layout).
    int32_t* order;    // [N] sequences, longest first
    int32_t* counter;  // [2]: work counter of the persistent kernels; number of
                       // work sequences (tokens, sane bounds: order's first entries)
    int* status;
    // Limit of each bounded hand-off wait inside the tensor-core kernel (ns);
    // 0: a wait whose phase is not complete at its first probe gives up.
    uint64_t wait_ns;
    // Causal conv + SiLU of the layer input fused into the tensor-core kernel
    // (conv_w != nullptr): q, k, v then point at the q, k, v channels of
    // x [T_tot, C] (ld_q = ld_k = ld_v = C) and hold the raw rows; the kernel
    // convolves each tile in shared memory before its first use.
    const void* conv_w = nullptr;      // [C, K] bf16
    int conv_K = 0;                    // taps, 1..4
    const void* conv_state = nullptr;  // [N_seq, C, K-1] bf16 window before each sequence, or null (zeros)
    const int32_t* conv_cu = nullptr;  // [N_seq + 1] sequence bounds of the conv windows
    int conv_seg = 1;                  // units' sequence index / conv_seg = conv sequence (the split)
    int conv_v = 1;                    // 0: the v tiles are used as loaded (the split's v = 0 pass)
};
// Default limit of the bounded hand-off waits (2 s) and the process-wide
// setting (gdn_set_wait_limit_ns).
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
uint64_t wait_limit_ns();

struct WorkspaceLayout {
    size_t counter_off, order_off, total;
};
WorkspaceLayout prefill_workspace_layout(int N);

// Sequence split for launches with few (sequence, head) units on the
// tensor-core path: the number of segments per sequence (1: no split, which
// also holds when dk, dv or the chunk rule it out), the workspace it needs,
// and the split launch itself (three prefill passes and the fp32 hand-off of
// the segments' start states).
int prefill_split_segments(int N, int64_t T_tot, int H, int dk, int dv, int chunk);
size_t prefill_split_workspace_bytes(int N, int64_t T_tot, int H, int S);
cudaError_t launch_prefill_split(const PrefillArgs& a, int S, void* workspace, cudaStream_t s);

// Builds the longest-first schedule and zeroes the work counter; `copies`
// counter pairs, 2 ints apart in the 256-byte counter line (launches that share
// one schedule each take their own pair).
// pdl: launch with programmatic dependent launch (the sequence split's chain;
// measured slower for the single-pass prefill, which launches ordinarily).
cudaError_t launch_prefill_schedule(const PrefillArgs& a, cudaStream_t s, int copies = 1, bool pdl = false);
cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s);
bool prefill_tc_supported(const PrefillArgs& a);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s, bool pdl = false);

}  // namespace gdn
