// C ABI of libgdn (declared in include/gdn.h): argument validation on the
// host, workspace carving, kernel dispatch. No allocation, no host sync except
// in gdn_check_device_status.
#include <atomic>
#include <mutex>

#include "../../include/gdn.h"
#include "common.cuh"
#include "launch.h"

namespace gdn {
size_t prefill_simt_smem_bytes(int chunk, int dk, int dv);
}

namespace {

// Device status word: kernels set it (first error wins) when they skip work.
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

// Address of the status word on the current device (looked up once per device).
int* status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

// Process-wide limit of the tensor-core prefill's bounded hand-off waits
// (gdn_set_wait_limit_ns); negative: the default.
std::atomic<int64_t> g_wait_limit_ns{-1};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_dim_ok(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }
bool dtype_ok(gdn_dtype_t t) { return t == GDN_F32 || t == GDN_BF16; }

gdn_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

gdn_status_t check_host_seqlens(const int32_t* cu, int N, int64_t T_tot) {
    if (!cu) return GDN_OK;
    if (cu[0] != 0 || cu[N] != T_tot) return GDN_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n]) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

}  // namespace

namespace gdn {
uint64_t wait_limit_ns() {
    const int64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
    return v < 0 ? kDefaultWaitNs : static_cast<uint64_t>(v);
}
}  // namespace gdn

extern "C" {

// 0.2.5: gdn_prefill_layer_workspace_size; 0.2.4: gdn_prefill_layer; 0.2.3:
// gdn_backward_workspace_size_kept; 0.2.2: gdn_prefill_gated; 0.2.1: gdn_set_wait_limit_ns;
// 0.2.0: Hk, undecayed, gdn_backward
int gdn_version(void) { return 205; }

void gdn_set_wait_limit_ns(int64_t ns) { g_wait_limit_ns.store(ns < 0 ? -1 : ns, std::memory_order_relaxed); }

const char* gdn_status_string(gdn_status_t s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    }
    return "GDN_ERR_UNKNOWN";
}

gdn_status_t gdn_check_device_status(void* stream) {
    int* p = status_ptr();
    if (!p) return GDN_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int word = 0;
    if (cudaMemcpyAsync(&word, p, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyAsync(p, &zero, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    if (word == gdn::kStatusBadSeqlens) return GDN_ERR_INVALID_ARG;
    if (word == gdn::kStatusTimeout) return GDN_ERR_TIMEOUT;
    return word == 0 ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_conv_silu(const void* x, gdn_dtype_t dtype, const void* w,
                           const int32_t* cu_seqlens, int N, int64_t T_tot, int C, int K,
                           const void* conv_state_in, void* conv_state_out, int qk_l2norm,
                           int n_qk_channels, int head_dim, float eps, void* y, void* stream) {
    if (!dtype_ok(dtype) || N < 0 || T_tot < 0 || C <= 0 || K < 1) return GDN_ERR_INVALID_ARG;
    if (N == 0 && T_tot > 0) return GDN_ERR_INVALID_ARG;
    if (N > 0 && !cu_seqlens) return GDN_ERR_INVALID_ARG;
    if (T_tot > 0 && (!x || !y || !w)) return GDN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(w)) return GDN_ERR_INVALID_ARG;
    if (K > 4 || C % 8 != 0) return GDN_ERR_UNSUPPORTED;
    if (qk_l2norm) {
        if (!(head_dim == 16 || head_dim == 32 || head_dim == 64 || head_dim == 128))
            return GDN_ERR_UNSUPPORTED;
        if (n_qk_channels < 0 || n_qk_channels % head_dim != 0 || n_qk_channels > C || !(eps >= 0.f))
            return GDN_ERR_INVALID_ARG;
    }
    if (x == y) return GDN_ERR_INVALID_ARG;
    if (N == 0) return GDN_OK;
    gdn::ConvArgs a{x, dtype == GDN_BF16, w, cu_seqlens, N, T_tot, C, K, conv_state_in,
                    conv_state_out, qk_l2norm, n_qk_channels, head_dim, eps, y, status_ptr()};
    if (!a.status) return GDN_ERR_CUDA;
    return from_cuda(gdn::launch_conv_silu(a, static_cast<cudaStream_t>(stream)));
}

size_t gdn_prefill_workspace_size(int N, int64_t T_tot, int H, int dk, int dv, int chunk) {
    const size_t base = gdn::prefill_workspace_layout(N < 0 ? 0 : N).total;
    if (H <= 0 || T_tot < 0) return base;
    const int S = gdn::prefill_split_segments(N, T_tot, H, dk, dv, chunk);
    if (S <= 1) return base;
    const size_t split = gdn::prefill_split_workspace_bytes(N, T_tot, H, S);
    return split > base ? split : base;
}

}  // extern "C"

namespace {

// The layer input's conv (gdn_prefill_layer): fused into the tensor-core
// prefill, or (y != nullptr) run first into y, whose channels the prefill then
// reads in place.
struct ConvIn {
    const void* w;
    int K;
    const void* state_in;
    void* state_out;
    void* y;  // [T_tot, C] in the workspace, or nullptr: fused
};

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// gdn_prefill, gdn_prefill_gated (z == nullptr: no gate) and gdn_prefill_layer
// (conv != nullptr: q, k, v are the channels of x, ld_q = ld_k = ld_v = C).
gdn_status_t prefill_impl(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                          const float* g, const float* beta, const int32_t* cu_seqlens,
                          const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H, int Hk,
                          int dk, int dv, int64_t ld_q, int64_t ld_k, int64_t ld_v, float scale,
                          int qk_l2norm, float eps, int undecayed, int chunk, const float* h0,
                          float* hT, void* o, void* workspace, size_t ws_bytes, gdn_algo_t algo,
                          const void* z, const float* norm_w, float norm_eps, void* stream,
                          const ConvIn* conv = nullptr) {
    if (Hk == 0) Hk = H;
    if (!dtype_ok(dtype) || N < 0 || T_tot < 0 || H <= 0 || Hk < 0 || H % Hk != 0)
        return GDN_ERR_INVALID_ARG;
    if (N == 0 && T_tot > 0) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (!(chunk == 16 || chunk == 32 || chunk == 64)) return GDN_ERR_UNSUPPORTED;
    if (!(algo == GDN_ALGO_AUTO || algo == GDN_ALGO_SIMT || algo == GDN_ALGO_TENSOR))
        return GDN_ERR_INVALID_ARG;
    if (N > 0 && !cu_seqlens) return GDN_ERR_INVALID_ARG;
    if (T_tot > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(h0) ||
        !aligned16(hT))
        return GDN_ERR_INVALID_ARG;
    if (qk_l2norm && !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (undecayed != 0 && undecayed != 1) return GDN_ERR_INVALID_ARG;
    const int64_t esz = dtype == GDN_BF16 ? 2 : 4;
    if (ld_q == 0) ld_q = (int64_t)Hk * dk;
    if (ld_k == 0) ld_k = (int64_t)Hk * dk;
    if (ld_v == 0) ld_v = (int64_t)H * dv;
    if (ld_q < (int64_t)Hk * dk || ld_k < (int64_t)Hk * dk || ld_v < (int64_t)H * dv ||
        (ld_q * esz) % 16 != 0 || (ld_k * esz) % 16 != 0 || (ld_v * esz) % 16 != 0)
        return GDN_ERR_INVALID_ARG;
    if ((int64_t)N * H * 2 >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    if (T_tot >= ((int64_t)1 << 31)) return GDN_ERR_UNSUPPORTED;  // cu_seqlens is int32
    if (gdn_status_t st = check_host_seqlens(cu_seqlens_host, N, T_tot)) return st;
    if (N == 0) return GDN_OK;
    const gdn::WorkspaceLayout wl = gdn::prefill_workspace_layout(N);
    if (!workspace || ws_bytes < wl.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GDN_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    gdn::PrefillArgs a{q, k, v, dtype == GDN_BF16, g, beta, cu_seqlens, N, T_tot, H, Hk, dk, dv,
                       ld_q, ld_k, ld_v, scale, qk_l2norm, eps, undecayed, chunk, h0, hT, o,
                       reinterpret_cast<int32_t*>(ws + wl.order_off),
                       reinterpret_cast<int32_t*>(ws + wl.counter_off), status_ptr(),
                       gdn::wait_limit_ns()};
    if (!a.status) return GDN_ERR_CUDA;
    const bool tc_ok = gdn::prefill_tc_supported(a);
    if (algo == GDN_ALGO_TENSOR && !tc_ok) return GDN_ERR_UNSUPPORTED;
    if (conv) {
        // only the tensor-core kernel convolves; without tokens there is nothing to convolve
        if (T_tot > 0 && !tc_ok) return GDN_ERR_UNSUPPORTED;
        if (conv->y) {
            // the conv (and the conv state) first, into y; the prefill reads y's channels
            gdn::ConvArgs ca{q, 1, conv->w, cu_seqlens, N, T_tot, (int)ld_q, conv->K, conv->state_in,
                             conv->state_out, 0, 0, 128, 0.f, conv->y, a.status};
            if (gdn::launch_conv_silu(ca, static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDN_ERR_CUDA;
            const char* x0 = static_cast<const char*>(q);
            const char* y0 = static_cast<const char*>(conv->y);
            a.q = y0;
            a.k = y0 + (static_cast<const char*>(k) - x0);
            a.v = y0 + (static_cast<const char*>(v) - x0);
        } else {
            a.conv_w = conv->w;
            a.conv_K = conv->K;
            a.conv_state = conv->state_in;
            a.conv_cu = cu_seqlens;
        }
    }
    const bool use_tc = tc_ok && algo != GDN_ALGO_SIMT;
    if (!use_tc && gdn::prefill_simt_smem_bytes(chunk, dk, dv) > 227 * 1024) return GDN_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Few (sequence, head) units: cut the sequences into segments so the
    // tensor-core passes fill the GPU (when the workspace has room for it).
    const int S = use_tc ? gdn::prefill_split_segments(N, T_tot, H, dk, dv, chunk) : 1;
    cudaError_t e;
    if (S > 1 && ws_bytes >= gdn::prefill_split_workspace_bytes(N, T_tot, H, S)) {
        e = gdn::launch_prefill_split(a, S, workspace, s);
    } else {
        e = gdn::launch_prefill_schedule(a, s);
        if (e != cudaSuccess) return GDN_ERR_CUDA;
        e = use_tc ? gdn::launch_prefill_tc(a, s) : gdn::launch_prefill_simt(a, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
    if (z && T_tot > 0) {
        // The gate as a second pass over o, in place: one warp per row reduces the
        // row's d_v values in registers. (Inside the tensor-core kernel's output
        // epilogue, where a thread holds one d_v column of 64 tokens, the per-token
        // reduction and gate loads cost more than this pass.)
        gdn::GatedNormArgs gn{o, z, norm_w, dtype == GDN_BF16, T_tot * H, dv, norm_eps, o};
        if ((e = gdn::launch_gated_rmsnorm(gn, s)) != cudaSuccess) return from_cuda(e);
    }
    if (conv && !conv->y && conv->state_out) {
        // the conv windows the next call continues from (after every pass that read
        // conv->state_in, so the update may be in place)
        gdn::ConvArgs ca{q, 1, conv->w, cu_seqlens, N, T_tot, (int)ld_q, conv->K, conv->state_in,
                         conv->state_out, 0, 0, 0, 0.f, nullptr, a.status};
        e = gdn::launch_conv_state(ca, s);
    }
    return from_cuda(e);
}

}  // namespace

extern "C" {

gdn_status_t gdn_prefill(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                         const float* g, const float* beta, const int32_t* cu_seqlens,
                         const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H, int Hk,
                         int dk, int dv, int64_t ld_q, int64_t ld_k, int64_t ld_v, float scale,
                         int qk_l2norm, float eps, int undecayed, int chunk, const float* h0,
                         float* hT, void* o, void* workspace, size_t ws_bytes, gdn_algo_t algo,
                         void* stream) {
    return prefill_impl(q, k, v, dtype, g, beta, cu_seqlens, cu_seqlens_host, N, T_tot, H, Hk, dk, dv,
                        ld_q, ld_k, ld_v, scale, qk_l2norm, eps, undecayed, chunk, h0, hT, o, workspace,
                        ws_bytes, algo, nullptr, nullptr, 0.f, stream);
}

gdn_status_t gdn_prefill_gated(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                               const float* g, const float* beta, const int32_t* cu_seqlens,
                               const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H, int Hk,
                               int dk, int dv, int64_t ld_q, int64_t ld_k, int64_t ld_v, float scale,
                               int qk_l2norm, float eps, int undecayed, int chunk, const float* h0,
                               float* hT, void* o, const void* z, const float* norm_w, float norm_eps,
                               void* workspace, size_t ws_bytes, gdn_algo_t algo, void* stream) {
    if (T_tot > 0 && (!z || !norm_w)) return GDN_ERR_INVALID_ARG;
    if (!aligned16(z) || !aligned16(norm_w) || !(norm_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (z && z == o) return GDN_ERR_INVALID_ARG;
    if (dv > 256 || dv % 4 != 0) return GDN_ERR_UNSUPPORTED;  // the CUDA-core path's gate kernel
    return prefill_impl(q, k, v, dtype, g, beta, cu_seqlens, cu_seqlens_host, N, T_tot, H, Hk, dk, dv,
                        ld_q, ld_k, ld_v, scale, qk_l2norm, eps, undecayed, chunk, h0, hT, o, workspace,
                        ws_bytes, algo, T_tot > 0 ? z : nullptr, norm_w, norm_eps, stream);
}

gdn_status_t gdn_prefill_layer(const void* x, const void* conv_w, int K, const void* conv_state_in,
                               void* conv_state_out, gdn_dtype_t dtype, const float* g, const float* beta,
                               const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int N,
                               int64_t T_tot, int H, int Hk, int dk, int dv, float scale, int qk_l2norm,
                               float eps, int undecayed, const float* h0, float* hT, void* o,
                               const void* z, const float* norm_w, float norm_eps, void* workspace,
                               size_t ws_bytes, void* stream) {
    if (Hk == 0) Hk = H;
    if (!dtype_ok(dtype) || N < 0 || T_tot < 0 || H <= 0 || Hk <= 0 || H % Hk != 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 || dk != 128 || dv != 128 || K < 1 || K > 4) return GDN_ERR_UNSUPPORTED;
    if (T_tot > 0 && (!x || !conv_w)) return GDN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(conv_w) || !aligned16(conv_state_in) || !aligned16(conv_state_out))
        return GDN_ERR_INVALID_ARG;
    if (x && x == o) return GDN_ERR_INVALID_ARG;
    if (z) {
        if (!norm_w || !aligned16(z) || !aligned16(norm_w) || !(norm_eps >= 0.f) || z == o)
            return GDN_ERR_INVALID_ARG;
    }
    const int64_t C = 2 * (int64_t)Hk * dk + (int64_t)H * dv;
    const char* xb = static_cast<const char*>(x);
    const void* q = x;
    const void* k = xb ? xb + 2 * (int64_t)Hk * dk : nullptr;
    const void* v = xb ? xb + 4 * (int64_t)Hk * dk : nullptr;
    // Where the prefill runs as the sequence split, the fused conv would be redone in
    // each of its three passes: there the conv goes first, into y at the end of the
    // workspace, when the workspace holds it (gdn_prefill_layer_workspace_size).
    void* y = nullptr;
    size_t ws_prefill = ws_bytes;
    if (N > 0 && T_tot > 0 && workspace && gdn::prefill_split_segments(N, T_tot, H, dk, dv, 64) > 1) {
        const size_t y_off = round256(gdn_prefill_workspace_size(N, T_tot, H, dk, dv, 64));
        if (ws_bytes >= y_off + (size_t)T_tot * C * 2) {
            y = static_cast<char*>(workspace) + y_off;
            ws_prefill = y_off;
        }
    }
    const ConvIn conv{conv_w, K, conv_state_in, conv_state_out, y};
    return prefill_impl(q, k, v, dtype, g, beta, cu_seqlens, cu_seqlens_host, N, T_tot, H, Hk, dk, dv, C, C,
                        C, scale, qk_l2norm, eps, undecayed, 64, h0, hT, o, workspace, ws_prefill,
                        GDN_ALGO_AUTO, T_tot > 0 ? z : nullptr, norm_w, norm_eps, stream, &conv);
}

size_t gdn_prefill_layer_workspace_size(int N, int64_t T_tot, int H, int Hk, int dk, int dv) {
    const size_t base = gdn_prefill_workspace_size(N, T_tot, H, dk, dv, 64);
    if (Hk == 0) Hk = H;
    if (N <= 0 || T_tot <= 0 || H <= 0 || Hk <= 0 || gdn::prefill_split_segments(N, T_tot, H, dk, dv, 64) <= 1)
        return base;
    const int64_t C = 2 * (int64_t)Hk * dk + (int64_t)H * dv;
    return round256(base) + round256((size_t)T_tot * C * 2);
}

int gdn_prefill_selected_algo(gdn_dtype_t dtype, int dk, int dv, int chunk, gdn_algo_t algo) {
    if (!dtype_ok(dtype) || !head_dim_ok(dk) || !head_dim_ok(dv)) return -1;
    if (!(chunk == 16 || chunk == 32 || chunk == 64)) return -1;
    gdn::PrefillArgs a{};
    a.is_bf16 = dtype == GDN_BF16;
    a.dk = dk;
    a.dv = dv;
    a.chunk = chunk;
    a.T_tot = 1;
    const bool tc_ok = gdn::prefill_tc_supported(a);
    if (algo == GDN_ALGO_TENSOR) return tc_ok ? GDN_ALGO_TENSOR : -1;
    if (algo == GDN_ALGO_SIMT || !tc_ok)
        return gdn::prefill_simt_smem_bytes(chunk, dk, dv) <= 227 * 1024 ? GDN_ALGO_SIMT : -1;
    return GDN_ALGO_TENSOR;
}

gdn_status_t gdn_decode_step(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                             const float* g, const float* beta, float* state, int N, int H, int Hk,
                             int dk, int dv, float scale, int qk_l2norm, float eps, int undecayed,
                             void* o, void* stream) {
    if (Hk == 0) Hk = H;
    if (!dtype_ok(dtype) || N < 0 || H <= 0 || Hk < 0 || H % Hk != 0) return GDN_ERR_INVALID_ARG;
    if (undecayed != 0 && undecayed != 1) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (N == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state))
        return GDN_ERR_INVALID_ARG;
    if (qk_l2norm && !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)N * H >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    gdn::DecodeArgs a{q, k, v, dtype == GDN_BF16, g, beta, state, N, H, Hk, dk, dv, scale, qk_l2norm, eps, undecayed, o,
                      nullptr, nullptr, nullptr, 0, nullptr, nullptr, 0.f, status_ptr(), gdn::wait_limit_ns()};
    return from_cuda(gdn::launch_decode_step(a, static_cast<cudaStream_t>(stream)));
}

gdn_status_t gdn_decode_layer_step(const void* x, const void* conv_w, void* conv_state, int K,
                                   gdn_dtype_t dtype, const float* g, const float* beta, float* state,
                                   const void* z, const float* norm_w, float norm_eps, int N, int H,
                                   int Hk, int dk, int dv, float scale, int qk_l2norm, float eps,
                                   int undecayed, void* o, void* stream) {
    if (Hk == 0) Hk = H;
    if (!dtype_ok(dtype) || N < 0 || H <= 0 || K < 1 || Hk < 0 || H % Hk != 0)
        return GDN_ERR_INVALID_ARG;
    if (undecayed != 0 && undecayed != 1) return GDN_ERR_INVALID_ARG;
    if (K > 4) return GDN_ERR_UNSUPPORTED;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (N == 0) return GDN_OK;
    if (!x || !conv_w || !g || !beta || !state || !o || (K > 1 && !conv_state))
        return GDN_ERR_INVALID_ARG;
    if (z && !norm_w) return GDN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(o) || !aligned16(state) || !aligned16(z) || !aligned16(norm_w) ||
        !aligned16(conv_w) || !aligned16(conv_state))
        return GDN_ERR_INVALID_ARG;
    if (qk_l2norm && !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (z && !(norm_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)N * H >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    gdn::DecodeArgs a{nullptr, nullptr, nullptr, dtype == GDN_BF16, g, beta, state, N, H, Hk, dk, dv,
                      scale, qk_l2norm, eps, undecayed, o, x, conv_w, conv_state, K, z, norm_w, norm_eps,
                      status_ptr(), gdn::wait_limit_ns()};
    return from_cuda(gdn::launch_decode_step(a, static_cast<cudaStream_t>(stream)));
}

size_t gdn_backward_workspace_size(int N, int64_t T_tot, int H, int dk, int dv) {
    if (N < 0 || T_tot < 0 || H <= 0 || dk <= 0 || dv <= 0) return 0;
    const size_t b = gdn::backward_workspace_floats(N, T_tot, H, dk, dv, gdn::kCk) * sizeof(float);
    return (b + 255) / 256 * 256 + 256;
}

size_t gdn_backward_workspace_size_kept(int N, int64_t T_tot, int H, int dk, int dv) {
    if (N < 0 || T_tot < 0 || H <= 0 || dk <= 0 || dv <= 0) return 0;
    const size_t b = gdn::backward_workspace_floats(N, T_tot, H, dk, dv, 1) * sizeof(float);
    return (b + 255) / 256 * 256 + 256;
}

gdn_status_t gdn_backward(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                          const float* g, const float* beta, const int32_t* cu_seqlens,
                          const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H, int Hk,
                          int dk, int dv, float scale, int qk_l2norm, float eps, const float* h0,
                          const float* dO, const float* dhT, float* dq, float* dk_out,
                          float* dv_out, float* dg, float* dbeta, float* dh0, void* workspace,
                          size_t ws_bytes, void* stream) {
    if (Hk == 0) Hk = H;
    if (!dtype_ok(dtype) || N < 0 || T_tot < 0 || H <= 0 || Hk < 0 || H % Hk != 0)
        return GDN_ERR_INVALID_ARG;
    if (N == 0 && T_tot > 0) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (N > 0 && !cu_seqlens) return GDN_ERR_INVALID_ARG;
    if (T_tot > 0 && (!q || !k || !v || !g || !beta || !dO || !dq || !dk_out || !dv_out || !dg ||
                      !dbeta))
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(h0) || !aligned16(dhT) || !aligned16(dh0) || !aligned16(q) || !aligned16(k) ||
        !aligned16(v))
        return GDN_ERR_INVALID_ARG;
    if (qk_l2norm && !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)N * H >= (int64_t)1 << 31 || T_tot >= ((int64_t)1 << 31)) return GDN_ERR_UNSUPPORTED;
    if (gdn_status_t st = check_host_seqlens(cu_seqlens_host, N, T_tot)) return st;
    if (N == 0) return GDN_OK;
    const size_t need = gdn_backward_workspace_size(N, T_tot, H, dk, dv);
    if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GDN_ERR_WORKSPACE;
    // every state kept (no recompute) when the workspace has room for it
    const int ck = ws_bytes >= gdn_backward_workspace_size_kept(N, T_tot, H, dk, dv) ? 1 : gdn::kCk;
    const int64_t slots = 2 * (int64_t)N + (T_tot + ck - 1) / ck + 1;
    float* ws = static_cast<float*>(workspace);
    gdn::BackwardArgs a{q, k, v, dtype == GDN_BF16, g, beta, cu_seqlens, N, T_tot, H, Hk, dk, dv,
                        scale, qk_l2norm, eps, h0, dO, dhT, dq, dk_out, dv_out, dg, dbeta, dh0,
                        ws, ck > 1 ? ws + slots * H * (int64_t)dk * dv : nullptr, slots, status_ptr(), ck};
    if (!a.status) return GDN_ERR_CUDA;
    return from_cuda(gdn::launch_backward(a, static_cast<cudaStream_t>(stream)));
}

gdn_status_t gdn_gated_rmsnorm(const void* y, const void* z, const float* w, gdn_dtype_t dtype,
                               int64_t rows, int dv, float eps, void* out, void* stream) {
    if (!dtype_ok(dtype) || rows < 0) return GDN_ERR_INVALID_ARG;
    if (dv < 4 || dv > 256 || dv % 4 != 0) return GDN_ERR_UNSUPPORTED;
    if (rows == 0) return GDN_OK;
    if (!y || !z || !w || !out) return GDN_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(z) || !aligned16(w) || !aligned16(out)) return GDN_ERR_INVALID_ARG;
    if (!(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    gdn::GatedNormArgs a{y, z, w, dtype == GDN_BF16, rows, dv, eps, out};
    return from_cuda(gdn::launch_gated_rmsnorm(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
