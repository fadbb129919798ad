/*
 * gdn.h -- C ABI of libgdn.so: the Gated DeltaNet token mixer on NVIDIA B200
 * (sm_100a). The conv stage, the chunked prefill and the recurrent decode
 * step as the Qwen3.5 linear-attention layer uses them, plus the fused decode
 * step of the whole mixer, the gated output and the gradients:
 *
 *   gdn_conv_silu    causal depthwise conv1d + SiLU over the fused q/k/v
 *                    channels, optional per-head L2 norm of q and k, with a
 *                    rolling conv state.
 *   gdn_prefill      chunked gated delta rule over packed variable-length
 *                    sequences, optional initial state, fp32 final state.
 *   gdn_prefill_layer  the whole mixer for a prefill: the conv and SiLU of
 *                    the layer input fused into the chunked prefill, L2 norms,
 *                    the rolling conv state and (optionally) the gated output.
 *   gdn_decode_step  one recurrent token per sequence, state updated in place.
 *   gdn_decode_layer_step  the whole mixer for one decode token: conv update
 *                    from the conv state, SiLU, L2 norm, the recurrent step
 *                    and (optionally) the gated RMSNorm output, in one kernel.
 *   gdn_gated_rmsnorm  the gated RMSNorm output for prefill outputs.
 *   gdn_backward     gradients of the recurrence (q, k, v, g, beta, h0).
 *
 * Sources (page title, section):
 *   [R] "Qwen3.5-MoE source walkthrough", 4.3 Qwen3_5MoeGatedDeltaNet: the
 *       recurrent rule. With the state S stored as [d_k, d_v]:
 *         S <- exp(g_t) S;  m = S^T k_t;  delta = beta_t (v_t - m);
 *         S <- S + k_t delta^T;  o_t = S^T q_t.
 *   [P] same page, 8.2 (linear_attention cache update): multi-token calls go
 *       through the chunked kernel and return (output, last recurrent state);
 *       single-token calls use the recurrent kernel and the conv update; the
 *       conv and recurrent states are carried between calls.
 *   [C] "7.6 Qwen3.5: linear-attention hybrid", 7.6.2: depthwise causal
 *       Conv1d, kernel 4, padding 3, over conv_dim = 2*key_dim + value_dim
 *       channels; L2 normalisation of q and k before the recurrence.
 *   [G] same page, 7.6.2 (gated RMSNorm output): o = RMSNorm(y) * SiLU(z), z
 *       a separate projection of the layer input; 7.6.3: RMSNorm(x) =
 *       x / sqrt(mean(x^2) + eps) times a per-feature scale (stored there as
 *       1 + w, zero-centred).
 *   [V] same page, 7.6.1 (config table): the value-head and key-head counts of
 *       the linear-attention layers are separate settings
 *       (linear_num_value_heads, linear_num_key_heads).
 *   [U] same page, 7.6.2, the recurrence as that page writes it:
 *         S_t = alpha_t S_{t-1} + k_t [beta_t (v_t - S_{t-1}^T k_t)]^T,
 *       the memory read from the state BEFORE the decay. Calls that take
 *       `undecayed` run this order when it is 1, [R]'s decay-first order
 *       (the default) when it is 0; any other value is GDN_ERR_INVALID_ARG.
 *
 * Heads: H is the number of value heads (v, g, beta, the recurrent state and
 * the output have H heads); q and k have Hk heads, Hk dividing H, and value
 * head h reads q, k head h / (H / Hk) -- each q, k head serves H / Hk
 * consecutive value heads ([V]; the grouping order is this library's reading).
 * Hk = 0 means Hk = H, the plain layer.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     contiguous, 16-byte aligned. The library never allocates or frees.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream) of the
 *     CURRENT device (cudaSetDevice), and every tensor lives on that device:
 *     the library looks up its per-device status word (and the fixed scratch
 *     array of gdn_prefill_noalloc) on the current device. All work is
 *     asynchronous on the stream. Argument errors are detected on the host
 *     and returned synchronously; nothing is launched in that case.
 *   - A launch failure returns GDN_ERR_CUDA (the CUDA error is left for the
 *     caller to query with cudaGetLastError()).
 *   - Problems that only the device can see (a cu_seqlens array that is not
 *     monotone, a bounded wait that ran out) set a device status word and the
 *     affected work is skipped; gdn_check_device_status() reports and clears it.
 *   - No call aborts, exits, traps or asserts on the device.
 *   - dtype applies to q/k/v/o (and x/w/y for the conv). Gates g, beta and the
 *     recurrent states are always fp32. Arithmetic is fp32 throughout.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or cu_seqlens */
    GDN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. head dim 80) */
    GDN_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    GDN_ERR_CUDA = 4,         /* a CUDA launch or query failed */
    GDN_ERR_TIMEOUT = 5       /* a bounded device-side wait ran out */
} gdn_status_t;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype_t;

/* Which prefill kernel runs. AUTO picks the tcgen05 tensor-core kernel for
 * bf16 with d_k = d_v = 128 and chunk 64, and the fp32 CUDA-core kernel
 * otherwise. SIMT forces the CUDA-core kernel (any supported shape).
 * TENSOR forces the tensor-core kernel (GDN_ERR_UNSUPPORTED if the shape is
 * not one it handles). */
typedef enum { GDN_ALGO_AUTO = 0, GDN_ALGO_SIMT = 1, GDN_ALGO_TENSOR = 2 } gdn_algo_t;

/*
 * Causal depthwise conv1d + SiLU (+ per-head L2 norm of q and k). [C], [P]
 *
 *   y[t, c] = SiLU( sum_{j=0}^{K-1} w[c, j] * x~[t - (K-1) + j, c] )
 *
 * where x~ is the sequence's own input, preceded by its conv state (or by
 * zeros when conv_state_in is NULL); sequences never mix. This is PyTorch
 * Conv1d(groups=C, padding=K-1) cross-correlation truncated to the first T
 * outputs. When qk_l2norm is set, the first n_qk_channels channels (q then k)
 * are then divided, per token and per group of head_dim channels, by
 * sqrt(sum of squares + eps).
 *
 *   x               [T_tot, C]     dtype   packed inputs (channels [q | k | v],
 *                                          head-major inside each block)
 *   w               [C, K]         dtype   conv taps
 *   cu_seqlens      [N+1]          int32   device prefix offsets, cu[0] = 0,
 *                                          cu[N] = T_tot, non-decreasing
 *   conv_state_in   [N, C, K-1]    dtype   nullable: the K-1 inputs preceding
 *                                          each sequence, oldest first
 *   conv_state_out  [N, C, K-1]    dtype   nullable: the K-1 latest inputs of
 *                                          each sequence (state_in's columns
 *                                          fill in when T < K-1); may alias
 *                                          conv_state_in (in-place update)
 *   y               [T_tot, C]     dtype   output; must not overlap x
 * Supported: 1 <= K <= 4; C a multiple of 8; when qk_l2norm, head_dim in
 * {16, 32, 64, 128} and n_qk_channels a multiple of head_dim, <= C.
 */
GDN_API gdn_status_t gdn_conv_silu(const void* x, gdn_dtype_t dtype, const void* w,
                           const int32_t* cu_seqlens, int N, int64_t T_tot, int C, int K,
                           const void* conv_state_in, void* conv_state_out,
                           int qk_l2norm, int n_qk_channels, int head_dim, float eps,
                           void* y, void* stream);

/*
 * Bytes of device workspace gdn_prefill needs for this problem on the current
 * device (a multiple of 256; never 0). The workspace holds the work schedule
 * (sequences ordered longest first) and a work counter; it is rewritten by
 * every call. When the (sequence, head) units are too few to fill the device
 * (bf16, dk = dv = 128, chunk 64, N * H at most a sixth of the SM count and
 * long enough sequences), the size also covers the sequence split: each
 * sequence is cut into S segments run as three tensor-core passes (zero and
 * identity initial states, then the true ones) with an fp32 hand-off of the
 * segment start states between them, about 4 * N * S * H * dk * dv * 4 bytes
 * plus a zero value buffer of T_tot * H * dv bf16. A workspace of only
 * 256 + 4 * N bytes (rounded up to 256) runs the plain single pass instead.
 */
GDN_API size_t gdn_prefill_workspace_size(int N, int64_t T_tot, int H, int dk, int dv, int chunk);

/*
 * Chunked gated delta rule over packed sequences. [R], [P]
 *
 * For each sequence n (tokens cu[n] .. cu[n+1]-1) and head h, starting from
 * S = h0[n, h] (zeros when h0 is NULL), every token t applies
 *   q^ = scale * L2(q_t), k^ = L2(k_t)  (L2(x) = x / sqrt(sum x^2 + eps) when
 *                                        qk_l2norm, else identity)
 *   S <- exp(g_t) S;  delta = beta_t (v_t - S^T k^);  S <- S + k^ delta^T;
 *   o_t = S^T q^
 * (with undecayed = 1: delta = beta_t (v_t - S^T k^) from S before the
 * decay, [U]) and the final S is written to hT[n, h]. The kernels evaluate this in chunks
 * of `chunk` tokens (cumulative decay, UT transform with a unit lower
 * triangular solve, inter-chunk state passing); the result equals the token
 * loop up to rounding.
 *
 *   q, k            [T_tot, Hk, dk] dtype   (Hk = 0: Hk = H; see "Heads" above)
 *   v               [T_tot, H, dv]  dtype
 *   g, beta         [T_tot, H]      fp32    g = log(alpha) <= 0 expected
 *   cu_seqlens      [N+1]           int32   device prefix offsets
 *   cu_seqlens_host [N+1]           int32   nullable host copy; when given it
 *                                           is validated on the host
 *   h0              [N, H, dk, dv]  fp32    nullable initial state
 *   hT              [N, H, dk, dv]  fp32    nullable final state; may alias h0
 *   o               [T_tot, H, dv]  dtype   output (dense)
 *   ld_q, ld_k, ld_v                        elements from one token of q, k, v
 *                                           to the next; 0 = dense (Hk*dk, Hk*dk,
 *                                           H*dv). Larger strides let q, k and v
 *                                           be views into one fused [T_tot, C]
 *                                           buffer, e.g. the conv output. Each
 *                                           stride must be at least the dense
 *                                           one and a multiple of 16 bytes.
 *   workspace       ws_bytes >= gdn_prefill_workspace_size(...)
 * A sequence of length 0 writes hT = h0 (or zeros) and no output.
 * Supported: dk, dv in {16, 32, ..., 128}; chunk in {16, 32, 64}.
 * Hk < 0 or H not a multiple of Hk: GDN_ERR_INVALID_ARG.
 * Except for hT == h0, no two buffers may overlap.
 */
GDN_API gdn_status_t gdn_prefill(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                         const float* g, const float* beta,
                         const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                         int N, int64_t T_tot, int H, int Hk, int dk, int dv,
                         int64_t ld_q, int64_t ld_k, int64_t ld_v,
                         float scale, int qk_l2norm, float eps, int undecayed, int chunk,
                         const float* h0, float* hT, void* o,
                         void* workspace, size_t ws_bytes, gdn_algo_t algo, void* stream);

/*
 * gdn_prefill followed by the layer's gated RMSNorm output, in one call. [G]
 * For every (token, value head) row of d_v features, with y the recurrence's
 * output as gdn_prefill computes it:
 *   o = y / sqrt(mean(y^2) + norm_eps) * norm_w * SiLU(z),   SiLU(x) = x / (1 + e^-x)
 * in fp32, rounded once to dtype: a second kernel over o, in place, after the
 * recurrence (the pass of gdn_gated_rmsnorm).
 *
 *   z        [T_tot, H, dv]   dtype, the gate (may not alias o)
 *   norm_w   [dv]             fp32, applied as given (a caller with zero-centred
 *                             weights passes 1 + w)
 *   norm_eps                  >= 0
 * Every other argument, result and error as gdn_prefill; in addition
 * GDN_ERR_UNSUPPORTED for dv > 256 or dv not a multiple of 4.
 */
GDN_API gdn_status_t gdn_prefill_gated(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                                       const float* g, const float* beta, const int32_t* cu_seqlens,
                                       const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H,
                                       int Hk, int dk, int dv, int64_t ld_q, int64_t ld_k,
                                       int64_t ld_v, float scale, int qk_l2norm, float eps,
                                       int undecayed, int chunk, const float* h0, float* hT, void* o,
                                       const void* z, const float* norm_w, float norm_eps,
                                       void* workspace, size_t ws_bytes, gdn_algo_t algo,
                                       void* stream);

/*
 * gdn_prefill without a caller-supplied workspace. The sources describe no
 * counterpart of this call: it exists for callers that cannot allocate device
 * memory where they run the mixer -- a runtime whose memory planner reserved
 * the whole device arena at start-up, or a serving loop that must not call
 * cudaMalloc/cudaFree (which can synchronise the device) once it is running.
 *
 * Arguments and results are those of gdn_prefill minus workspace/ws_bytes.
 * The scratch gdn_prefill keeps in the workspace lives instead in one fixed
 * array in device global memory, gdn_prefill_noalloc_max_scratch() bytes
 * (64 KiB: schedules of up to 16320 sequences), which every GPU that loads the
 * library holds until the process exits. Arguments are checked exactly as
 * gdn_prefill checks them; a valid problem that needs more scratch than the
 * array holds then returns GDN_ERR_WORKSPACE before anything is launched. The
 * call itself allocates nothing.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. All calls on a device share the array and it keeps the last call's
 * contents (each call resets what must start at zero): calls whose kernels
 * overlap on the GPU race on it, so order them on one stream.
 */
GDN_API gdn_status_t gdn_prefill_noalloc(const void* q, const void* k, const void* v,
                                         gdn_dtype_t dtype, const float* g, const float* beta,
                                         const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                         int N, int64_t T_tot, int H, int Hk, int dk, int dv,
                                         int64_t ld_q, int64_t ld_k, int64_t ld_v,
                                         float scale, int qk_l2norm, float eps, int undecayed,
                                         int chunk,
                                         const float* h0, float* hT, void* o, gdn_algo_t algo,
                                         void* stream);

/* Size in bytes of the fixed scratch array behind gdn_prefill_noalloc. */
GDN_API size_t gdn_prefill_noalloc_max_scratch(void);

/*
 * The whole mixer for a prefill: gdn_conv_silu and gdn_prefill (or
 * gdn_prefill_gated when z is given) as one call in which the conv never
 * leaves the chip. [C] [R] [G] [P]
 *
 * x holds the fused projections [q | k | v] (C = 2*Hk*dk + H*dv channels,
 * head-major inside each block) of packed sequences, before the conv. For
 * each channel c and token t of sequence n (start s_n):
 *   y[t, c] = SiLU( sum_{j<K} w[c, j] * x'[t - K + 1 + j, c] )
 * with x'[p] = x[p] for p >= s_n and, before the sequence, the sequence's
 * conv window: x'[s_n - K + 1 + j] = conv_state_in[n, c, j] (oldest first;
 * zeros when conv_state_in is null). y's q, k, v channels then enter the
 * recurrence exactly as gdn_prefill's q, k, v (L2 norms of q and k when
 * qk_l2norm, query scale, undecayed order, h0 -> hT), and o is gated as in
 * gdn_prefill_gated when z is given. conv_state_out[n, c, j] receives the
 * window the next call continues from: the last K-1 inputs of sequence n
 * (reaching back into conv_state_in for sequences shorter than K-1).
 *
 * Where the prefill runs in one pass, the conv runs inside the tensor-core
 * prefill: its producer warps load raw rows of x with the tile copies the plain
 * prefill uses for q, k, v and convolve each tile in shared memory (with the
 * chunk's three preceding rows) before the chunk's first matrix product, so y
 * is never written to memory. Where the prefill runs as the sequence split
 * (few sequence-head units; see gdn_prefill_workspace_size), whose three passes
 * would each convolve again, the call instead runs gdn_conv_silu's kernels into
 * y at the end of the workspace and the split prefill on y -- when ws_bytes is
 * at least gdn_prefill_layer_workspace_size (with only
 * gdn_prefill_workspace_size bytes it stays fused). Either way the arithmetic
 * is gdn_conv_silu's (fp32, SiLU through tanh.approx, y rounded to bf16) and
 * the L2 norms are applied in the prefill after that rounding.
 *
 *   x               [T_tot, C]       bf16   layer input (pre-conv)
 *   conv_w          [C, K]           bf16   depthwise taps, K in 1..4
 *   conv_state_in   [N, C, K-1]      bf16   nullable: zeros
 *   conv_state_out  [N, C, K-1]      bf16   nullable: not written; may equal
 *                                           conv_state_in (updated in place)
 *   g, beta, cu_seqlens, cu_seqlens_host, h0, hT, o, workspace: as gdn_prefill
 *   z, norm_w, norm_eps: as gdn_prefill_gated; z nullable (no gate)
 * Supported: bf16, dk = dv = 128 (the tensor-core kernel; chunk 64); any H / Hk.
 * The workspace is gdn_prefill_layer_workspace_size bytes (at least
 * gdn_prefill_workspace_size(N, T_tot, H, dk, dv, 64)).
 * No buffer may overlap another except conv_state_out == conv_state_in, and o
 * must not overlap x. Errors as gdn_prefill, plus GDN_ERR_UNSUPPORTED for
 * another dtype, head dims or K.
 */
GDN_API gdn_status_t gdn_prefill_layer(const void* x, const void* conv_w, int K, const void* conv_state_in,
                                       void* conv_state_out, gdn_dtype_t dtype, const float* g,
                                       const float* beta, const int32_t* cu_seqlens,
                                       const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H,
                                       int Hk, int dk, int dv, float scale, int qk_l2norm, float eps,
                                       int undecayed, const float* h0, float* hT, void* o,
                                       const void* z, const float* norm_w, float norm_eps,
                                       void* workspace, size_t ws_bytes, void* stream);

/*
 * Bytes of device workspace for gdn_prefill_layer (a multiple of 256):
 * gdn_prefill_workspace_size(N, T_tot, H, dk, dv, 64), plus T_tot * C * 2
 * bytes for y (C = 2*Hk*dk + H*dv; Hk = 0: H) when the prefill runs as the
 * sequence split. Depends on the current device's SM count, like
 * gdn_prefill_workspace_size.
 */
GDN_API size_t gdn_prefill_layer_workspace_size(int N, int64_t T_tot, int H, int Hk, int dk, int dv);

/*
 * The prefill kernel gdn_prefill would run for these arguments:
 * GDN_ALGO_SIMT or GDN_ALGO_TENSOR, or -1 if the combination is unsupported.
 */
GDN_API int gdn_prefill_selected_algo(gdn_dtype_t dtype, int dk, int dv, int chunk, gdn_algo_t algo);

/*
 * One recurrent step for N independent sequences (one token each). [R], [P]
 * Same per-token rule as gdn_prefill (undecayed selects [U]'s order); `state`
 * is read and overwritten in place with the post-token state.
 *
 *   q, k     [N, Hk, dk]      dtype   (Hk = 0: Hk = H; see "Heads" above)
 *   v        [N, H, dv]       dtype
 *   g, beta  [N, H]           fp32
 *   state    [N, H, dk, dv]   fp32   in/out
 *   o        [N, H, dv]       dtype
 * Supported: dk, dv in {16, 32, ..., 128}.
 */
GDN_API gdn_status_t gdn_decode_step(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                             const float* g, const float* beta, float* state,
                             int N, int H, int Hk, int dk, int dv, float scale, int qk_l2norm,
                             float eps, int undecayed, void* o, void* stream);

/*
 * The whole mixer for one decode token per sequence, in one kernel. [C] [R] [G] [P]
 *
 * For each sequence n the fused channels x[n] = [q | k | v] (C = 2*Hk*dk + H*dv,
 * head-major inside each block) go through the causal conv against the
 * sequence's conv state (the K-1 previous inputs, oldest first):
 *   y_c = w[c, K-1] * x[n, c] + sum_{j<K-1} w[c, j] * conv_state[n, c, j]
 * after which conv_state[n, c] shifts by one and takes x[n, c] as its newest
 * entry; then SiLU, the L2 norm of q and k (when qk_l2norm), and the recurrent
 * step of gdn_decode_step on state[n] (undecayed as there). When z is given
 * the output is gated:
 *   o = y / sqrt(mean(y^2) + norm_eps) * norm_w * SiLU(z)   per (n, head),
 * norm_w applied as given (a zero-centred scale w is passed as 1 + w).
 *
 *   x           [N, C]            dtype   the token's fused projections (pre-conv)
 *   conv_w      [C, K]            dtype   depthwise taps, K in 1..4
 *   conv_state  [N, C, K-1]       dtype   updated in place (ignored when K == 1)
 *   g, beta     [N, H]            fp32
 *   state       [N, H, dk, dv]    fp32    updated in place
 *   z           [N, H, dv]        dtype   nullable: no gate
 *   norm_w      [dv]              fp32    required when z is given
 *   o           [N, H, dv]        dtype   output
 * Supported: dk, dv in {16, 32, ..., 128}; any H / Hk (a CTA runs the value
 * heads of one q/k head back to back, so the shared q, k conv state is
 * shifted once). No buffer may overlap another. The step runs as a persistent
 * kernel whose wait for each state copy is bounded (see
 * gdn_set_wait_limit_ns): a wait that runs out leaves some (sequence, head)
 * units unprocessed and records GDN_ERR_TIMEOUT for gdn_check_device_status.
 */
GDN_API gdn_status_t gdn_decode_layer_step(const void* x, const void* conv_w, void* conv_state, int K,
                                           gdn_dtype_t dtype, const float* g, const float* beta,
                                           float* state, const void* z, const float* norm_w,
                                           float norm_eps, int N, int H, int Hk, int dk, int dv,
                                           float scale, int qk_l2norm, float eps, int undecayed,
                                           void* o, void* stream);

/*
 * Bytes of device workspace gdn_backward needs (a multiple of 256): state
 * checkpoints every 16 tokens plus 16 recomputed states per (sequence, head),
 * 4 * dk * dv * (H * (2N + ceil(T_tot / 16) + 1) + 16 N H) bytes, rounded up.
 */
GDN_API size_t gdn_backward_workspace_size(int N, int64_t T_tot, int H, int dk, int dv);

/*
 * Bytes with which gdn_backward keeps the state before every token from its
 * forward pass instead of recomputing blocks of 16 (one of its three
 * token-sequential passes fewer): 4 * dk * dv * H * (2N + T_tot + 1) bytes,
 * rounded up. gdn_backward uses this mode whenever ws_bytes is at least this.
 */
GDN_API size_t gdn_backward_workspace_size_kept(int N, int64_t T_tot, int H, int dk, int dv);

/*
 * Gradients of the recurrence gdn_prefill computes (decay-first order, [R]),
 * for upstream gradients dO of the output and dhT of the final state. fp32
 * arithmetic on CUDA cores, one CTA per (sequence, value head), token by
 * token: a forward pass stores the state every 16 tokens in the workspace,
 * then each block of 16 tokens, last first, recomputes its states and is
 * swept in reverse (with a workspace of gdn_backward_workspace_size_kept
 * bytes every state is stored and nothing is recomputed). Gradients flow through the L2 norms (when qk_l2norm) and
 * the query scale; the q, k gradients of a q/k head shared by several value
 * heads are the sums over them.
 *
 *   q, k           [T_tot, Hk, dk]  dtype   (dense; Hk = 0: Hk = H)
 *   v              [T_tot, H, dv]   dtype
 *   g, beta        [T_tot, H]       fp32
 *   cu_seqlens     [N+1] int32 device (cu_seqlens_host: nullable host copy)
 *   h0             [N, H, dk, dv]   fp32    nullable initial state
 *   dO             [T_tot, H, dv]   fp32    gradient of the output
 *   dhT            [N, H, dk, dv]   fp32    nullable gradient of the final state
 *   dq, dk         [T_tot, Hk, dk]  fp32    out
 *   dv             [T_tot, H, dv]   fp32    out
 *   dg, dbeta      [T_tot, H]       fp32    out
 *   dh0            [N, H, dk, dv]   fp32    nullable out
 *   workspace      ws_bytes >= gdn_backward_workspace_size(...), 256-byte aligned
 * Supported: dk, dv in {16, 32, ..., 128}. Outputs must not overlap inputs.
 */
GDN_API gdn_status_t gdn_backward(const void* q, const void* k, const void* v, gdn_dtype_t dtype,
                                  const float* g, const float* beta, const int32_t* cu_seqlens,
                                  const int32_t* cu_seqlens_host, int N, int64_t T_tot, int H,
                                  int Hk, int dk, int dv, float scale, int qk_l2norm, float eps,
                                  const float* h0, const float* dO, const float* dhT, float* dq,
                                  float* dk_out, float* dv_out, float* dg, float* dbeta,
                                  float* dh0, void* workspace, size_t ws_bytes, void* stream);

/*
 * Gated RMSNorm output over rows of dv features (a row = one (token, head)). [G]
 *   out[r] = y[r] / sqrt(mean(y[r]^2) + eps) * w * SiLU(z[r]),  SiLU(z) = z / (1 + e^-z)
 * w is applied as given (a zero-centred scale is passed as 1 + w).
 *
 *   y, z, out   [rows, dv]   dtype   (out may alias y)
 *   w           [dv]         fp32
 * Supported: dv a multiple of 4, 4 <= dv <= 256.
 */
GDN_API gdn_status_t gdn_gated_rmsnorm(const void* y, const void* z, const float* w, gdn_dtype_t dtype,
                                       int64_t rows, int dv, float eps, void* out, void* stream);

/* Static, human-readable name of a status code. */
GDN_API const char* gdn_status_string(gdn_status_t status);

/*
 * Diagnostic setting, process-wide: the limit in nanoseconds of each bounded
 * wait between the warp groups of the tensor-core prefill kernel and of the
 * wait for a state copy in the streaming whole-mixer decode step (the default
 * is 2 s; a negative value restores it). A wait that runs out records
 * GDN_ERR_TIMEOUT in the device status word; the kernel then stops its work,
 * waits (again bounded) for the copies and tensor-core operations it has in
 * flight, frees its tensor memory and returns, leaving the context usable.
 * 0 makes every such wait whose phase is not already complete at its first
 * probe give up at once, which exercises that path on purpose (tests). The
 * setting applies to launches made after the call.
 */
GDN_API void gdn_set_wait_limit_ns(int64_t ns);

/*
 * Synchronises `stream`, then reads and clears the device status word that
 * kernels set when they skip work they cannot do safely. Returns GDN_OK,
 * GDN_ERR_INVALID_ARG (a device-side cu_seqlens check failed),
 * GDN_ERR_TIMEOUT (a bounded wait ran out) or GDN_ERR_CUDA.
 */
GDN_API gdn_status_t gdn_check_device_status(void* stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH (0.2.0: q/k head count Hk,
 * the `undecayed` order, gdn_backward; 0.2.1: gdn_set_wait_limit_ns; 0.2.2:
 * gdn_prefill_gated; 0.2.3: gdn_backward_workspace_size_kept; 0.2.4:
 * gdn_prefill_layer; 0.2.5: gdn_prefill_layer_workspace_size). Argument
 * lists change between minor versions; a binding checks the version before
 * calling anything else. */
GDN_API int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
