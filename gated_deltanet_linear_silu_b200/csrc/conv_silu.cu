// Causal depthwise conv1d (kernel K <= 4) + SiLU + per-head L2 norm of q, k.
//
// "7.6 Qwen3.5: linear-attention hybrid", 7.6.2: a depthwise causal Conv1d of
// kernel 4 (padding 3) mixes each channel over the 4 latest tokens before the
// recurrence, and q and k are L2-normalised per head. The activation after the
// conv is SiLU. One pass over HBM: every input row is read once by the CTA
// that owns it (plus a 3-row halo that hits L2), every output row written once.
//
// Thread layout: a thread owns 8 consecutive channels (one 16-byte bf16
// vector) of TT consecutive tokens. A warp covers 256 channels; the L2 norm of
// a head (head_dim channels = head_dim/8 lanes) is a shuffle reduction inside
// the warp. When the CTA's tokens and their 3-token halo lie inside one
// sequence (the common case) every thread issues all TT + 3 row loads before
// the first use, so a CTA keeps (TT + 3) x 16 bytes per thread in flight; tiles
// that touch a sequence start take a token-by-token path that reads the conv
// state (or zeros) for positions before the start.
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 128;
constexpr int kVec = 8;                       // channels per thread
constexpr int kChanPerCta = kThreads * kVec;  // 1024
constexpr int kTT = 8;                        // tokens per CTA

template <typename T> struct Vec8;
template <> struct Vec8<uint16_t> {
    __device__ __forceinline__ static void load(const uint16_t* p, float (&x)[8]) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    __device__ __forceinline__ static void store(uint16_t* p, const float (&x)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = static_cast<uint32_t>(f32_to_bf16(x[2 * i])) |
                   (static_cast<uint32_t>(f32_to_bf16(x[2 * i + 1])) << 16);
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Vec8<float> {
    __device__ __forceinline__ static void load(const float* p, float (&x)[8]) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
    __device__ __forceinline__ static void store(float* p, const float (&x)[8]) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
    }
};

// One token's 8 channels as loaded (converted to fp32 at first use).
template <typename T> struct Raw8;
template <> struct Raw8<uint16_t> {
    uint4 u;
    __device__ __forceinline__ void load(const uint16_t* p) { u = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void get(float (&x)[8]) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = *reinterpret_cast<const float4*>(p);
        b = *reinterpret_cast<const float4*>(p + 4);
    }
    __device__ __forceinline__ void get(float (&x)[8]) const {
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};

// SiLU(x) = x * sigmoid(x) = x / (1 + e^-x), with the fast exponential and
// divide (both within a few ulp of fp32; the result is 0 when e^-x overflows).
__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// One token's 8 channels as four fp32 pairs (bf16: exact widening).
template <typename T> struct Pairs;
template <> struct Pairs<uint16_t> {
    __device__ __forceinline__ static void get(const uint4& u, float2 (&x)[4]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    }
};

// conv (4-wide window, taps right-aligned) + SiLU for one token; returns the
// squared norm of the 8 outputs.
template <typename T>
__device__ __forceinline__ float conv_token(const float (&wp)[4][8], const float (&xm3)[8],
                                            const float (&xm2)[8], const float (&xm1)[8],
                                            const float (&xt)[8], float (&y)[8]) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float acc = wp[0][i] * xm3[i];
        acc = fmaf(wp[1][i], xm2[i], acc);
        acc = fmaf(wp[2][i], xm1[i], acc);
        acc = fmaf(wp[3][i], xt[i], acc);
        acc = silu(acc);
        y[i] = acc;
        ss = fmaf(acc, acc, ss);
    }
    return ss;
}

// Input of sequence n at absolute token p for the thread's 8 channels; p may
// precede the sequence start, in which case the conv state (or 0) supplies it.
template <typename T>
__device__ __forceinline__ void fetch(const ConvArgs& a, int n, int64_t seq_start, int64_t p,
                                      int c0, bool active, float (&x)[8]) {
    if (!active) {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = 0.f;
        return;
    }
    if (p >= seq_start) {
        Vec8<T>::load(static_cast<const T*>(a.x) + p * a.C + c0, x);
        return;
    }
    const int64_t s = (a.K - 1) + (p - seq_start);  // state column
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float val = 0.f;
        if (a.state_in && s >= 0)
            val = Elem<T>::load(static_cast<const T*>(a.state_in),
                                ((int64_t)n * a.C + c0 + i) * (a.K - 1) + s);
        x[i] = val;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) conv_silu_kernel(ConvArgs a) {
    pdl_launch_dependents();  // the conv-state kernel may start launching (it waits for this one)
    const int c0 = blockIdx.y * kChanPerCta + threadIdx.x * kVec;
    const bool active = c0 < a.C;
    const int64_t t0 = (int64_t)blockIdx.x * kTT;
    const int64_t t1 = (t0 + kTT < a.T_tot) ? t0 + kTT : a.T_tot;

    // Taps, right-aligned into a 4-wide window: y = sum_j wp[j] * x[t-3+j].
    float wp[4][8];
    if (a.K == 4 && active && (reinterpret_cast<uintptr_t>(a.w) & 15u) == 0) {
        // the thread's 8 x 4 taps are 32 contiguous values
        const T* wr = static_cast<const T*>(a.w) + (int64_t)c0 * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            Raw8<T> r;
            r.load(wr + 8 * q);
            float f[8];
            r.get(f);
#pragma unroll
            for (int e = 0; e < 8; ++e) wp[e & 3][2 * q + (e >> 2)] = f[e];  // channel 2q + e/4, tap e%4
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int jj = j - (4 - a.K);
                wp[j][i] = (active && jj >= 0)
                               ? Elem<T>::load(static_cast<const T*>(a.w), (int64_t)(c0 + i) * a.K + jj)
                               : 0.f;
            }
    }

    int n = find_sequence(a.cu, a.N, t0);
    int64_t seq_start = a.cu[n], seq_end = a.cu[n + 1];
    if (!(seq_start >= 0 && seq_start <= t0 && t0 < seq_end && seq_end <= a.T_tot)) {
        if (threadIdx.x == 0) set_status(a.status, kStatusBadSeqlens);
        return;
    }
    const int lanes_per_head = a.head_dim / kVec;
    const bool norm_me = a.qk_l2norm && c0 < a.n_qk;
    if (t0 - 3 >= seq_start && t1 <= seq_end) {
        // All rows of the window in one sequence: issue every load first.
        Raw8<T> r[kTT + 3];
        const T* xp = static_cast<const T*>(a.x) + (t0 - 3) * a.C + c0;
#pragma unroll
        for (int u = 0; u < kTT + 3; ++u)
            if (active && t0 - 3 + u < t1) r[u].load(xp + (int64_t)u * a.C);
        if constexpr (std::is_same<T, uint16_t>::value) {
            // bf16: packed fp32 pairs (two channels per FFMA2), one-XU SiLU, pair
            // packing to bf16 -- about 10 instructions per element
            float2 w2[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int p = 0; p < 4; ++p) w2[j][p] = make_float2(wp[j][2 * p], wp[j][2 * p + 1]);
            float2 xm3[4], xm2[4], xm1[4];
            Pairs<T>::get(r[0].u, xm3);
            Pairs<T>::get(r[1].u, xm2);
            Pairs<T>::get(r[2].u, xm1);
#pragma unroll
            for (int u = 0; u < kTT; ++u) {
                const int64_t t = t0 + u;
                if (t >= t1) break;  // uniform over the CTA
                float2 xt[4], y[4];
                Pairs<T>::get(r[u + 3].u, xt);
                float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    float2 acc = __fmul2_rn(w2[0][p], xm3[p]);
                    acc = __ffma2_rn(w2[1][p], xm2[p], acc);
                    acc = __ffma2_rn(w2[2][p], xm1[p], acc);
                    acc = __ffma2_rn(w2[3][p], xt[p], acc);
                    acc = make_float2(silu_tanh(acc.x), silu_tanh(acc.y));
                    y[p] = acc;
                    ss2 = __ffma2_rn(acc, acc, ss2);
                }
                if (a.qk_l2norm) {
                    const float ss = group_sum(ss2.x + ss2.y, lanes_per_head);
                    if (norm_me) {
                        const float inv = rsqrtf(ss + a.eps);
#pragma unroll
                        for (int p = 0; p < 4; ++p) y[p] = __fmul2_rn(y[p], make_float2(inv, inv));
                    }
                }
                if (active) {
                    __nv_bfloat162 o[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) o[p] = __floats2bfloat162_rn(y[p].x, y[p].y);
                    *reinterpret_cast<uint4*>(static_cast<T*>(a.y) + t * a.C + c0) = *reinterpret_cast<uint4*>(o);
                }
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    xm3[p] = xm2[p];
                    xm2[p] = xm1[p];
                    xm1[p] = xt[p];
                }
            }
            return;
        }
        float xm3[8], xm2[8], xm1[8];
        r[0].get(xm3);
        r[1].get(xm2);
        r[2].get(xm1);
#pragma unroll
        for (int u = 0; u < kTT; ++u) {
            const int64_t t = t0 + u;
            if (t >= t1) break;  // uniform over the CTA
            float xt[8], y[8];
            r[u + 3].get(xt);
            float ss = conv_token<T>(wp, xm3, xm2, xm1, xt, y);
            if (a.qk_l2norm) {
                ss = group_sum(ss, lanes_per_head);
                if (norm_me) {
                    const float inv = 1.f / sqrtf(ss + a.eps);
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] *= inv;
                }
            }
            if (active) Vec8<T>::store(static_cast<T*>(a.y) + t * a.C + c0, y);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                xm3[i] = xm2[i];
                xm2[i] = xm1[i];
                xm1[i] = xt[i];
            }
        }
        return;
    }
    float xm3[8], xm2[8], xm1[8], xt[8];
    fetch<T>(a, n, seq_start, t0 - 3, c0, active, xm3);
    fetch<T>(a, n, seq_start, t0 - 2, c0, active, xm2);
    fetch<T>(a, n, seq_start, t0 - 1, c0, active, xm1);

    for (int64_t t = t0; t < t1; ++t) {
        if (t == seq_end) {  // next non-empty sequence: window restarts from its state
            while (n + 1 < a.N && a.cu[n + 1] <= t) ++n;
            seq_start = a.cu[n];
            seq_end = a.cu[n + 1];
            if (!(seq_start == t && seq_end > t && seq_end <= a.T_tot)) {
                if (threadIdx.x == 0) set_status(a.status, kStatusBadSeqlens);
                return;
            }
            fetch<T>(a, n, seq_start, t - 3, c0, active, xm3);
            fetch<T>(a, n, seq_start, t - 2, c0, active, xm2);
            fetch<T>(a, n, seq_start, t - 1, c0, active, xm1);
        }
        fetch<T>(a, n, seq_start, t, c0, active, xt);
        float y[8];
        float ss = conv_token<T>(wp, xm3, xm2, xm1, xt, y);
        if (a.qk_l2norm) {  // every lane joins the shuffle; only q/k lanes use it
            ss = group_sum(ss, lanes_per_head);
            if (norm_me) {
                const float inv = 1.f / sqrtf(ss + a.eps);
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] *= inv;
            }
        }
        if (active) Vec8<T>::store(static_cast<T*>(a.y) + t * a.C + c0, y);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            xm3[i] = xm2[i];
            xm2[i] = xm1[i];
            xm1[i] = xt[i];
        }
    }
}

// conv_state_out[n, c, s] = input at relative position T_n - (K-1) + s.
template <typename T>
__global__ void conv_state_kernel(ConvArgs a) {
    // launched as a dependent of the conv kernel: the conv state may be updated
    // in place, so nothing is touched before that kernel has finished
    pdl_wait_previous();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)a.N * a.C) return;
    const int n = (int)(idx / a.C);
    const int c = (int)(idx % a.C);
    const int64_t start = a.cu[n], end = a.cu[n + 1];
    if (!(start >= 0 && start <= end && end <= a.T_tot)) {
        set_status(a.status, kStatusBadSeqlens);
        return;
    }
    const int W = a.K - 1;
    float vals[3];
    for (int s = 0; s < W; ++s) {
        const int64_t rel = (end - start) - W + s;
        float v = 0.f;
        if (rel >= 0)
            v = Elem<T>::load(static_cast<const T*>(a.x), (start + rel) * a.C + c);
        else if (a.state_in && W + rel >= 0)
            v = Elem<T>::load(static_cast<const T*>(a.state_in), idx * W + (W + rel));
        vals[s] = v;
    }
    for (int s = 0; s < W; ++s) Elem<T>::store(static_cast<T*>(a.state_out), idx * W + s, vals[s]);
}

template <typename T>
cudaError_t launch_t(const ConvArgs& a, cudaStream_t s) {
    if (a.T_tot > 0) {
        dim3 grid((unsigned)((a.T_tot + kTT - 1) / kTT), (unsigned)((a.C + kChanPerCta - 1) / kChanPerCta));
        conv_silu_kernel<T><<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.state_out && a.N > 0 && a.K > 1) {
        const int64_t total = (int64_t)a.N * a.C;
        return launch_pdl(conv_state_kernel<T>, dim3((unsigned)((total + 255) / 256)), dim3(256), 0, s, a);
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_conv_silu(const ConvArgs& a, cudaStream_t s) {
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

cudaError_t launch_conv_state(const ConvArgs& a, cudaStream_t s) {
    if (!a.state_out || a.N <= 0 || a.K <= 1) return cudaSuccess;
    const int64_t total = (int64_t)a.N * a.C;
    const dim3 grid((unsigned)((total + 255) / 256));
    if (a.is_bf16)
        conv_state_kernel<uint16_t><<<grid, 256, 0, s>>>(a);
    else
        conv_state_kernel<float><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace gdn
