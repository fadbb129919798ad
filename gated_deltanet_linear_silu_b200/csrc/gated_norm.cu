// Gated RMSNorm output of the linear-attention layer over rows of d_v features
// ("7.6 Qwen3.5: linear-attention hybrid", 7.6.2 gated RMSNorm output; RMSNorm
// as in 7.6.3):
//   out = y / sqrt(mean(y^2) + eps) * w * SiLU(z),   SiLU(z) = z / (1 + e^-z).
// HBM-bound (read y and z, write out, once each): one warp per row, four
// features per lane per pass; each warp keeps two batches of eight rows' loads
// in flight (raw, streaming): the next batch is requested before the current one
// is reduced and written. w stays in registers.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ float silu_g(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// Four features of a row as loaded (bf16: 8 bytes, fp32: 16 bytes).
template <typename T> struct Raw4;
template <> struct Raw4<uint16_t> {
    uint2 u;
    __device__ __forceinline__ void load(const uint16_t* p) { u = __ldcs(reinterpret_cast<const uint2*>(p)); }
    __device__ __forceinline__ float4 get() const {
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
};
template <> struct Raw4<float> {
    float4 f;
    __device__ __forceinline__ void load(const float* p) { f = __ldcs(reinterpret_cast<const float4*>(p)); }
    __device__ __forceinline__ float4 get() const { return f; }
};

// One warp per row; QUADS groups of four features per lane (dv <= 128 * QUADS);
// each warp keeps ROWS rows' loads in flight (held raw) before the first
// reduction.
template <typename T, int QUADS, int ROWS>
__global__ void __launch_bounds__(kWarps * 32) gated_rmsnorm_kernel(GatedNormArgs a) {
    const int lane = threadIdx.x & 31;
    const int dv = a.dv, quads = dv >> 2;
    float4 w4[QUADS];
#pragma unroll
    for (int p = 0; p < QUADS; ++p) {
        const int qd = lane + 32 * p;
        w4[p] = qd < quads ? *reinterpret_cast<const float4*>(a.w + 4 * qd) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int64_t warp_id = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    const T* y = static_cast<const T*>(a.y);
    const T* z = static_cast<const T*>(a.z);
    T* out = static_cast<T*>(a.out);
    const int64_t stride = nwarps * ROWS;
    // two batches of ROWS rows in flight: the next batch's loads are issued before
    // the current one is reduced and written
    Raw4<T> ya[ROWS][QUADS], za[ROWS][QUADS], yb[ROWS][QUADS], zb[ROWS][QUADS];
    auto load = [&](Raw4<T> (&yv)[ROWS][QUADS], Raw4<T> (&zv)[ROWS][QUADS], int64_t r0) {
#pragma unroll
        for (int i = 0; i < ROWS; ++i)
#pragma unroll
            for (int p = 0; p < QUADS; ++p) {
                const int qd = lane + 32 * p;
                if (r0 + i < a.rows && qd < quads) {
                    const int64_t off = (r0 + i) * dv + 4 * qd;
                    yv[i][p].load(y + off);
                    zv[i][p].load(z + off);
                }
            }
    };
    auto finish = [&](const Raw4<T> (&yv)[ROWS][QUADS], const Raw4<T> (&zv)[ROWS][QUADS], int64_t r0) {
#pragma unroll
        for (int i = 0; i < ROWS; ++i) {
            float4 v[QUADS];
            float ss = 0.f;
#pragma unroll
            for (int p = 0; p < QUADS; ++p) {
                const int qd = lane + 32 * p;
                v[p] = (r0 + i < a.rows && qd < quads) ? yv[i][p].get() : make_float4(0.f, 0.f, 0.f, 0.f);
                ss += v[p].x * v[p].x + v[p].y * v[p].y + v[p].z * v[p].z + v[p].w * v[p].w;
            }
            ss = warp_sum(ss);
            if (r0 + i >= a.rows) continue;  // uniform over the warp
            const float inv = 1.f / sqrtf(ss / (float)dv + a.eps);
#pragma unroll
            for (int p = 0; p < QUADS; ++p) {
                const int qd = lane + 32 * p;
                if (qd >= quads) continue;
                const float4 g = zv[i][p].get(), s = w4[p];
                float4 o;
                o.x = v[p].x * inv * s.x * silu_g(g.x);
                o.y = v[p].y * inv * s.y * silu_g(g.y);
                o.z = v[p].z * inv * s.z * silu_g(g.z);
                o.w = v[p].w * inv * s.w * silu_g(g.w);
                store4(out + (r0 + i) * dv + 4 * qd, o);
            }
        }
    };
    int64_t r0 = warp_id * ROWS;
    if (r0 < a.rows) load(ya, za, r0);
    while (r0 < a.rows) {
        const int64_t r1 = r0 + stride;
        if (r1 < a.rows) load(yb, zb, r1);
        finish(ya, za, r0);
        if (r1 >= a.rows) break;
        const int64_t r2 = r1 + stride;
        if (r2 < a.rows) load(ya, za, r2);
        finish(yb, zb, r1);
        r0 = r2;
    }
}

// d_v = 128: half a warp per row, eight features per lane (one 16-byte bf16
// vector), so a warp finishes two rows per pass with a 4-step shuffle
// reduction; eight row pairs in flight per warp; no bounds checks on full batches.
template <typename T> struct Raw8;
template <> struct Raw8<uint16_t> {
    uint4 u;
    __device__ __forceinline__ void load(const uint16_t* p) { u = __ldcs(reinterpret_cast<const uint4*>(p)); }
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
        a = __ldcs(reinterpret_cast<const float4*>(p));
        b = __ldcs(reinterpret_cast<const float4*>(p + 4));
    }
    __device__ __forceinline__ void get(float (&x)[8]) const {
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};
__device__ __forceinline__ void store8(uint16_t* p, const float (&x)[8]) {
    uint4 u;
    u.x = (uint32_t)f32_to_bf16(x[0]) | ((uint32_t)f32_to_bf16(x[1]) << 16);
    u.y = (uint32_t)f32_to_bf16(x[2]) | ((uint32_t)f32_to_bf16(x[3]) << 16);
    u.z = (uint32_t)f32_to_bf16(x[4]) | ((uint32_t)f32_to_bf16(x[5]) << 16);
    u.w = (uint32_t)f32_to_bf16(x[6]) | ((uint32_t)f32_to_bf16(x[7]) << 16);
    *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float (&x)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) gated_rmsnorm_d128_kernel(GatedNormArgs a) {
    constexpr int kPairs = 8;  // row pairs in flight per warp
    const int lane = threadIdx.x & 31, half = lane >> 4, l16 = lane & 15;
    float w8[8];
    {
        const float4 p = *reinterpret_cast<const float4*>(a.w + 8 * l16);
        const float4 q = *reinterpret_cast<const float4*>(a.w + 8 * l16 + 4);
        w8[0] = p.x; w8[1] = p.y; w8[2] = p.z; w8[3] = p.w;
        w8[4] = q.x; w8[5] = q.y; w8[6] = q.z; w8[7] = q.w;
    }
    const int64_t warp_id = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    const T* y = static_cast<const T*>(a.y);
    const T* z = static_cast<const T*>(a.z);
    T* out = static_cast<T*>(a.out);
    constexpr int64_t kRows = 2 * kPairs;
    for (int64_t r0 = warp_id * kRows; r0 < a.rows; r0 += nwarps * kRows) {
        const bool full = r0 + kRows <= a.rows;
        Raw8<T> yv[kPairs], zv[kPairs];
#pragma unroll
        for (int i = 0; i < kPairs; ++i) {
            const int64_t r = r0 + 2 * i + half;
            if (full || r < a.rows) {
                yv[i].load(y + r * 128 + 8 * l16);
                zv[i].load(z + r * 128 + 8 * l16);
            }
        }
#pragma unroll
        for (int i = 0; i < kPairs; ++i) {
            const int64_t r = r0 + 2 * i + half;
            float v[8];
            yv[i].get(v);
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (!full && r >= a.rows) continue;
            const float inv = 1.f / sqrtf(ss * (1.f / 128.f) + a.eps);
            float g[8];
            zv[i].get(g);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = v[e] * inv * w8[e] * silu_g(g[e]);
            store8(out + r * 128 + 8 * l16, v);
        }
    }
}

template <typename T, int QUADS, int ROWS>
cudaError_t launch_q(const GatedNormArgs& a, cudaStream_t s) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t per_cta = (int64_t)kWarps * ROWS;
    const int64_t need = (a.rows + per_cta - 1) / per_cta;
    const int64_t cap = (int64_t)sms * 16;  // up to 16 CTAs of 4 warps per SM
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    gated_rmsnorm_kernel<T, QUADS, ROWS><<<grid, kWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const GatedNormArgs& a, cudaStream_t s) {
    if (a.dv == 128) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t per_cta = (int64_t)kWarps * 16;
        const int64_t need = (a.rows + per_cta - 1) / per_cta;
        const int64_t cap = (int64_t)sms * 16;
        gated_rmsnorm_d128_kernel<T><<<(unsigned)(need < cap ? need : cap), kWarps * 32, 0, s>>>(a);
        return cudaGetLastError();
    }
    return a.dv <= 128 ? launch_q<T, 1, 8>(a, s) : launch_q<T, 2, 4>(a, s);
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const GatedNormArgs& a, cudaStream_t s) {
    if (a.rows == 0) return cudaSuccess;
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
