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
    return a.dv <= 128 ? launch_q<T, 1, 8>(a, s) : launch_q<T, 2, 4>(a, s);
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const GatedNormArgs& a, cudaStream_t s) {
    if (a.rows == 0) return cudaSuccess;
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
