// Gated RMSNorm output of the linear-attention layer over rows of d_v features
// ("7.6 Qwen3.5: linear-attention hybrid", 7.6.2 gated RMSNorm output; RMSNorm
// as in 7.6.3):
//   out = y / sqrt(mean(y^2) + eps) * w * SiLU(z),   SiLU(z) = z / (1 + e^-z).
// HBM-bound (read y and z, write out, once each): one warp per row, four
// features per lane per pass, each warp keeping four rows' loads in flight
// before the first reduction; w stays in registers.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 4;  // rows in flight per warp
constexpr int kMaxQuads = 2;     // dv / 4 / 32 <= 2, i.e. dv <= 256

__device__ __forceinline__ float silu_g(float x) { return __fdividef(x, 1.f + __expf(-x)); }

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) gated_rmsnorm_kernel(GatedNormArgs a) {
    const int lane = threadIdx.x & 31;
    const int dv = a.dv, quads = dv >> 2;
    float4 w4[kMaxQuads];
#pragma unroll
    for (int p = 0; p < kMaxQuads; ++p) {
        const int qd = lane + 32 * p;
        w4[p] = qd < quads ? *reinterpret_cast<const float4*>(a.w + 4 * qd) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int64_t warp_id = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    const T* y = static_cast<const T*>(a.y);
    const T* z = static_cast<const T*>(a.z);
    T* out = static_cast<T*>(a.out);
    for (int64_t r0 = warp_id * kRowsPerWarp; r0 < a.rows; r0 += nwarps * kRowsPerWarp) {
        float4 yv[kRowsPerWarp][kMaxQuads], zv[kRowsPerWarp][kMaxQuads];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i)
#pragma unroll
            for (int p = 0; p < kMaxQuads; ++p) {
                const int qd = lane + 32 * p;
                const bool ok = r0 + i < a.rows && qd < quads;
                const int64_t off = (r0 + i) * dv + 4 * qd;
                yv[i][p] = ok ? load4(y + off) : make_float4(0.f, 0.f, 0.f, 0.f);
                zv[i][p] = ok ? load4(z + off) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            float ss = 0.f;
#pragma unroll
            for (int p = 0; p < kMaxQuads; ++p) {
                const float4 v = yv[i][p];
                ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
            }
            ss = warp_sum(ss);
            if (r0 + i >= a.rows) continue;  // uniform over the warp
            const float inv = 1.f / sqrtf(ss / (float)dv + a.eps);
#pragma unroll
            for (int p = 0; p < kMaxQuads; ++p) {
                const int qd = lane + 32 * p;
                if (qd >= quads) continue;
                const float4 v = yv[i][p], g = zv[i][p], s = w4[p];
                float4 o;
                o.x = v.x * inv * s.x * silu_g(g.x);
                o.y = v.y * inv * s.y * silu_g(g.y);
                o.z = v.z * inv * s.z * silu_g(g.z);
                o.w = v.w * inv * s.w * silu_g(g.w);
                store4(out + (r0 + i) * dv + 4 * qd, o);
            }
        }
    }
}

template <typename T>
cudaError_t launch_t(const GatedNormArgs& a, cudaStream_t s) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t need = (a.rows + (int64_t)kWarps * kRowsPerWarp - 1) / ((int64_t)kWarps * kRowsPerWarp);
    const int64_t cap = (int64_t)sms * 8;  // 8 CTAs of 8 warps per SM
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    gated_rmsnorm_kernel<T><<<grid, kWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const GatedNormArgs& a, cudaStream_t s) {
    if (a.rows == 0) return cudaSuccess;
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
