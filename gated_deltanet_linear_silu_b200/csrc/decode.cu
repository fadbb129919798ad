// Recurrent single-token gated delta rule (decode), one CTA per (sequence, head).
//
// Rule ("Qwen3.5-MoE source walkthrough", 4.3, recurrent mode), state S [dk, dv]:
//   S <- exp(g) S;  m = S^T k;  delta = beta (v - m);  S <- S + k delta^T;  o = S^T q
// Both reductions are taken from the state as loaded, so the state crosses HBM
// exactly once in each direction:
//   a = S^T k^, b = S^T q^ (undecayed S),  m = alpha a,
//   delta = beta (v - m),  o = alpha b + (k^ . q^) delta,  S' = alpha S + k^ delta^T.
// Layout: thread (rg, cg) owns columns [4cg, 4cg+4) of rows [rg*RPT, rg*RPT+RPT);
// a warp reads whole 512-byte state rows (float4 per lane), fully coalesced.
// Grouped value heads (H = G * Hk): value head h reads q, k head h / G.
//
// The whole mixer for the decode token (conv update, SiLU, norms, this step and
// the gated output) is the persistent streaming kernel of decode_stream.cu.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

// Two CTAs of 256 threads per SM (128 registers a thread): the state streams
// from HBM, so the kernel needs both CTAs' loads in flight.
template <typename T, int RPT>
__global__ void __launch_bounds__(256, 2) decode_step_kernel(DecodeArgs a) {
    extern __shared__ float sm[];
    const int dk = a.dk, dv = a.dv;
    const int cols4 = dv >> 2;
    const int RG = dk / RPT;
    const int tid = threadIdx.x;
    const int cg = tid % cols4;
    const int rg = tid / cols4;
    const int64_t nh = blockIdx.x;  // n * H + h

    float* qs = sm;                   // [dk]
    float* ks = qs + dk;              // [dk]
    float* red = ks + dk;             // [2][RG][dv]
    float* scal = red + 2 * RG * dv;  // [4]: inv_k, q_scale, kq

    // 0. The next step may start launching; this one reads the state the
    // previous step wrote only after that step has finished.
    pdl_launch_dependents();
    pdl_wait_previous();

    // 1. Issue the state loads: they are the bulk of the traffic.
    float* Sg = a.state + nh * dk * dv;
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r)
        s[r] = __ldcs(reinterpret_cast<const float4*>(Sg + (int64_t)(rg * RPT + r) * dv + 4 * cg));

    {
        const int n = (int)(nh / a.H), hk = (int)(nh % a.H) / (a.H / a.Hk);
        const T* qg = static_cast<const T*>(a.q) + ((int64_t)n * a.Hk + hk) * dk;
        const T* kg = static_cast<const T*>(a.k) + ((int64_t)n * a.Hk + hk) * dk;
        for (int i = tid; i < dk; i += blockDim.x) {
            qs[i] = Elem<T>::load(qg, i);
            ks[i] = Elem<T>::load(kg, i);
        }
    }
    const float4 v4 = load4(static_cast<const T*>(a.v) + nh * dv + 4 * cg);
    const float alpha = expf(a.g[nh]);
    const float beta = a.beta[nh];
    __syncthreads();

    // 2. Norms and k.q (warp 0), broadcast through shared memory.
    if (tid < 32) {
        float sq = 0.f, sk = 0.f, kq = 0.f;
        for (int i = tid; i < dk; i += 32) {
            sq += qs[i] * qs[i];
            sk += ks[i] * ks[i];
            kq += qs[i] * ks[i];
        }
        sq = warp_sum(sq);
        sk = warp_sum(sk);
        kq = warp_sum(kq);
        if (tid == 0) {
            float inv_q = 1.f, inv_k = 1.f;
            if (a.qk_l2norm) {
                inv_q = 1.f / sqrtf(sq + a.eps);
                inv_k = 1.f / sqrtf(sk + a.eps);
            }
            scal[0] = inv_k;
            scal[1] = inv_q * a.scale;
            scal[2] = kq * inv_k * inv_q * a.scale;
        }
    }

    // 3. Partial S^T k and S^T q over this thread's rows (raw q, k).
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const float kv = ks[rg * RPT + r], qv = qs[rg * RPT + r];
        pa.x = fmaf(s[r].x, kv, pa.x); pa.y = fmaf(s[r].y, kv, pa.y);
        pa.z = fmaf(s[r].z, kv, pa.z); pa.w = fmaf(s[r].w, kv, pa.w);
        pb.x = fmaf(s[r].x, qv, pb.x); pb.y = fmaf(s[r].y, qv, pb.y);
        pb.z = fmaf(s[r].z, qv, pb.z); pb.w = fmaf(s[r].w, qv, pb.w);
    }
    *reinterpret_cast<float4*>(red + rg * dv + 4 * cg) = pa;
    *reinterpret_cast<float4*>(red + (RG + rg) * dv + 4 * cg) = pb;
    __syncthreads();

    float4 A = make_float4(0.f, 0.f, 0.f, 0.f), B = A;
    for (int r = 0; r < RG; ++r) {
        const float4 x = *reinterpret_cast<const float4*>(red + r * dv + 4 * cg);
        const float4 y = *reinterpret_cast<const float4*>(red + (RG + r) * dv + 4 * cg);
        A.x += x.x; A.y += x.y; A.z += x.z; A.w += x.w;
        B.x += y.x; B.y += y.y; B.z += y.z; B.w += y.w;
    }
    const float inv_k = scal[0], qsc = scal[1], kq = scal[2];

    // 4. delta, output, state update. The memory is alpha a (decay first) or a
    // (read from the state before the decay).
    const float mk = a.undecayed ? inv_k : alpha * inv_k;
    float4 d;
    d.x = beta * (v4.x - mk * A.x);
    d.y = beta * (v4.y - mk * A.y);
    d.z = beta * (v4.z - mk * A.z);
    d.w = beta * (v4.w - mk * A.w);
    if (rg == 0) {  // the output
        float4 o;
        o.x = alpha * qsc * B.x + kq * d.x;
        o.y = alpha * qsc * B.y + kq * d.y;
        o.z = alpha * qsc * B.z + kq * d.z;
        o.w = alpha * qsc * B.w + kq * d.w;
        store4(static_cast<T*>(a.o) + nh * dv + 4 * cg, o);
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const float kn = ks[rg * RPT + r] * inv_k;
        float4 x = s[r];
        x.x = fmaf(alpha, x.x, kn * d.x);
        x.y = fmaf(alpha, x.y, kn * d.y);
        x.z = fmaf(alpha, x.z, kn * d.z);
        x.w = fmaf(alpha, x.w, kn * d.w);
        __stcs(reinterpret_cast<float4*>(Sg + (int64_t)(rg * RPT + r) * dv + 4 * cg), x);
    }
}

template <typename T, int RPT>
cudaError_t launch_rpt(const DecodeArgs& a, cudaStream_t s) {
    const int cols4 = a.dv / 4;
    const int RG = a.dk / RPT;
    const int threads = cols4 * RG;
    const size_t smem = sizeof(float) * (2 * a.dk + 2 * RG * a.dv + 4);
    return launch_pdl(decode_step_kernel<T, RPT>, dim3((unsigned)((int64_t)a.N * a.H)), dim3(threads), smem, s, a);
}

template <typename T>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t s) {
    // Rows per thread: the smallest power of two (<= 16, dividing dk) that
    // keeps the CTA at <= 256 threads.
    const int need = (a.dk * (a.dv / 4) + 255) / 256;
    int rpt = 1;
    while (rpt < need) rpt <<= 1;
    switch (rpt) {
        case 1: return launch_rpt<T, 1>(a, s);
        case 2: return launch_rpt<T, 2>(a, s);
        case 4: return launch_rpt<T, 4>(a, s);
        case 8: return launch_rpt<T, 8>(a, s);
        default: return launch_rpt<T, 16>(a, s);
    }
}

}  // namespace

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s) {
    if ((int64_t)a.N * a.H == 0) return cudaSuccess;
    if (a.x)  // the whole-mixer step
        return decode_stream_supported(a) ? launch_decode_stream(a, s) : cudaErrorNotSupported;
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
