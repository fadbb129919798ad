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
//
// The same kernel runs the whole mixer for the decode token when CONV is set
// ("7.6 Qwen3.5: linear-attention hybrid", 7.6.2): the CTA of (n, h) owns the
// conv channels of its head's q, k and v, so it applies the causal conv to the
// token's fused projections against the conv state, shifts that state, and
// applies SiLU before the recurrent step -- q, k, v never leave the SM. With a
// gate z the output goes through the gated RMSNorm of 7.6.2 (RMSNorm as in
// 7.6.3, scale vector as given) on the way out.
//
// Grouped value heads (H = G * Hk, the config's linear_num_value_heads over
// linear_num_key_heads, 7.6.1): value head h reads q, k head h / G. In the
// whole-mixer step the G CTAs of one group all need the group's q, k conv
// channels; they run as one thread-block cluster, every CTA computes those
// channels' conv from the old conv state, and after a cluster barrier (every
// CTA has read the old state) only the group's first CTA writes the shifted
// q, k conv state back.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// Cluster-wide barrier in two halves (hardware barrier; no spinning in code).
// The arrive is relaxed: what it has to order are reads of the conv state that
// have already completed (cp.async waited, the data is in shared memory), and
// a release would also wait for the state loads still in flight.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Two CTAs of 256 threads per SM (128 registers a thread): the state streams
// from HBM, so the kernel needs both CTAs' loads in flight.
template <typename T, int RPT, bool CONV>
__global__ void __launch_bounds__(256, 2) decode_step_kernel(DecodeArgs a) {
    extern __shared__ float sm[];
    const int dk = a.dk, dv = a.dv;
    const int cols4 = dv >> 2;
    const int RG = dk / RPT;
    const int tid = threadIdx.x;
    const int cg = tid % cols4;
    const int rg = tid / cols4;
    const int64_t nh = blockIdx.x;  // n * H + h

    float* qs = sm;              // [dk]
    float* ks = qs + dk;         // [dk]
    float* red = ks + dk;        // [2][RG][dv]
    float* scal = red + 2 * RG * dv;  // [4]: inv_k, q_scale, kq
    float* vs = scal + 4;        // [dv] (CONV only)

    // 0. (whole-mixer step) the conv inputs of this head's q, k, v channels -- x,
    // the taps and the conv state, a few KB -- are copied to shared memory
    // asynchronously ahead of the state's 64 KB, so they are in when needed and
    // hold no registers meanwhile. Three contiguous channel blocks: q (dk channels
    // from hk*dk), k (dk from Hk*dk + hk*dk), v (dv from 2*Hk*dk + h*dv).
    const int nconv = 2 * dk + dv;
    T* cx_s = reinterpret_cast<T*>(vs + dv);          // [nconv]
    T* cw_s = cx_s + nconv;                           // [nconv][K]
    T* cs_s = cw_s + nconv * a.K;                     // [nconv][K-1]
    if constexpr (CONV) {
        const int H = a.H, Hk = a.Hk, G = H / Hk, K = a.K;
        const int n = (int)(nh / H), h = (int)(nh % H), hk = h / G;
        const int64_t C = 2 * Hk * dk + H * dv;
        const T* x = static_cast<const T*>(a.x) + n * C;
        const T* w = static_cast<const T*>(a.conv_w);
        const T* cs = static_cast<const T*>(a.conv_state) + n * C * (K - 1);
        constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte piece
#pragma unroll
        for (int b = 0; b < 3; ++b) {
            const int nb = b < 2 ? dk : dv;                       // channels in the block
            const int64_t ch0 = b == 0 ? hk * dk : (b == 1 ? Hk * dk + hk * dk : 2 * Hk * dk + h * dv);
            const int c0 = b == 0 ? 0 : (b == 1 ? dk : 2 * dk);  // first local channel
            for (int p = tid; p < nb / E; p += blockDim.x) cp_async_16(cx_s + c0 + p * E, x + ch0 + p * E);
            for (int p = tid; p < nb * K / E; p += blockDim.x)
                cp_async_16(cw_s + c0 * K + p * E, w + ch0 * K + p * E);
            for (int p = tid; p < nb * (K - 1) / E; p += blockDim.x)
                cp_async_16(cs_s + c0 * (K - 1) + p * E, cs + ch0 * (K - 1) + p * E);
        }
        cp_async_commit_group();
    }

    // 1. Issue the state loads: they are the bulk of the traffic.
    float* Sg = a.state + nh * dk * dv;
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r)
        s[r] = __ldcs(reinterpret_cast<const float4*>(Sg + (int64_t)(rg * RPT + r) * dv + 4 * cg));

    float4 v4;
    if constexpr (CONV) {
        // causal conv of this head's q, k, v channels against the conv state
        // (window: the K-1 stored inputs, oldest first, then x); the state shifts
        // by one and takes x as its newest entry
        const int H = a.H, Hk = a.Hk, G = H / Hk, K = a.K;
        const int n = (int)(nh / H), h = (int)(nh % H), hk = h / G;
        const int64_t C = 2 * Hk * dk + H * dv;
        T* cs = static_cast<T*>(a.conv_state) + n * C * (K - 1);
        cp_async_wait_all_groups();
        __syncthreads();
        if (G > 1) cluster_arrive_relaxed();  // this CTA's copy of the old conv state is in
        for (int c = tid; c < nconv; c += blockDim.x) {
            const float xt = Elem<T>::load(cx_s, c);
            float acc;
            if (K == 4) {
                const float4 w4 = load4(cw_s + 4 * c);  // the channel's four taps at once
                const float p0 = Elem<T>::load(cs_s, 3 * c), p1 = Elem<T>::load(cs_s, 3 * c + 1),
                            p2 = Elem<T>::load(cs_s, 3 * c + 2);
                acc = fmaf(w4.x, p0, fmaf(w4.y, p1, fmaf(w4.z, p2, w4.w * xt)));
                Elem<T>::store(cs_s, 3 * c, p1);  // shifted state, stored below
                Elem<T>::store(cs_s, 3 * c + 1, p2);
                Elem<T>::store(cs_s, 3 * c + 2, xt);
            } else {
                float pv[3] = {0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    if (j < K - 1) pv[j] = Elem<T>::load(cs_s, c * (K - 1) + j);
                acc = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float in = (j == K - 1) ? xt : (j < K - 1 ? pv[j < 3 ? j : 2] : 0.f);
                    if (j < K) acc = fmaf(Elem<T>::load(cw_s, c * K + j), in, acc);
                }
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    if (j < K - 1) Elem<T>::store(cs_s, c * (K - 1) + j, j < K - 2 ? pv[j < 2 ? j + 1 : 2] : xt);
            }
            const float y = silu_f(acc);
            if (c < dk) qs[c] = y;
            else if (c < 2 * dk) ks[c - dk] = y;
            else vs[c - 2 * dk] = y;
        }
        __syncthreads();
        if (G > 1) cluster_wait_acquire();  // every CTA of the group has read the old state
        // the shifted conv state back to global memory, 16 bytes per store (the
        // shared q, k channels by the group's first CTA only)
        if (K > 1) {
            constexpr int E = 16 / (int)sizeof(T);
#pragma unroll
            for (int b = 0; b < 3; ++b) {
                if (b < 2 && h % G != 0) continue;
                const int nb = b < 2 ? dk : dv;
                const int64_t ch0 = b == 0 ? hk * dk : (b == 1 ? Hk * dk + hk * dk : 2 * Hk * dk + h * dv);
                const int c0 = b == 0 ? 0 : (b == 1 ? dk : 2 * dk);
                for (int p = tid; p < nb * (K - 1) / E; p += blockDim.x)
                    *reinterpret_cast<uint4*>(cs + ch0 * (K - 1) + p * E) =
                        *reinterpret_cast<const uint4*>(cs_s + c0 * (K - 1) + p * E);
            }
        }
        __syncthreads();
        v4 = *reinterpret_cast<const float4*>(vs + 4 * cg);
    } else {
        const int n = (int)(nh / a.H), hk = (int)(nh % a.H) / (a.H / a.Hk);
        const T* qg = static_cast<const T*>(a.q) + ((int64_t)n * a.Hk + hk) * dk;
        const T* kg = static_cast<const T*>(a.k) + ((int64_t)n * a.Hk + hk) * dk;
        for (int i = tid; i < dk; i += blockDim.x) {
            qs[i] = Elem<T>::load(qg, i);
            ks[i] = Elem<T>::load(kg, i);
        }
        v4 = load4(static_cast<const T*>(a.v) + nh * dv + 4 * cg);
    }
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
    // output: the rg == 0 threads, all in warp 0 (dv / 4 <= 32 columns groups)
    if (tid < 32) {
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        if (rg == 0) {
            o.x = alpha * qsc * B.x + kq * d.x;
            o.y = alpha * qsc * B.y + kq * d.y;
            o.z = alpha * qsc * B.z + kq * d.z;
            o.w = alpha * qsc * B.w + kq * d.w;
        }
        if (a.z) {  // gated RMSNorm over this head's dv outputs
            float ss = o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
            ss = warp_sum(ss);
            const float inv = 1.f / sqrtf(ss / (float)dv + a.norm_eps);
            if (rg == 0) {
                const float4 z4 = load4(static_cast<const T*>(a.z) + nh * dv + 4 * cg);
                const float4 w4 = *reinterpret_cast<const float4*>(a.norm_w + 4 * cg);
                o.x = o.x * inv * w4.x * silu_f(z4.x);
                o.y = o.y * inv * w4.y * silu_f(z4.y);
                o.z = o.z * inv * w4.z * silu_f(z4.z);
                o.w = o.w * inv * w4.w * silu_f(z4.w);
            }
        }
        if (rg == 0) store4(static_cast<T*>(a.o) + nh * dv + 4 * cg, o);
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
    size_t smem = sizeof(float) * (2 * a.dk + 2 * RG * a.dv + 4 + a.dv);
    if (a.x)  // conv inputs: x, taps, conv state of the head's channels
        smem += (size_t)(2 * a.dk + a.dv) * (2 * a.K) * (a.is_bf16 ? 2 : 4);
    const int64_t blocks = (int64_t)a.N * a.H;
    const int G = a.H / a.Hk;
    if (a.x && G > 1) {  // one cluster per group of value heads sharing a q, k head
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)blocks);
        cfg.blockDim = dim3(threads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = G;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, decode_step_kernel<T, RPT, true>, a);
    }
    if (a.x)
        decode_step_kernel<T, RPT, true><<<(unsigned)blocks, threads, smem, s>>>(a);
    else
        decode_step_kernel<T, RPT, false><<<(unsigned)blocks, threads, smem, s>>>(a);
    return cudaGetLastError();
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
    if (decode_stream_supported(a)) return launch_decode_stream(a, s);
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
