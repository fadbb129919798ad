// The whole mixer for one decode token as a persistent streaming kernel: two
// CTAs per SM walk the (sequence, head) units; each CTA brings its next unit's
// fp32 state (dk x dv, contiguous) and conv inputs into a shared-memory slot
// with bulk copies while it computes the current unit from registers, so the
// state load of one unit overlaps the conv, the arithmetic and the state store
// of the previous one. (The plain step, without the conv, keeps the
// per-(sequence, head) kernel: with less work per unit, its CTAs already keep
// enough state loads in flight.)
//
// Rule ("Qwen3.5-MoE source walkthrough", 4.3, recurrent mode), state S [dk, dv]:
//   S <- exp(g) S;  m = S^T k;  delta = beta (v - m);  S <- S + k delta^T;  o = S^T q
// with both reductions taken from the state as loaded (a = S^T k^, b = S^T q^,
// m = alpha a (or a: memory read before the decay), o = alpha b + (k^.q^) delta,
// S' = alpha S + k^ delta^T), so the state crosses HBM once each way. The unit
// first applies the causal conv update of its head's q, k, v channels ("7.6
// Qwen3.5: linear-attention hybrid", 7.6.2; conv state = the K-1 latest
// inputs) and SiLU; with a gate z the output goes through the gated RMSNorm.
// Value heads that share q, k heads (grouped) keep the per-(sequence, head)
// kernel, whose clusters share the q, k conv channels.
//
// Thread (rg, cg) owns columns [4cg, 4cg+4) of rows [rg*RPT, rg*RPT+RPT). The
// squared norms of q and k and their dot product are summed in the phase that
// produces q and k (thread j makes q_j and k_j), one partial per warp, added in
// a fixed order, so results do not depend on timing.
//
// The only wait, thread 0's on the slot's copy, is bounded: on timeout it
// records the timeout status, the CTA leaves its loop, waits (bounded) for
// the copy in flight and returns.
#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCtasPerSm = 2;
constexpr uint64_t kDrainNs = kDefaultWaitNs / 4;

__device__ __forceinline__ float silu_s(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// Bounded wait on the slot's copy; limit 0: only a copy already complete at
// the first probe passes.
__device__ __noinline__ bool wait_slot(uint64_t* bar, uint32_t parity, uint64_t limit) {
    if (limit == 0) return mbar_test_wait(bar, parity);
    if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 100000u))
        if (globaltimer_ns() - t0 > limit) return false;
    return true;
}

struct Geometry {
    uint32_t state_bytes, in_bytes, z_off, slot_bytes, fixed_off, smem;
};

// Slot = [state fp32 dk x dv][x, taps, conv state of the head's nconv =
// 2 dk + dv channels][gate z, when given], 128-byte aligned; then q, k, v in
// fp32, the reduction buffer [2][RG][dv], the per-warp norm partials
// [kWarps][4] and the barrier.
Geometry geometry(const DecodeArgs& a, int rpt) {
    Geometry g;
    const int nconv = 2 * a.dk + a.dv;
    const int esz = a.is_bf16 ? 2 : 4;
    g.state_bytes = (uint32_t)(a.dk * a.dv * 4);
    g.z_off = g.state_bytes + (uint32_t)(nconv * 2 * a.K * esz);
    g.in_bytes = g.z_off - g.state_bytes + (uint32_t)(a.z ? a.dv * esz : 0);
    g.slot_bytes = (g.state_bytes + g.in_bytes + 127u) & ~127u;
    g.fixed_off = g.slot_bytes;
    const uint32_t fixed = (uint32_t)(4 * nconv + 4 * 2 * (a.dk / rpt) * a.dv + 16 * kWarps + 16);
    g.smem = g.fixed_off + fixed + 128;  // + alignment slack
    return g;
}

// Issue the bulk copies of unit u into the slot (one thread).
template <typename T>
__device__ __forceinline__ void load_unit(const DecodeArgs& a, const Geometry& geo, uint8_t* sl, int64_t u,
                                          uint64_t* full) {
    const int dk = a.dk, dv = a.dv, H = a.H, K = a.K;
    const int nconv = 2 * dk + dv;
    mbar_arrive_expect_tx(full, geo.state_bytes + geo.in_bytes);
    bulk_load(sl, a.state + u * dk * dv, geo.state_bytes, full);
    const int n = (int)(u / H), h = (int)(u % H);
    const int64_t C = 2 * (int64_t)H * dk + (int64_t)H * dv;
    const T* x = static_cast<const T*>(a.x) + n * C;
    const T* w = static_cast<const T*>(a.conv_w);
    const T* cs = static_cast<const T*>(a.conv_state) + n * C * (K - 1);
    T* cx = reinterpret_cast<T*>(sl + geo.state_bytes);
    T* cw = cx + nconv;
    T* ccs = cw + nconv * K;
#pragma unroll
    for (int b = 0; b < 3; ++b) {  // q, k, v channel blocks of the head
        const int nb = b < 2 ? dk : dv;
        const int64_t ch0 = b == 0 ? (int64_t)h * dk : (b == 1 ? (int64_t)H * dk + h * dk : 2 * (int64_t)H * dk + h * dv);
        const int c0 = b == 0 ? 0 : (b == 1 ? dk : 2 * dk);
        bulk_load(cx + c0, x + ch0, nb * sizeof(T), full);
        bulk_load(cw + c0 * K, w + ch0 * K, nb * K * sizeof(T), full);
        if (K > 1) bulk_load(ccs + c0 * (K - 1), cs + ch0 * (K - 1), nb * (K - 1) * sizeof(T), full);
    }
    if (a.z) bulk_load(sl + geo.z_off, static_cast<const T*>(a.z) + u * dv, dv * sizeof(T), full);
}

// Causal conv of one channel (local index c of the slot's nconv) against its
// K-1 stored inputs (oldest first), then x; the shifted conv state goes back
// to global channel ch. Returns SiLU of the conv.
template <typename T>
__device__ __forceinline__ float conv_channel(const T* cx, const T* cw, const T* ccs, T* cs, int c, int64_t ch,
                                              int K) {
    const float xt = Elem<T>::load(cx, c);
    float pv[3] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 3; ++j)
        if (j < K - 1) pv[j] = Elem<T>::load(ccs, c * (K - 1) + j);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (j < K) acc = fmaf(Elem<T>::load(cw, c * K + j), j == K - 1 ? xt : pv[j < 3 ? j : 2], acc);
#pragma unroll
    for (int j = 0; j < 3; ++j)
        if (j < K - 1) Elem<T>::store(cs, ch * (K - 1) + j, j < K - 2 ? pv[j + 1 < 3 ? j + 1 : 2] : xt);
    return silu_s(acc);
}

template <typename T, int RPT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_layer_stream_kernel(DecodeArgs a, Geometry geo) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sl = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const int dk = a.dk, dv = a.dv;
    const int cols4 = dv >> 2;
    const int RG = dk / RPT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nthr = cols4 * RG;  // threads with state rows (<= kThreads)
    const int cg = tid % cols4, rg = tid / cols4;
    const int nconv = 2 * dk + dv;
    const int64_t total = (int64_t)a.N * a.H;
    const int H = a.H, K = a.K;

    const float* Ss = reinterpret_cast<const float*>(sl);
    const T* cx = reinterpret_cast<const T*>(sl + geo.state_bytes);  // [nconv]
    const T* cw = cx + nconv;                                           // [nconv][K]
    const T* ccs = cw + nconv * K;                                      // [nconv][K-1]
    float* qs = reinterpret_cast<float*>(sl + geo.fixed_off);  // [dk]
    float* ks = qs + dk;                                         // [dk]
    float* vs = ks + dk;                                         // [dv]
    float* red = vs + dv;                                        // [2][RG][dv]
    float4* part = reinterpret_cast<float4*>(red + 2 * RG * dv);  // [kWarps]: |q|^2, |k|^2, q.k
    uint64_t* full = reinterpret_cast<uint64_t*>(part + kWarps);

    int64_t u = blockIdx.x;
    if (tid == 0) {
        mbar_init(full, 1);
        fence_mbar_init();
        if (u < total) load_unit<T>(a, geo, sl, u, full);
    }
    float g_next = 0.f, b_next = 0.f;  // gate and beta one unit ahead
    if (u < total) {
        g_next = a.g[u];
        b_next = a.beta[u];
    }
    float4 nw4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.z && tid < cols4) nw4 = *reinterpret_cast<const float4*>(a.norm_w + 4 * cg);
    __syncthreads();

    bool in_flight = u < total;
    for (int i = 0; u < total; u += gridDim.x, ++i) {
        const float alpha = expf(g_next);
        const float beta = b_next;
        const int64_t un = u + gridDim.x;
        if (un < total) {
            g_next = a.g[un];
            b_next = a.beta[un];
        }
        {
            const bool ok = tid != 0 || wait_slot(full, i & 1, a.wait_ns);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) set_status(a.status, kStatusTimeout);
                break;
            }
        }
        // conv update + SiLU of q, k, v into fp32 shared memory; item j < dk
        // makes q_j and k_j and sums their squares and product
        float sq = 0.f, sk = 0.f, kq = 0.f;
        {
            const int n = (int)(u / H), h = (int)(u % H);
            const int64_t C = 2 * (int64_t)H * dk + (int64_t)H * dv;
            T* cs = static_cast<T*>(a.conv_state) + n * C * (K - 1);
            for (int j = tid; j < dk + dv; j += kThreads) {
                if (j < dk) {
                    const float qv = conv_channel(cx, cw, ccs, cs, j, (int64_t)h * dk + j, K);
                    const float kv = conv_channel(cx, cw, ccs, cs, dk + j, (int64_t)H * dk + h * dk + j, K);
                    qs[j] = qv;
                    ks[j] = kv;
                    sq = fmaf(qv, qv, sq);
                    sk = fmaf(kv, kv, sk);
                    kq = fmaf(qv, kv, kq);
                } else {
                    const int c = j - dk;
                    vs[c] = conv_channel(cx, cw, ccs, cs, 2 * dk + c, 2 * (int64_t)H * dk + h * dv + c, K);
                }
            }
        }
        sq = warp_sum(sq);
        sk = warp_sum(sk);
        kq = warp_sum(kq);
        if (lane == 0) part[warp] = make_float4(sq, sk, kq, 0.f);
        // this thread's state rows and gate
        float4 st[RPT];
        if (tid < nthr) {
#pragma unroll
            for (int r = 0; r < RPT; ++r)
                st[r] = *reinterpret_cast<const float4*>(Ss + (rg * RPT + r) * dv + 4 * cg);
        }
        float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.z && tid < cols4) z4 = load4(reinterpret_cast<const T*>(sl + geo.z_off) + 4 * cg);
        __syncthreads();  // the slot is read; q, k, v and the norm partials are in
        if (tid == 0) {
            in_flight = un < total;
            if (in_flight) {
                fence_proxy_async();  // the slot's reads come before the copy's writes
                load_unit<T>(a, geo, sl, un, full);
            }
        }
        float4 nrm = part[0];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            const float4 p = part[w];
            nrm.x += p.x;
            nrm.y += p.y;
            nrm.z += p.z;
        }
        float inv_q = 1.f, inv_k = 1.f;
        if (a.qk_l2norm) {
            inv_q = 1.f / sqrtf(nrm.x + a.eps);
            inv_k = 1.f / sqrtf(nrm.y + a.eps);
        }
        const float qsc = inv_q * a.scale;
        const float kqs = nrm.z * inv_k * qsc;
        // partial S^T k and S^T q over this thread's rows (raw q, k)
        if (tid < nthr) {
            float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float kv = ks[rg * RPT + r], qv = qs[rg * RPT + r];
                pa.x = fmaf(st[r].x, kv, pa.x); pa.y = fmaf(st[r].y, kv, pa.y);
                pa.z = fmaf(st[r].z, kv, pa.z); pa.w = fmaf(st[r].w, kv, pa.w);
                pb.x = fmaf(st[r].x, qv, pb.x); pb.y = fmaf(st[r].y, qv, pb.y);
                pb.z = fmaf(st[r].z, qv, pb.z); pb.w = fmaf(st[r].w, qv, pb.w);
            }
            *reinterpret_cast<float4*>(red + rg * dv + 4 * cg) = pa;
            *reinterpret_cast<float4*>(red + (RG + rg) * dv + 4 * cg) = pb;
        }
        __syncthreads();
        if (tid < nthr) {
            float4 A = make_float4(0.f, 0.f, 0.f, 0.f), Bq = A;
            for (int r = 0; r < RG; ++r) {
                const float4 x = *reinterpret_cast<const float4*>(red + r * dv + 4 * cg);
                const float4 y = *reinterpret_cast<const float4*>(red + (RG + r) * dv + 4 * cg);
                A.x += x.x; A.y += x.y; A.z += x.z; A.w += x.w;
                Bq.x += y.x; Bq.y += y.y; Bq.z += y.z; Bq.w += y.w;
            }
            const float4 v4 = *reinterpret_cast<const float4*>(vs + 4 * cg);
            const float mk = a.undecayed ? inv_k : alpha * inv_k;
            float4 d;
            d.x = beta * (v4.x - mk * A.x);
            d.y = beta * (v4.y - mk * A.y);
            d.z = beta * (v4.z - mk * A.z);
            d.w = beta * (v4.w - mk * A.w);
            if (tid < 32) {  // the output: the rg == 0 threads, all in warp 0
                float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                if (rg == 0) {
                    o.x = alpha * qsc * Bq.x + kqs * d.x;
                    o.y = alpha * qsc * Bq.y + kqs * d.y;
                    o.z = alpha * qsc * Bq.z + kqs * d.z;
                    o.w = alpha * qsc * Bq.w + kqs * d.w;
                }
                if (a.z) {  // gated RMSNorm over this head's dv outputs
                    float ss = o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
                    ss = warp_sum(ss);
                    const float inv = 1.f / sqrtf(ss / (float)dv + a.norm_eps);
                    o.x = o.x * inv * nw4.x * silu_s(z4.x);
                    o.y = o.y * inv * nw4.y * silu_s(z4.y);
                    o.z = o.z * inv * nw4.z * silu_s(z4.z);
                    o.w = o.w * inv * nw4.w * silu_s(z4.w);
                }
                if (rg == 0) store4(static_cast<T*>(a.o) + u * dv + 4 * cg, o);
            }
            float* Sg = a.state + u * dk * dv;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float kn = ks[rg * RPT + r] * inv_k;
                float4 x = st[r];
                x.x = fmaf(alpha, x.x, kn * d.x);
                x.y = fmaf(alpha, x.y, kn * d.y);
                x.z = fmaf(alpha, x.z, kn * d.z);
                x.w = fmaf(alpha, x.w, kn * d.w);
                __stcs(reinterpret_cast<float4*>(Sg + (int64_t)(rg * RPT + r) * dv + 4 * cg), x);
            }
        }
    }
    // after a timeout the copy being waited on may still land: let it
    if (tid == 0 && in_flight) {
        const int64_t done = (u - blockIdx.x) / gridDim.x;  // units this CTA finished
        mbar_wait(full, (uint32_t)(done & 1), kDrainNs);
    }
}

template <typename T, int RPT>
cudaError_t launch_rpt(const DecodeArgs& a, cudaStream_t s) {
    const Geometry geo = geometry(a, RPT);
    auto kernel = decode_layer_stream_kernel<T, RPT>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)geo.smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t units = (int64_t)a.N * a.H;
    const int64_t slots = (int64_t)kCtasPerSm * sms;
    kernel<<<(unsigned)(units < slots ? units : slots), kThreads, geo.smem, s>>>(a, geo);
    return cudaGetLastError();
}

int stream_rpt(const DecodeArgs& a) {
    // rows per thread: the smallest power of two that spreads the state's
    // float4 columns over the threads
    const int need = (a.dk * (a.dv / 4) + kThreads - 1) / kThreads;
    int rpt = 1;
    while (rpt < need) rpt <<= 1;
    return rpt;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool decode_stream_supported(const DecodeArgs& a) {
    // the whole-mixer step with ungrouped heads; the state rows of a thread
    // fit its registers; every bulk copy starts on a 16-byte boundary and
    // moves a multiple of 16 bytes; two CTAs fit in an SM's shared memory
    if (!a.x || a.H != a.Hk || a.dv % 4 != 0 || a.dv > 128 || a.dk % 16 != 0 || a.dk > 128) return false;
    const int esz = a.is_bf16 ? 2 : 4;
    if ((a.dk * esz) % 16 != 0 || (a.dv * esz) % 16 != 0) return false;
    const int rpt = stream_rpt(a);
    if (rpt > 16 || a.dk % rpt != 0 || (a.dk / rpt) * (a.dv / 4) < 32) return false;
    if (!a16(a.state) || (a.z && !a16(a.z))) return false;
    if (a.K < 1 || a.K > 4 || !a16(a.x) || !a16(a.conv_w) || (a.K > 1 && !a16(a.conv_state))) return false;
    return geometry(a, rpt).smem <= 113u * 1024u;
}

cudaError_t launch_decode_stream(const DecodeArgs& a, cudaStream_t s) {
    switch (stream_rpt(a)) {
        case 1: return a.is_bf16 ? launch_rpt<uint16_t, 1>(a, s) : launch_rpt<float, 1>(a, s);
        case 2: return a.is_bf16 ? launch_rpt<uint16_t, 2>(a, s) : launch_rpt<float, 2>(a, s);
        case 4: return a.is_bf16 ? launch_rpt<uint16_t, 4>(a, s) : launch_rpt<float, 4>(a, s);
        case 8: return a.is_bf16 ? launch_rpt<uint16_t, 8>(a, s) : launch_rpt<float, 8>(a, s);
        default: return a.is_bf16 ? launch_rpt<uint16_t, 16>(a, s) : launch_rpt<float, 16>(a, s);
    }
}

}  // namespace gdn
