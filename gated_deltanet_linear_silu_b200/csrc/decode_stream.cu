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
// With grouped value heads (H = G Hk, value head h reading q, k head h / G)
// a CTA takes whole groups: the G units of (sequence, q/k head) run back to
// back, the first one computes the shared q, k channels' conv (and shifts
// their conv state: this CTA is the only reader), the others reuse q, k and
// their norms from shared memory and bring in only their own v channels.
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

// Issue the bulk copies of unit u (value head h of sequence n) into the slot
// (one thread): the state, the v channels' conv inputs, z, and with `qk` also
// the conv inputs of the q, k channels of the head's q/k group.
template <typename T>
__device__ __forceinline__ void load_unit(const DecodeArgs& a, const Geometry& geo, uint8_t* sl, int u, bool qk,
                                          uint64_t* full) {
    const int dk = a.dk, dv = a.dv, H = a.H, Hk = a.Hk, K = a.K;
    const int nconv = 2 * dk + dv;
    const int esz = (int)sizeof(T);
    const uint32_t v_bytes = (uint32_t)(dv * 2 * K * esz), qk_bytes = (uint32_t)(2 * dk * 2 * K * esz);
    mbar_arrive_expect_tx(full, geo.state_bytes + v_bytes + (qk ? qk_bytes : 0u) + (a.z ? dv * esz : 0));
    bulk_load(sl, a.state + (int64_t)u * dk * dv, geo.state_bytes, full);
    const int n = u / H, h = u % H, hk = h / (H / Hk);
    const int64_t C = 2 * (int64_t)Hk * dk + (int64_t)H * dv;
    const T* x = static_cast<const T*>(a.x) + n * C;
    const T* w = static_cast<const T*>(a.conv_w);
    const T* cs = static_cast<const T*>(a.conv_state) + n * C * (K - 1);
    T* cx = reinterpret_cast<T*>(sl + geo.state_bytes);
    T* cw = cx + nconv;
    T* ccs = cw + nconv * K;
#pragma unroll
    for (int b = qk ? 0 : 2; b < 3; ++b) {  // q, k, v channel blocks
        const int nb = b < 2 ? dk : dv;
        const int64_t ch0 = b == 0 ? (int64_t)hk * dk : (b == 1 ? (int64_t)Hk * dk + hk * dk : 2 * (int64_t)Hk * dk + h * dv);
        const int c0 = b == 0 ? 0 : (b == 1 ? dk : 2 * dk);
        bulk_load(cx + c0, x + ch0, nb * esz, full);
        bulk_load(cw + c0 * K, w + ch0 * K, nb * K * esz, full);
        if (K > 1) bulk_load(ccs + c0 * (K - 1), cs + ch0 * (K - 1), nb * (K - 1) * esz, full);
    }
    if (a.z) bulk_load(sl + geo.z_off, static_cast<const T*>(a.z) + (int64_t)u * dv, dv * esz, full);
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
    const int H = a.H, Hk = a.Hk, G = H / Hk, K = a.K;
    // units u = n H + h (N H < 2^31) in group order: the CTA takes groups
    // blockIdx.x, blockIdx.x + gridDim.x, ... (a group is (sequence, q/k head),
    // its G value heads are units group G + g, g = 0 .. G-1); -1 past the last
    const int total = a.N * H;
    const int skip = (int)(gridDim.x - 1) * G;  // from a group's last unit to the next group's first

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

    int u = (int)blockIdx.x * G < total ? (int)blockIdx.x * G : -1;
    int gpos = 0;  // u's position in its group
    pdl_launch_dependents();  // the next step may start launching
    if (tid == 0) {
        mbar_init(full, 1);
        fence_mbar_init();
    }
    pdl_wait_previous();  // the previous step's states and conv states are written
    if (tid == 0 && u >= 0) load_unit<T>(a, geo, sl, u, true, full);
    float g_next = 0.f, b_next = 0.f;  // gate and beta one unit ahead
    if (u >= 0) {
        g_next = a.g[u];
        b_next = a.beta[u];
    }
    float4 nw4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.z && tid < cols4) nw4 = *reinterpret_cast<const float4*>(a.norm_w + 4 * cg);
    __syncthreads();

    bool in_flight = u >= 0;
    int i = 0;
    for (; u >= 0; ++i) {
        const float alpha = expf(g_next);
        const float beta = b_next;
        const bool first = gpos == 0;  // the group's first unit: q, k conv
        const int gpos_n = gpos + 1 == G ? 0 : gpos + 1;
        const int64_t un64 = (int64_t)u + 1 + (gpos_n == 0 ? skip : 0);
        const int un = un64 < total ? (int)un64 : -1;
        if (un >= 0) {
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
        // conv update + SiLU into fp32 shared memory: the v channels, and in the
        // group's first unit the q, k channels too (item j < dk makes q_j and k_j
        // and sums their squares and product); later units of the group keep
        // q, k and the norm partials
        {
            const int n = u / H, h = u % H, hk = h / G;
            const int64_t C = 2 * (int64_t)Hk * dk + (int64_t)H * dv;
            T* cs = static_cast<T*>(a.conv_state) + n * C * (K - 1);
            const int j0 = first ? 0 : dk;
            float sq = 0.f, sk = 0.f, kq = 0.f;
            for (int j = j0 + tid; j < dk + dv; j += kThreads) {
                if (j < dk) {
                    const float qv = conv_channel(cx, cw, ccs, cs, j, (int64_t)hk * dk + j, K);
                    const float kv = conv_channel(cx, cw, ccs, cs, dk + j, (int64_t)Hk * dk + hk * dk + j, K);
                    qs[j] = qv;
                    ks[j] = kv;
                    sq = fmaf(qv, qv, sq);
                    sk = fmaf(kv, kv, sk);
                    kq = fmaf(qv, kv, kq);
                } else {
                    const int c = j - dk;
                    vs[c] = conv_channel(cx, cw, ccs, cs, 2 * dk + c, 2 * (int64_t)Hk * dk + h * dv + c, K);
                }
            }
            if (first) {
                sq = warp_sum(sq);
                sk = warp_sum(sk);
                kq = warp_sum(kq);
                if (lane == 0) part[warp] = make_float4(sq, sk, kq, 0.f);
            }
        }
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
            in_flight = un >= 0;
            if (in_flight) {
                fence_proxy_async();  // the slot's reads come before the copy's writes
                load_unit<T>(a, geo, sl, un, gpos_n == 0, full);
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
                if (rg == 0) store4(static_cast<T*>(a.o) + (int64_t)u * dv + 4 * cg, o);
            }
            float* Sg = a.state + (int64_t)u * dk * dv;
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
        u = un;
        gpos = gpos_n;
    }
    // after a timeout the copy being waited on (the i-th) may still land: let it
    if (tid == 0 && in_flight) mbar_wait(full, (uint32_t)(i & 1), kDrainNs);
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
    const int64_t groups = (int64_t)a.N * a.Hk;  // a CTA takes whole q/k groups
    const int64_t slots = (int64_t)kCtasPerSm * sms;
    return launch_pdl(kernel, dim3((unsigned)(groups < slots ? groups : slots)), dim3(kThreads), geo.smem, s, a,
                      geo);
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
    // the whole-mixer step (any q/k grouping); the state rows of a thread
    // fit its registers; every bulk copy starts on a 16-byte boundary and
    // moves a multiple of 16 bytes; two CTAs fit in an SM's shared memory
    if (!a.x || a.Hk <= 0 || a.H % a.Hk != 0 || a.dv % 4 != 0 || a.dv > 128 || a.dk % 16 != 0 || a.dk > 128) return false;
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
