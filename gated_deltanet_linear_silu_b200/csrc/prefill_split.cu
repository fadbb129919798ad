// Sequence-split prefill for launches with few (sequence, head) units.
//
// The recurrence is linear in the state: over a segment of a sequence,
//   S_end = Phi S_start + L,
// where Phi [dk, dk] is the product of the tokens' alpha_t (I - beta_t k^_t k^_t^T)
// ("Qwen3.5-MoE source walkthrough", 4.3: decay, then the delta-rule
// correction) and L is the segment's final state from a zero start. With
// dk == dv the tensor-core prefill gives both from two runs over the segment:
// a zero initial state yields L, and the identity as initial state with all
// values v = 0 yields Phi. So when N * H units leave most SMs idle, each
// sequence is cut into S chunk-aligned segments and
//   pass 1a: every segment from a zero state (segment 0 from the caller's h0),
//            final states -> L (segment 0's is the true state at segment 1);
//   pass 1b: every segment from the identity with v = 0, final states -> Phi;
//   combine: S_start(k+1) = Phi_k S_start(k) + L_k, k = 1 .. S-2, in fp32;
//   pass 2:  every segment from its true start state, writing o; the last
//            segment's final state is the sequence's hT.
// The three passes are the ordinary prefill kernel over the segments as
// sequences, each with S times the units of the plain launch; passes 1a and
// 1b write o too, and pass 2 overwrites it. Outputs of pass 2 differ from the
// plain launch only by rounding.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kMaxSegments = 16;
constexpr int kMinSegmentChunks = 4;  // average 64-token chunks per segment
// Fewest segments worth the three passes: each pass has a fixed cost of about
// four chunks' time (pipeline fill, state load and store), so 4 segments of
// 16 chunks measured no faster than the plain launch, 9 segments 1.2x faster
// and 16 segments about 1.9x faster.
constexpr int kMinSegments = 6;
constexpr int kSplitD = 128;          // dk = dv of the tensor-core prefill
constexpr int64_t kStateFloats = (int64_t)kSplitD * kSplitD;

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

struct SplitLayout {
    WorkspaceLayout base;  // schedule of the N * S segment sequences
    size_t cu_off, a_off, b_off, l_off, r_off, zv_off, total;
};

SplitLayout split_layout(int N, int64_t T_tot, int H, int S) {
    SplitLayout l;
    const int64_t NS = (int64_t)N * S;
    l.base = prefill_workspace_layout((int)NS);
    l.cu_off = round256(l.base.total);
    const size_t states = (size_t)NS * H * kStateFloats * sizeof(float);
    l.a_off = round256(l.cu_off + sizeof(int32_t) * (size_t)(NS + 1));
    l.b_off = l.a_off + states;
    l.l_off = l.b_off + states;
    l.r_off = l.l_off + states;
    l.zv_off = l.r_off + states;  // bf16 zeros standing in for v in pass 1b
    l.total = l.zv_off + round256((size_t)T_tot * H * kSplitD * 2);
    return l;
}

// One launch prepares the three passes (grid-stride over all of it):
//  - segment bounds: sequence n = [st, en) of c = ceil(len / 64) chunks gives
//    segment k = [st + 64 floor(k c / S), st + 64 floor((k+1) c / S)) clipped
//    to en (empty segments when c < S); a sequence with bad bounds gets empty
//    segments and keeps its bad end, so the prefill flags it;
//  - A (pass 1a and pass 2 initial states): segment 0 <- h0 (zeros if none),
//    the rest zeros; B (pass 1b initial states): the identity;
//  - the bf16 zero values of pass 1b.
__global__ void split_init_kernel(const int32_t* cu, const float* h0, int N, int H, int S, int32_t* cu_seg,
                                  float* A, float* B, uint4* zeros_v, int64_t n_zero16) {
    pdl_launch_dependents();
    pdl_wait_previous();
    const int64_t NS = (int64_t)N * S;
    const int64_t n4 = NS * H * kStateFloats / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t idx = i0; idx <= NS; idx += stride) {
        if (idx == NS) {
            cu_seg[idx] = cu[N];
            continue;
        }
        const int n = (int)(idx / S), k = (int)(idx % S);
        const int64_t st = cu[n], en = cu[n + 1];
        const int64_t len = en > st ? en - st : 0;
        const int64_t c = (len + 63) / 64;
        const int64_t off = 64 * ((k * c) / S);
        cu_seg[idx] = (int32_t)(st + (off < len ? off : len));
    }
    for (int64_t e4 = i0; e4 < n4; e4 += stride) {
        const int64_t e = 4 * e4;
        const int64_t blk = e / kStateFloats, within = e % kStateFloats;
        const int h = (int)(blk % H);
        const int k = (int)((blk / H) % S);
        const int64_t n = blk / ((int64_t)H * S);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k == 0 && h0) x = *reinterpret_cast<const float4*>(h0 + (n * H + h) * kStateFloats + within);
        reinterpret_cast<float4*>(A)[e4] = x;
        const int row = (int)(within / kSplitD), col = (int)(within % kSplitD);  // col % 4 == 0
        const float4 id = make_float4(row == col ? 1.f : 0.f, row == col + 1 ? 1.f : 0.f,
                                      row == col + 2 ? 1.f : 0.f, row == col + 3 ? 1.f : 0.f);
        reinterpret_cast<float4*>(B)[e4] = id;
    }
    for (int64_t z = i0; z < n_zero16; z += stride) zeros_v[z] = make_uint4(0u, 0u, 0u, 0u);
}

// The chain of segment start states, per (sequence, head) and block of 16
// state columns (columns evolve independently: Phi acts on the rows), one CTA
// each (N * H * 8 CTAs: one wave when the split applies). Each step is a
// 128 x 128 by 128 x 16 product on the tensor cores (mma.sync m16n8k8 tf32) in
// split precision: x = hi + lo with hi = tf32(x), and hi*hi + hi*lo + lo*hi
// keeps about fp32 accuracy. Warp w owns rows [16w, 16w + 16) of the block.
// Phi_k is staged in shared memory (rows padded to 132 floats, so the A
// fragments of a warp hit 32 distinct banks), the next one prefetched with
// cp.async while step k runs; the current start state's block sits in shared
// memory with rows padded to 24 floats (conflict-free B fragments).
constexpr int kCombCols = 16;
constexpr int kCombThreads = 256;
constexpr int kPhiLd = 132;
constexpr int kCurLd = 24;
constexpr size_t kCombSmem = sizeof(float) * (2 * kSplitD * kPhiLd + kSplitD * kCurLd);

__device__ __forceinline__ void stage_phi(float* dst, const float* src) {
    for (int p = threadIdx.x; p < kSplitD * kSplitD / 4; p += kCombThreads) {
        const int r = p / (kSplitD / 4), c4 = p % (kSplitD / 4);
        cp_async_16(dst + r * kPhiLd + 4 * c4, src + (int64_t)r * kSplitD + 4 * c4);
    }
    cp_async_commit_group();
}

__device__ __forceinline__ uint32_t tf32_hi(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kCombThreads) split_combine_kernel(int N, int H, int S, const float* Lst,
                                                                    const float* Phi, float* A) {
    extern __shared__ float4 comb_smem4[];
    pdl_launch_dependents();
    pdl_wait_previous();
    float* phi_s = reinterpret_cast<float*>(comb_smem4);  // [2][128][kPhiLd]
    float* cur = phi_s + 2 * kSplitD * kPhiLd;             // [128][kCurLd]
    const int nh = blockIdx.x;                             // n * H + h
    const int n = nh / H, h = nh % H;
    const int cb = blockIdx.y * kCombCols;                 // first state column of the block
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int r0 = 16 * warp;
    const int64_t off0 = ((int64_t)n * S * H + h) * kStateFloats;  // segment 0 of (n, h)
    const int64_t seg = (int64_t)H * kStateFloats;                  // between segments
    if (S > 2) stage_phi(phi_s, Phi + off0 + seg);
    // S_start(1) = L_0 (segment 0 ran from the true initial state)
    for (int e = threadIdx.x; e < kSplitD * kCombCols / 4; e += kCombThreads) {
        const int row = e / (kCombCols / 4), c4 = e % (kCombCols / 4);
        const float4 x = *reinterpret_cast<const float4*>(Lst + off0 + (int64_t)row * kSplitD + cb + 4 * c4);
        *reinterpret_cast<float4*>(cur + row * kCurLd + 4 * c4) = x;
        *reinterpret_cast<float4*>(A + off0 + seg + (int64_t)row * kSplitD + cb + 4 * c4) = x;
    }
    for (int k = 1; k + 1 < S; ++k) {
        // accumulators start from L_k at the fragment positions: rows r0 + g (+8),
        // columns 8 nt + 2 t (+1) of the block
        float acc[2][4];
        const float* lk = Lst + off0 + k * seg + cb;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float2 x0 = *reinterpret_cast<const float2*>(lk + (int64_t)(r0 + g) * kSplitD + 8 * nt + 2 * t);
            const float2 x1 = *reinterpret_cast<const float2*>(lk + (int64_t)(r0 + g + 8) * kSplitD + 8 * nt + 2 * t);
            acc[nt][0] = x0.x; acc[nt][1] = x0.y; acc[nt][2] = x1.x; acc[nt][3] = x1.y;
        }
        if (k + 2 < S) {
            // buffer (k & 1) was last read in step k - 1, which ended with a barrier
            stage_phi(phi_s + (k & 1) * kSplitD * kPhiLd, Phi + off0 + (k + 1) * seg);
            cp_async_wait_group1();  // Phi_k is in; Phi_{k+1} may still be in flight
        } else {
            cp_async_wait_all_groups();
        }
        __syncthreads();  // Phi_k and cur visible to every thread
        const float* pk = phi_s + ((k - 1) & 1) * kSplitD * kPhiLd;
#pragma unroll 4
        for (int kk = 0; kk < kSplitD / 8; ++kk) {
            const float af[4] = {pk[(r0 + g) * kPhiLd + 8 * kk + t], pk[(r0 + g + 8) * kPhiLd + 8 * kk + t],
                                 pk[(r0 + g) * kPhiLd + 8 * kk + t + 4], pk[(r0 + g + 8) * kPhiLd + 8 * kk + t + 4]};
            uint32_t ahi[4], alo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                ahi[q] = tf32_hi(af[q]);
                alo[q] = tf32_hi(af[q] - __uint_as_float(ahi[q]));
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float b0 = cur[(8 * kk + t) * kCurLd + 8 * nt + g];
                const float b1 = cur[(8 * kk + t + 4) * kCurLd + 8 * nt + g];
                const uint32_t bh0 = tf32_hi(b0), bh1 = tf32_hi(b1);
                const uint32_t bl0 = tf32_hi(b0 - __uint_as_float(bh0)), bl1 = tf32_hi(b1 - __uint_as_float(bh1));
                mma_16x8x8_tf32(acc[nt], alo, bh0, bh1);
                mma_16x8x8_tf32(acc[nt], ahi, bl0, bl1);
                mma_16x8x8_tf32(acc[nt], ahi, bh0, bh1);
            }
        }
        __syncthreads();  // every thread has read cur and Phi_k
        float* an = A + off0 + (k + 1) * seg + cb;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float2 y0 = make_float2(acc[nt][0], acc[nt][1]), y1 = make_float2(acc[nt][2], acc[nt][3]);
            *reinterpret_cast<float2*>(cur + (r0 + g) * kCurLd + 8 * nt + 2 * t) = y0;
            *reinterpret_cast<float2*>(cur + (r0 + g + 8) * kCurLd + 8 * nt + 2 * t) = y1;
            *reinterpret_cast<float2*>(an + (int64_t)(r0 + g) * kSplitD + 8 * nt + 2 * t) = y0;
            *reinterpret_cast<float2*>(an + (int64_t)(r0 + g + 8) * kSplitD + 8 * nt + 2 * t) = y1;
        }
    }
}

// hT[n] <- the final state of sequence n's last segment (pass 2's output).
__global__ void split_final_kernel(const float* B, int N, int H, int S, float* hT) {
    pdl_wait_previous();
    const int64_t n4 = (int64_t)N * H * kStateFloats / 4;
    for (int64_t e4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e4 < n4;
         e4 += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = 4 * e4;
        const int64_t nh = e / kStateFloats, within = e % kStateFloats;
        const int64_t n = nh / H, h = nh % H;
        reinterpret_cast<float4*>(hT)[e4] =
            *reinterpret_cast<const float4*>(B + ((n * S + S - 1) * H + h) * kStateFloats + within);
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

int prefill_split_segments(int N, int64_t T_tot, int H, int dk, int dv, int chunk) {
    if (N <= 0 || T_tot <= 0 || dk != kSplitD || dv != kSplitD || chunk != 64) return 1;
    const int64_t units = (int64_t)N * H;
    int64_t S = sm_count() / units;  // segments per sequence that still fit one wave
    const int64_t by_len = T_tot / N / 64 / kMinSegmentChunks;
    if (by_len < S) S = by_len;
    if (S > kMaxSegments) S = kMaxSegments;
    return S >= kMinSegments ? (int)S : 1;
}

size_t prefill_split_workspace_bytes(int N, int64_t T_tot, int H, int S) {
    return split_layout(N, T_tot, H, S).total;
}

cudaError_t launch_prefill_split(const PrefillArgs& a, int S, void* workspace, cudaStream_t s) {
    const SplitLayout l = split_layout(a.N, a.T_tot, a.H, S);
    char* ws = static_cast<char*>(workspace);
    int32_t* cu_seg = reinterpret_cast<int32_t*>(ws + l.cu_off);
    float* A = reinterpret_cast<float*>(ws + l.a_off);
    float* B = reinterpret_cast<float*>(ws + l.b_off);
    float* Lst = reinterpret_cast<float*>(ws + l.l_off);
    float* Phi = reinterpret_cast<float*>(ws + l.r_off);
    void* zeros_v = ws + l.zv_off;
    const int NS = a.N * S;
    const int fill_blocks = 4 * sm_count();

    cudaError_t e = launch_pdl(split_init_kernel, dim3(fill_blocks), dim3(256), 0, s, a.cu, a.h0, a.N, a.H, S,
                               cu_seg, A, B, static_cast<uint4*>(zeros_v),
                               (int64_t)a.T_tot * a.H * kSplitD * 2 / 16);
    if (e != cudaSuccess) return e;

    // One schedule of the N S segments serves the three passes, each with its
    // own work counter.
    PrefillArgs p = a;
    p.cu = cu_seg;
    p.N = NS;
    p.conv_seg = S;  // fused conv: segment n of the split belongs to sequence n / S (a.cu's)
    p.order = reinterpret_cast<int32_t*>(ws + l.base.order_off);
    int32_t* counters = reinterpret_cast<int32_t*>(ws + l.base.counter_off);
    p.counter = counters;
    if ((e = launch_prefill_schedule(p, s, 3, true)) != cudaSuccess) return e;
    auto pass = [&](int which, const float* h0, float* hT) {
        p.h0 = h0;
        p.hT = hT;
        p.counter = counters + 2 * which;
        return launch_prefill_tc(p, s, true);
    };
    if ((e = pass(0, a.h0 ? A : nullptr, Lst)) != cudaSuccess) return e;  // 1a
    p.v = zeros_v;
    p.ld_v = (int64_t)a.H * kSplitD;
    p.conv_v = 0;  // fused conv: the zero values are used as loaded
    e = pass(1, B, Phi);  // 1b
    p.v = a.v;
    p.ld_v = a.ld_v;
    p.conv_v = a.conv_v;
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(split_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kCombSmem)) != cudaSuccess)
        return e;
    e = launch_pdl(split_combine_kernel, dim3((unsigned)(a.N * a.H), kSplitD / kCombCols), dim3(kCombThreads),
                   kCombSmem, s, a.N, a.H, S, static_cast<const float*>(Lst), static_cast<const float*>(Phi), A);
    if (e != cudaSuccess) return e;
    if ((e = pass(2, A, a.hT ? B : nullptr)) != cudaSuccess) return e;  // 2
    if (a.hT) {
        e = launch_pdl(split_final_kernel, dim3(fill_blocks), dim3(256), 0, s, static_cast<const float*>(B), a.N,
                       a.H, S, a.hT);
    }
    return e;
}

}  // namespace gdn
