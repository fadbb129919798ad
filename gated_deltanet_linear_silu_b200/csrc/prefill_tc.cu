// Chunked gated delta rule on the 5th-generation tensor cores (tcgen05):
// bf16 q/k/v, d_k = d_v = 128, chunk C = 64, fp32 state and accumulation.
//
// The recurrence is the decay-first rule of "Qwen3.5-MoE source walkthrough",
// 4.3; the chunk algebra (cumulative decay gamma, UT transform with a unit
// lower-triangular solve, inter-chunk state passing) is that of
// "Parallelizing Linear Transformers with the Delta Rule over Sequence Length"
// (Yang et al., 2024) with the gating of "Gated Delta Networks" (Yang, Kautz,
// Hatamizadeh, 2024). Per chunk (rows r = tokens, S = state [dk, dv]):
//   P = (Q^ K^^T) o M,  A = strict_tril(diag(beta) (K^ K^^T) o M),  T = (I+A)^-1
//   W = T diag(beta e^gamma) K^,   U~ = T diag(beta) V,   U = U~ - W S
//   O = diag(e^gamma) Q^ S + P U,  S <- e^{gamma_L} S + (diag(e^{gamma_L-gamma}) K^)^T U
// with M[r][j] = e^{gamma_r - gamma_j} for j <= r and ^ the per-row L2 norm.
//
// B200 mapping. Every contraction is issued as an M = 128 tcgen05.mma by
// computing the transposed products, so the 128-wide head dimension is the
// MMA's M and no tile is padded:
//   [Q;K][Q;K]^T       -> TMEM  R_A   (128 lanes = 64 q rows + 64 k rows)
//   W^T  = K^T T1^T    -> TMEM  R_W   (lanes = dk, cols = tokens)
//   U~^T = V^T T2^T    -> TMEM  R_U   (lanes = dv, cols = tokens)
//   U^T  = U~^T + S^T (-W^T)         (accumulated in R_U)
//   O^T  = S^T Q~^T + U^T P^T        (R_O, lanes = dv, cols = tokens)
//   S^T <- e^{gamma_L} S^T + U^T K~  (R_S, fp32 master state, lanes = dv, cols = dk)
// The algorithmic 11.5 MFLOP per (chunk, head) are the MMAs issued, plus the
// q-by-q block of the Gram matrix, whose diagonal gives the q norms.
// The L2 norms, scale and decays are applied as per-row factors in the
// epilogues, so the MMAs read the raw bf16 input tiles that TMA brings in
// (128-byte swizzle). The state chain's A operands, S^T and U^T, never touch
// shared memory: the epilogues write them back to TMEM as packed bf16 and the
// MMAs read A from there, so those MMAs stream only B from shared memory. The
// solve for T runs on CUDA cores in fp32 (with tf32 tensor-core merges).
//
// Warp specialisation (one CTA of 12 warps per SM, persistent over units):
//   warps 0-7   prep group: everything that does not depend on the state --
//               gates, norms, [Q;K]K^T, P, A, the triangular solve, W^T, U~^T,
//               Q~ and K~ -- for chunk c+1 ...
//   warps 8-11  state group: ... while these run the state chain of chunk c
//               (U, the state update, O) with the state resident in TMEM. When
//               the state group is done with a stage of the two-stage ring one
//               of its lanes refills it by TMA with the chunk two ahead.
// The prep group's second warp turns a chunk's gates into beta and the cumulative
// decay gamma while the Gram MMA runs and signals the state group, which needs
// only gamma_L (to pre-decay its state for the coming chunk).
// The groups hand off through mbarriers; TMEM holds double-buffered U~/U
// and O regions so the prep of c+1 never waits for the epilogues of c.
// Every wait is bounded: on timeout the kernel records the timeout status,
// all groups leave their loops, MMAs and TMA copies are drained (bounded),
// TMEM is freed and the kernel returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int kC = 64;          // chunk
constexpr int kD = 128;         // head dim (dk = dv)
constexpr int kPrepThreads = 256;
constexpr int kStateThreads = 128;
constexpr int kThreads = kPrepThreads + kStateThreads;
constexpr int kStateWarp0 = kPrepThreads / 32;               // 8
constexpr int kBarPrep = 1, kBarState = 2;                   // named barrier ids
constexpr uint64_t kWaitNs = kDefaultWaitNs;  // drains: a quarter of this

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t kBox = 8192;                   // 64 rows x 128 B (64 bf16)
constexpr uint32_t kQb0 = 0, kKb0 = kBox, kQb1 = 2 * kBox, kKb1 = 3 * kBox;
constexpr uint32_t kVb0 = 4 * kBox, kVb1 = 5 * kBox;
constexpr uint32_t kStageBytes = 6 * kBox;        // 48 KB: Q, K, V tiles (V later holds O)
constexpr uint32_t kOffVec = 2 * kStageBytes;     // per stage: g, beta, gamma, bet, rq, rk (6 x 64 fp32)
constexpr uint32_t kVecBytes = 2048;
constexpr uint32_t kOffWT = kOffVec + 2 * kVecBytes;  // -W^T bf16 [128 dk][64 tok] MN-major
constexpr uint32_t kOffO = kOffWT + 16384;        // O staging bf16, 2 x [64 tok][64 dv] row-major
constexpr uint32_t kOffP = kOffO + 16384;         // P bf16 [64 r][64 j] K-major, per stage
constexpr int kLdA = 68;                          // padded fp32 row stride (272 B)
constexpr uint32_t kOffA = kOffP + 2 * 8192;      // A fp32 [64][kLdA]; after the solve T1^T, T2^T
constexpr uint32_t kOffT1 = kOffA, kOffT2 = kOffA + 8192;
constexpr uint32_t kOffTf = kOffA + 64 * kLdA * 4;  // T fp32 [64][kLdA]
constexpr uint32_t kOffBar = kOffTf + 64 * kLdA * 4;  // mbarriers
constexpr uint32_t kOffMisc = kOffBar + 128;      // tmem base, abort flag, scan carry
constexpr uint32_t kSmemBytes = kOffMisc + 64;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kOffA % 1024 == 0 && kOffWT % 1024 == 0 && kOffP % 1024 == 0, "swizzle alignment");

// TMEM columns (fp32, 128 lanes).
constexpr uint32_t kTmemCols = 512;
// R_S: fp32 state S^T (128 columns). R_SB: S^T as packed bf16 (64 columns), the
// TMEM-resident A operand of MMA1. R_O: O^T of the chunk in flight (64).
// R_U: U~^T / U^T per stage (2 x 64); after the U epilogue its first 32 columns
// hold U^T as packed bf16, the A operand of MMA2. R_A holds the 128 x 128 Gram
// matrix [Q;K][Q;K]^T and is reused for W^T once the P/A epilogue has read it.
constexpr uint32_t kRS = 0, kRSB = 128, kRO = 192, kRU = 256, kRA = 384, kRW = 384;

constexpr uint32_t kIdescA = idesc_bf16(128, 128, 0, 0);   // [Q;K] [Q;K]^T (Gram)
constexpr uint32_t kIdescMN = idesc_bf16(128, 64, 1, 1);   // K^T T1^T, V^T T2^T
constexpr uint32_t kIdescSW = idesc_bf16(128, 64, 0, 1);   // S^T (-W^T)
constexpr uint32_t kIdescSQ = idesc_bf16(128, 64, 0, 0);   // S^T Q~^T, U^T P^T
constexpr uint32_t kIdescUK = idesc_bf16(128, 128, 0, 1);  // U^T K~

struct TcParams {
    PrefillArgs a;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// 2^x on the XU unit (PTX ex2.approx: relative error about 2^-22; 0 for very
// negative x).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 32 fp32 values (times f) as 16 packed bf16 pairs, even index in the low half.
__device__ __forceinline__ void pack_row32(const float (&v)[32], float f, uint32_t (&w)[16]) {
#pragma unroll
    for (int c = 0; c < 16; ++c) w[c] = pack_bf16(v[2 * c] * f, v[2 * c + 1] * f);
}
__device__ __forceinline__ void unpack_bf16(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

// Write 32 fp32 values (times f) as columns [32*half, 32*half + 32) of one
// 128-byte bf16 row of a swizzled tile.
__device__ __forceinline__ void store_half_row(uint8_t* tile, int row, int half, const float (&v)[32],
                                               float f) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = pack_bf16(v[8 * c + 0] * f, v[8 * c + 1] * f);
        u.y = pack_bf16(v[8 * c + 2] * f, v[8 * c + 3] * f);
        u.z = pack_bf16(v[8 * c + 4] * f, v[8 * c + 5] * f);
        u.w = pack_bf16(v[8 * c + 6] * f, v[8 * c + 7] * f);
        *reinterpret_cast<uint4*>(tile + sw128_off(row, 4 * half + c)) = u;
    }
}

// Scale the 128-byte row `row` of a swizzled bf16 tile in place.
__device__ __forceinline__ void scale_row(uint8_t* tile, int row, float f) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4* p = reinterpret_cast<uint4*>(tile + sw128_off(row, c));  // spreads banks
        uint4 u = *p;
        float a, b;
        unpack_bf16(u.x, a, b); u.x = pack_bf16(a * f, b * f);
        unpack_bf16(u.y, a, b); u.y = pack_bf16(a * f, b * f);
        unpack_bf16(u.z, a, b); u.z = pack_bf16(a * f, b * f);
        unpack_bf16(u.w, a, b); u.w = pack_bf16(a * f, b * f);
        *p = u;
    }
}

// Warp-level m16n8k8 TF32 tensor-core product (fp32 accumulate) used by the
// merges of the triangular solve: d(16x8) += A(16x8) * B(8x8), both read from
// fp32 shared memory (A row-major with stride lda, B row-major k x n with
// stride ldb) and rounded to tf32.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const float* A, int lda, const float* B,
                                                int ldb) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t a0 = to_tf32(A[g * lda + t]), a1 = to_tf32(A[(g + 8) * lda + t]);
    const uint32_t a2 = to_tf32(A[g * lda + t + 4]), a3 = to_tf32(A[(g + 8) * lda + t + 4]);
    const uint32_t b0 = to_tf32(B[t * ldb + g]), b1 = to_tf32(B[(t + 4) * ldb + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Store the 16x8 accumulator tile (times f) row-major with stride ld.
__device__ __forceinline__ void store_acc_16x8(float* D, int ld, const float (&d)[4], float f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2*>(D + g * ld + 2 * t) = make_float2(f * d[0], f * d[1]);
    *reinterpret_cast<float2*>(D + (g + 8) * ld + 2 * t) = make_float2(f * d[2], f * d[3]);
}

struct Unit {
    int n, h;
    int64_t start, end;
};

__device__ __forceinline__ bool load_unit(const PrefillArgs& a, int64_t u, Unit& U) {
    U.h = (int)(u % a.H);
    U.n = a.order[u / a.H];
    if (U.n < 0 || U.n >= a.N) return false;
    U.start = a.cu[U.n];
    U.end = a.cu[U.n + 1];
    return U.start >= 0 && U.start <= U.end && U.end <= a.T_tot;
}

// Next unit index >= u of this CTA's stride with at least one token (or total).
__device__ __forceinline__ int64_t next_nonempty(const PrefillArgs& a, int64_t u, int64_t total) {
    for (; u < total; u += gridDim.x) {
        Unit U;
        if (load_unit(a, u, U) && U.end > U.start) return u;
    }
    return total;
}

__device__ __forceinline__ void issue_tiles(uint8_t* stage, uint64_t* bar, const CUtensorMap* mq,
                                            const CUtensorMap* mk, const CUtensorMap* mv, int hk,
                                            int h, int64_t c0) {
    mbar_arrive_expect_tx(bar, kStageBytes);
    const int t = (int)c0;
    tma_load_3d(stage + kQb0, mq, bar, 0, hk, t);
    tma_load_3d(stage + kQb1, mq, bar, 64, hk, t);
    tma_load_3d(stage + kKb0, mk, bar, 0, hk, t);
    tma_load_3d(stage + kKb1, mk, bar, 64, hk, t);
    tma_load_3d(stage + kVb0, mv, bar, 0, h, t);
    tma_load_3d(stage + kVb1, mv, bar, 64, h, t);
}


// Named barrier over `count` threads (warp multiple) with an OR-reduction.
__device__ __forceinline__ bool group_any(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void group_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// The CTA's work list: chunks of its units (u = blockIdx.x + k * gridDim.x,
// non-empty ones), in order. Every group walks the same list.
struct Item {
    int64_t u;
    Unit U;
    int64_t c0;
    int L;
    bool first, last;
};

__device__ __forceinline__ bool item_first(const PrefillArgs& a, int64_t total, Item& it) {
    it.u = next_nonempty(a, blockIdx.x, total);
    if (it.u >= total) return false;
    load_unit(a, it.u, it.U);
    it.c0 = it.U.start;
    it.first = true;
    it.L = (int)((it.U.end - it.c0 < kC) ? it.U.end - it.c0 : kC);
    it.last = it.c0 + kC >= it.U.end;
    return true;
}

__device__ __forceinline__ bool item_next(const PrefillArgs& a, int64_t total, Item& it) {
    it.c0 += kC;
    it.first = false;
    if (it.c0 >= it.U.end) {
        it.u = next_nonempty(a, it.u + gridDim.x, total);
        if (it.u >= total) return false;
        load_unit(a, it.u, it.U);
        it.c0 = it.U.start;
        it.first = true;
    }
    it.L = (int)((it.U.end - it.c0 < kC) ? it.U.end - it.c0 : kC);
    it.last = it.c0 + kC >= it.U.end;
    return true;
}

// Bounded wait that also gives up once another group has aborted. limit 0:
// only a phase already complete at the first (non-blocking) probe passes.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort_flag, uint64_t limit) {
    if (limit == 0) return mbar_test_wait(bar, parity);
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit) return false;
    }
    return true;
}

struct Smem {
    uint8_t* base;
    __device__ uint8_t* stage(int s) const { return base + s * kStageBytes; }
    __device__ float* vec(int s) const { return reinterpret_cast<float*>(base + kOffVec + s * kVecBytes); }
    // vec layout: [0,64) e^{gmax - gamma}, [64] gmax, [65] factored-decay flag,
    // [128,192) gamma, [192,256) beta (written by the prep group's second warp),
    // [256,320) rq, [320,384) rk (written by the prep group)
};

// kUndecayed: each token reads the state before its own decay (row decay
// gamma_{r-1} in A and W). A template parameter, so the default order's code is
// not touched by the option.
template <bool kUndecayed>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ TcParams P, const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_o) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the shared-window address (swizzle atoms, TMA).
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Smem S{sm};
    const PrefillArgs& a = P.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int group = H / a.Hk;  // value heads per q, k head
    const int64_t total = (int64_t)a.N * H;

    uint8_t* sWT = sm + kOffWT;
    uint8_t* sO = sm + kOffO;
    uint8_t* sT1 = sm + kOffT1;
    uint8_t* sT2 = sm + kOffT2;
    float* sA = reinterpret_cast<float*>(sm + kOffA);
    float* sT = reinterpret_cast<float*>(sm + kOffTf);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
    uint64_t* full = bars + 0;      // [2] q/k/v tiles of a stage landed (TMA -> prep)
    uint64_t* gready = bars + 2;    // [2] gamma/beta of a stage written (prep -> state)
    uint64_t* pdone = bars + 4;     // [2] prep -> state        (count 1)
    uint64_t* pa_bar = bars + 6;    // prep MMA completions
    uint64_t* u_bar = bars + 7;     // state MMA1 (U) completion
    uint64_t* s_bar = bars + 8;     // state MMA2 (S) completion
    uint64_t* o_bar = bars + 9;     // state MMA2 (O) completion
    uint64_t* wt_free = bars + 10;  // state MMA1 done reading -W^T
    uint64_t* drain_p = bars + 11;  // exit: all prep MMAs done
    uint64_t* drain_s = bars + 12;  // exit: all state MMAs done
    uint32_t* tmem_base_p = reinterpret_cast<uint32_t*>(sm + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&gready[0], 1);
        mbar_init(&gready[1], 1);
        mbar_init(&pdone[0], 1);
        mbar_init(&pdone[1], 1);
        mbar_init(pa_bar, 1);
        mbar_init(u_bar, 1);
        mbar_init(s_bar, 1);
        mbar_init(o_bar, 1);
        mbar_init(wt_free, 1);
        mbar_init(drain_p, 1);
        mbar_init(drain_s, 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == 0) tmem_alloc(tmem_base_p, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_p;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lane quarter

    auto abort_now = [&](int code) {
        *abort_flag = 1;
        set_status(a.status, code);
    };

    if (warp < kStateWarp0) {
        // ================================================================ prep
        const int ptid = tid;  // 0..255
        const int half = warp >> 2;
        const int row = 32 * (warp & 3) + lane;  // TMEM lane owned by this thread
        uint32_t pa_phase = 0;
        Item it;
        bool have = item_first(a, total, it);
        for (int i = 0; have; ++i, have = item_next(a, total, it)) {
            const int s = i & 1, ns = i >> 1;
            const int L = it.L;
            uint8_t* st = S.stage(s);
            float* vec = S.vec(s);
            float* gam = vec + 128;
            float* bet = vec + 192;
            float* rq = vec + 256;
            float* rk = vec + 320;
            uint8_t* sP = sm + kOffP + s * 8192;
            // gates g, beta of rows 2*lane and 2*lane+1 (second warp: the first one
            // issues the Gram MMA), in flight across the tile wait
            float4 gb = make_float4(0.f, 0.f, 0.f, 0.f);
            if (warp == 1) {
                const int r = 2 * lane;
                const float* gp = a.g + (it.c0 + r) * H + it.U.h;
                const float* bp = a.beta + (it.c0 + r) * H + it.U.h;
                if (r < L) { gb.x = gp[0]; gb.z = bp[0]; }
                if (r + 1 < L) { gb.y = gp[H]; gb.w = bp[H]; }
            }
            {
                const bool ok = mbar_wait_or_abort(&full[s], ns & 1, abort_flag, a.wait_ns);
                if (group_any(kBarPrep, kPrepThreads, !ok)) {
                    if (ptid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                    break;
                }
            }

            // ---- Gram matrix G = [Q;K][Q;K]^T -> R_A (128 x 128). Its diagonal gives
            // the squared norms of the q and k rows; its lower-right 64 x 64 block is
            // K K^T and its upper-right block Q K^T.
            if (ptid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t qo = (k < 4 ? kQb0 : kQb1) + 32 * (k & 3);
                    const uint64_t d = sw128_desc(smem_u32(st + qo), 16, 1024);  // 128 rows: Q then K
                    mma_bf16(tmem + kRA, d, d, kIdescA, k > 0);
                }
                mma_commit(pa_bar);
            }
            // gamma = inclusive prefix sum of g (scan of the row-pair sums over the
            // warp) and beta into the stage's vector block; the state group waits
            // for them on gready[s].
            if (warp == 1) {
                const float pair = gb.x + gb.y;
                float x = pair;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                const int r = 2 * lane;
                const float g0 = x - pair + gb.x, g1 = x;
                *reinterpret_cast<float2*>(gam + r) = make_float2(g0, g1);
                *reinterpret_cast<float2*>(bet + r) = make_float2(gb.z, gb.w);
                __syncwarp();
                if (lane == 0) mbar_arrive(&gready[s]);
                // range of gamma over the chunk: when it is below 80, e^{gamma_r - gamma_j}
                // factors as e^{gamma_r - gmax} e^{gmax - gamma_j} within fp32, and the
                // P/A epilogue needs no exponential per element
                float mx = fmaxf(g0, g1), mn = fminf(g0, g1);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                }
                if (kUndecayed) {  // A's row decay then reaches back to gamma_{-1} = 0
                    mx = fmaxf(mx, 0.f);
                    mn = fminf(mn, 0.f);
                }
                constexpr float kLog2e = 1.4426950408889634f;
                *reinterpret_cast<float2*>(vec + r) =
                    make_float2(ex2((mx - g0) * kLog2e), ex2((mx - g1) * kLog2e));
                if (lane == 0) {
                    vec[64] = mx;
                    vec[65] = (mx - mn < 80.f) ? 1.f : 0.f;
                }
            }
            {
                const bool ok = mbar_wait_or_abort(pa_bar, pa_phase, abort_flag, a.wait_ns);
                if (group_any(kBarPrep, kPrepThreads, !ok)) {
                    if (ptid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                    break;
                }
                pa_phase ^= 1;
            }
            tc_fence_after();
            // L2-norm factors of row `row` from G[row][row] (half-0 threads), beta copied
            {
                float dg[32];
                tmem_ld32(tmem + lane_off + kRA + 32 * (warp & 3), dg);
                tmem_wait_ld();
                if (half == 0) {
                    float d2 = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) d2 = (e == lane) ? dg[e] : d2;
                    const int r = row & 63;
                    float f = 0.f;
                    if (r < L) f = a.qk_l2norm ? 1.f / sqrtf(d2 + a.eps) : 1.f;
                    if (row < 64) rq[r] = f * a.scale;
                    else rk[r] = f;
                }
            }
            group_sync(kBarPrep, kPrepThreads);

            // ---- P rows (lanes < 64) and A rows (lanes >= 64), 32 columns per
            // thread; a warp covers one 32 x 32 block. Blocks above the diagonal are
            // zero: P's is stored as zeros, A's is never read (the solve uses it as
            // scratch). Inside the diagonal blocks P keeps j <= r; A needs no mask
            // (the solve reads only its strictly lower part). Every element is
            // computed branch-free (exponent clamped at 0 so masked or unread
            // entries stay finite), then selected. When the chunk's decay range is
            // below 80 the decay factors split into a row and a column factor.
            {
                const int rb = warp & 1, cb = half;  // row and column block of this warp
                const bool is_p = row < 64;
                const int r = row & 63;
                const int j0 = 32 * half;
                float x[32];
                if (rb >= cb) {
                    tmem_ld32(tmem + lane_off + kRA + 64 + 32 * half, x);  // columns = k rows
                    tmem_wait_ld();
                    // row decay: gamma_r, or for A rows with the read-before-decay
                    // order gamma_{r-1} (gamma_{-1} = 0)
                    const float gr = (kUndecayed && !is_p) ? (r > 0 ? gam[r - 1] : 0.f) : gam[r];
                    const float fr = is_p ? rq[r] : bet[r] * rk[r];
                    const int lim = (is_p && rb == cb) ? r : 64;  // keep j <= lim
                    if (vec[65] != 0.f) {
                        // factored decay: row factor e^{gamma_r - gmax} <= 1, column
                        // factors e^{gmax - gamma_j} < e^80 from the scan
                        const float frr = fr * ex2((gr - vec[64]) * 1.4426950408889634f);
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int j = j0 + e;
                            const float val = (frr * (vec[j] * rk[j])) * x[e];
                            x[e] = (j <= lim) ? val : 0.f;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int j = j0 + e;
                            const float ex = __expf(fminf(gr - gam[j], 0.f));
                            const float val = ex * (fr * rk[j]) * x[e];
                            x[e] = (j <= lim) ? val : 0.f;
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = 0.f;
                }
                if (is_p) {
                    store_half_row(sP, r, half, x, 1.f);
                } else if (rb >= cb) {
                    float4* Ar = reinterpret_cast<float4*>(sA + r * kLdA + j0);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        Ar[q4] = make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync(kBarPrep, kPrepThreads);

            // ---- solve T = (I + A)^-1 by blocks: 16x16 diagonal inverses by forward
            // substitution (one column per thread, ptid < 64), each warp then merging
            // its pair to 32x32 (T_10 = -T_11 A_10 T_00), then all warps to 64x64.
            // Meanwhile ptid 64..191 turn Q into Q~ and ptid 192..255 clear the
            // upper-right 32x32 block.
            if (ptid < 64) {
                const int o = 16 * (ptid >> 4), c = ptid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s0 = (r == c) ? 1.f : 0.f, s1 = 0.f;
                    const float* Ar = sA + (o + r) * kLdA + o;
#pragma unroll
                    for (int m4 = 0; m4 < r / 4; ++m4) {
                        const float4 av = *reinterpret_cast<const float4*>(Ar + 4 * m4);
                        s0 = fmaf(-av.x, x[4 * m4 + 0], s0);
                        s1 = fmaf(-av.y, x[4 * m4 + 1], s1);
                        s0 = fmaf(-av.z, x[4 * m4 + 2], s0);
                        s1 = fmaf(-av.w, x[4 * m4 + 3], s1);
                    }
#pragma unroll
                    for (int m = (r / 4) * 4; m < r; ++m) s0 = fmaf(-Ar[m], x[m], s0);
                    x[r] = s0 + s1;
                }
                const bool left = ((ptid >> 4) & 1) == 0;  // blocks 0 and 2 clear their right neighbour
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    sT[(o + r) * kLdA + o + c] = x[r];
                    if (left) sT[(o + r) * kLdA + o + 16 + c] = 0.f;
                }
                __syncwarp();
                // 16 -> 32 for this warp's block pair at op (its T_00 and T_11 were just
                // written by the warp): Y = A_10 T_00 into the unused upper-right block
                // of A, then T_10 = -T_11 Y.
                const int op = 32 * warp;
                float* Y = sA + op * kLdA + op + 16;  // 16 x 16 scratch, row-major
                {
                    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const float* a10 = sA + (op + 16) * kLdA + op + 8 * ks;
                        const float* t00 = sT + (op + 8 * ks) * kLdA + op;
                        mma_tf32_16x8x8(d0, a10, kLdA, t00, kLdA);
                        mma_tf32_16x8x8(d1, a10, kLdA, t00 + 8, kLdA);
                    }
                    store_acc_16x8(Y, kLdA, d0, 1.f);
                    store_acc_16x8(Y + 8, kLdA, d1, 1.f);
                }
                __syncwarp();
                {
                    float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const float* t11 = sT + (op + 16) * kLdA + op + 16 + 8 * ks;
                        mma_tf32_16x8x8(z0, t11, kLdA, Y + 8 * ks * kLdA, kLdA);
                        mma_tf32_16x8x8(z1, t11, kLdA, Y + 8 * ks * kLdA + 8, kLdA);
                    }
                    store_acc_16x8(sT + (op + 16) * kLdA + op, kLdA, z0, -1.f);
                    store_acc_16x8(sT + (op + 16) * kLdA + op + 8, kLdA, z1, -1.f);
                }
            } else if (ptid < 192) {
                const int rr = ptid - 64, r = rr & 63;
                scale_row(st + ((rr >> 6) ? kQb1 : kQb0), r, expf(gam[r]) * rq[r]);
            } else {
                for (int e = ptid - 192; e < 32 * 32; e += 64) sT[(e >> 5) * kLdA + 32 + (e & 31)] = 0.f;
            }
            group_sync(kBarPrep, kPrepThreads);
            {
                // 32 -> 64 (all 8 warps: 16-row x 8-column tile each): Y = A_10 T_00 into the
                // unused upper-right 32 x 32 block of A, then T_10 = -T_11 Y.
                const int mt = 16 * (warp & 1), nt = 8 * (warp >> 1);
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_tf32_16x8x8(d, sA + (32 + mt) * kLdA + 8 * ks, kLdA, sT + 8 * ks * kLdA + nt, kLdA);
                float* Y = sA + 32;  // rows 0..31, columns 32..63 of A
                store_acc_16x8(Y + mt * kLdA + nt, kLdA, d, 1.f);
                group_sync(kBarPrep, kPrepThreads);
                float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_tf32_16x8x8(z, sT + (32 + mt) * kLdA + 32 + 8 * ks, kLdA, Y + 8 * ks * kLdA + nt, kLdA);
                store_acc_16x8(sT + (32 + mt) * kLdA + nt, kLdA, z, -1.f);
            }
            group_sync(kBarPrep, kPrepThreads);
            // T1^T, T2^T rows (row m = column m of T) as bf16 MN-major B operands,
            // written over A (dead by now)
            {
                // thread -> (tile, row j, half): 32 values of row j of T1^T or T2^T
                const int j = ptid & 63, hf = (ptid >> 6) & 1, which = ptid >> 7;
                float x[32];
#pragma unroll
                for (int r = 0; r < 32; ++r) x[r] = sT[(32 * hf + r) * kLdA + j];
                const float gj = kUndecayed ? (j > 0 ? gam[j - 1] : 0.f) : gam[j];
                const float f = which == 0 ? bet[j] * expf(gj) * rk[j] : bet[j];
                store_half_row(which == 0 ? sT1 : sT2, j, hf, x, f);
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync(kBarPrep, kPrepThreads);

            // ---- W^T = K^T T1^T -> R_W ;  U~^T = V^T T2^T -> R_U[s]
            if (ptid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + kRW, sw128_desc(smem_u32(st + kKb0 + 2048 * k), kKb1 - kKb0, 1024),
                             sw128_desc(smem_u32(sT1 + 2048 * k), 8192, 1024), kIdescMN, k > 0);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + kRU + 64 * s, sw128_desc(smem_u32(st + kVb0 + 2048 * k), kVb1 - kVb0, 1024),
                             sw128_desc(smem_u32(sT2 + 2048 * k), 8192, 1024), kIdescMN, k > 0);
                mma_commit(pa_bar);
            }
            {
                bool ok = mbar_wait_or_abort(pa_bar, pa_phase, abort_flag, a.wait_ns);
                // -W^T is about to be overwritten: the state group's MMA1 of the
                // previous chunk must be done reading it.
                if (ok && i > 0) ok = mbar_wait_or_abort(wt_free, (i - 1) & 1, abort_flag, a.wait_ns);
                if (group_any(kBarPrep, kPrepThreads, !ok)) {
                    if (ptid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                    break;
                }
                pa_phase ^= 1;
            }
            tc_fence_after();

            // ---- -W^T rows (lane = dk i, 32 columns each)
            {
                float x[32];
                tmem_ld32(tmem + lane_off + kRW + 32 * half, x);
                tmem_wait_ld();
                store_half_row(sWT, row, half, x, -1.f);
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync(kBarPrep, kPrepThreads);
            if (ptid == 0) mbar_arrive(&pdone[s]);
        }
        // drain this issuer's MMAs before TMEM is freed
        if (ptid == 0) {
            mma_commit(drain_p);
            mbar_wait(drain_p, 0, kWaitNs / 4);
        }
    } else {
        // ================================================================ state
        const int stid = tid - kPrepThreads;  // 0..127 = TMEM lane = dv index j
        const int j = stid;
        uint32_t ph = 0;  // parity of u_bar / s_bar / o_bar (one completion each per chunk)
        // Units with no tokens on this CTA's stride still need hT = h0.
        for (int64_t e = blockIdx.x; e < total; e += gridDim.x) {
            Unit U;
            if (!load_unit(a, e, U)) {
                if (stid == 0) set_status(a.status, kStatusBadSeqlens);
                continue;
            }
            if (U.end > U.start || !a.hT) continue;
            const int64_t base = ((int64_t)U.n * H + U.h) * kD * kD;
            for (int x = stid; x < kD * kD; x += kStateThreads) a.hT[base + x] = a.h0 ? a.h0[base + x] : 0.f;
        }
        // Refill of stage s with item `f`: one lane outside the MMA-issuing warp arms
        // the stage barrier and issues the six TMA tile loads.
        constexpr int kRefill = 32;
        uint32_t issued = 0, issued_par = 0;  // for the bounded drain at exit
        auto fill = [&](const Item& f, int s, int use) {
            if (stid != kRefill) return;
            issue_tiles(S.stage(s), &full[s], &map_q, &map_k, &map_v, f.U.h / group, f.U.h, f.c0);
            issued |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | ((uint32_t)(use & 1) << s);
        };
        if (stid == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
            prefetch_tmap(&map_o);
        }
        Item it, ahead;
        bool have = item_first(a, total, it);
        bool have_ahead = have;
        if (have) {
            ahead = it;
            fill(ahead, 0, 0);
            have_ahead = item_next(a, total, ahead);
            if (have_ahead) {
                fill(ahead, 1, 0);
                have_ahead = item_next(a, total, ahead);  // ahead = item 2
            }
        }
        bool drained = true;
        for (int i = 0; have; ++i, have = item_next(a, total, it)) {
            const int s = i & 1, ns = i >> 1;
            const int L = it.L;
            const int64_t c0 = it.c0;
            uint8_t* st = S.stage(s);
            const float* vec = S.vec(s);
            const int64_t sbase = ((int64_t)it.U.n * H + it.U.h) * kD * kD;
            if (it.first) {
                // initial state: S^T as the bf16 A operand in R_SB (thread = dv lane j)
                // and e^{gamma_L} S^T in R_S -- R_S always holds the state pre-decayed
                // by the coming chunk, ready for the accumulation of K~^T U.
                {
                    const bool ok = mbar_wait_or_abort(&gready[s], ns & 1, abort_flag, a.wait_ns);
                    if (group_any(kBarState, kStateThreads, !ok)) {
                        if (stid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                        break;
                    }
                }
                const float* h0p = a.h0 ? a.h0 + sbase + j : nullptr;  // column j of S
                const float eL = expf(vec[128 + 63]);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float v[32];
                    if (h0p) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = h0p[(32 * cc + e) * kD];
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = 0.f;
                    }
                    uint32_t w[16];
                    pack_row32(v, 1.f, w);
                    tmem_st16(tmem + lane_off + kRSB + 16 * cc, w);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] *= eL;
                    tmem_st32(tmem + lane_off + kRS + 32 * cc, v);
                }
                tmem_wait_st();
                tc_fence_before();
                group_sync(kBarState, kStateThreads);
            }
            {
                const bool ok = mbar_wait_or_abort(&pdone[s], ns & 1, abort_flag, a.wait_ns);
                if (group_any(kBarState, kStateThreads, !ok)) {
                    if (stid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                    break;
                }
            }
            tc_fence_after();
            drained = false;
            // ---- MMA1: U^T += S^T (-W^T) (R_U[s]) ; O^T = S^T Q~^T (R_O), A = S^T from R_SB
            if (stid == 0) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ta(tmem + kRU + 64 * s, tmem + kRSB + 8 * k,
                                sw128_desc(smem_u32(sWT + 2048 * k), 8192, 1024), kIdescSW, 1);
                mma_commit(u_bar);
                mma_commit(wt_free);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t qo = (k < 4 ? kQb0 : kQb1) + 32 * (k & 3);
                    mma_bf16_ta(tmem + kRO, tmem + kRSB + 8 * k, sw128_desc(smem_u32(st + qo), 16, 1024),
                                kIdescSQ, k > 0);
                }
            } else if (stid >= 32) {
                // while MMA1 runs: K -> K~ = diag(e^{gamma_L - gamma} / |k|) K in place
                // for MMA2 (the prep group's W^T MMA has read the raw K), 128 rows
                // over the state group's other three warps
                const float gL = vec[128 + 63];
                for (int x = stid - 32; x < 128; x += kStateThreads - 32) {
                    const int r = x & 63;
                    scale_row(st + (x < 64 ? kKb0 : kKb1), r, expf(gL - vec[128 + r]) * vec[320 + r]);
                }
            }
            {
                const bool ok = mbar_wait_or_abort(u_bar, ph, abort_flag, a.wait_ns);
                if (group_any(kBarState, kStateThreads, !ok)) {
                    if (stid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                    break;
                }
            }
            tc_fence_after();
            // ---- U^T row j (64 tokens) as packed bf16 in the first 32 columns of
            // R_U[s]: the TMEM-resident A operand of MMA2
            {
                uint32_t w[32];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float x[32];
                    tmem_ld32(tmem + lane_off + kRU + 64 * s + 32 * hf, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 16; ++c) w[16 * hf + c] = pack_bf16(x[2 * c], x[2 * c + 1]);
                }
                tmem_st32(tmem + lane_off + kRU + 64 * s, w);
                tmem_wait_st();
            }
            fence_proxy_async();  // K~ (generic writes) is read by MMA2
            tc_fence_before();
            group_sync(kBarState, kStateThreads);
            // ---- MMA2: S^T += U^T K~ (R_S) ; O^T += U^T P^T (R_O[s])
            if (stid == 0) {
                tc_fence_after();
                uint8_t* sP = sm + kOffP + s * 8192;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ta(tmem + kRS, tmem + kRU + 64 * s + 8 * k,
                                sw128_desc(smem_u32(st + kKb0 + 2048 * k), kKb1 - kKb0, 1024), kIdescUK, 1);
                mma_commit(s_bar);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ta(tmem + kRO, tmem + kRU + 64 * s + 8 * k,
                                sw128_desc(smem_u32(sP + 32 * k), 16, 1024), kIdescSQ, 1);
                mma_commit(o_bar);
                bulk_wait_group_read0();  // the previous O store has read the staging tile
            }
            {
                bool ok = mbar_wait_or_abort(s_bar, ph, abort_flag, a.wait_ns);
                // gamma of the next chunk (other stage), for the pre-decay below
                if (ok && !it.last) ok = mbar_wait_or_abort(&gready[s ^ 1], ((i + 1) >> 1) & 1, abort_flag, a.wait_ns);
                if (group_any(kBarState, kStateThreads, !ok)) {
                    if (stid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                    break;
                }
            }
            // MMA1 and MMA2's state half, the last readers of stage s, are done:
            // refill it with the chunk two ahead
            if (have_ahead) {
                fill(ahead, s, ns + 1);
                have_ahead = item_next(a, total, ahead);
            }
            tc_fence_after();
            // ---- new state: bf16 S^T for the next chunk's MMA1, and R_S pre-decayed
            // by the next chunk's e^{gamma_L} (its gates are already in the other
            // stage's vector block); the final state at the end of a sequence.
            {
                const float eL = it.last ? 1.f : expf(S.vec(s ^ 1)[128 + 63]);
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    float v[32];
                    tmem_ld32(tmem + lane_off + kRS + 32 * cc, v);
                    tmem_wait_ld();
                    {
                        uint32_t w[16];
                        pack_row32(v, 1.f, w);
                        tmem_st16(tmem + lane_off + kRSB + 16 * cc, w);
                    }
                    if (it.last) {
                        if (a.hT) {
                            float* hTp = a.hT + sbase + j + 32 * cc * kD;
#pragma unroll
                            for (int e = 0; e < 32; ++e) hTp[e * kD] = v[e];
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] *= eL;
                        tmem_st32(tmem + lane_off + kRS + 32 * cc, v);
                    }
                }
                tmem_wait_st();
            }
            {
                const bool ok = mbar_wait_or_abort(o_bar, ph, abort_flag, a.wait_ns);
                if (group_any(kBarState, kStateThreads, !ok)) {
                    if (stid == 0 && !*abort_flag) abort_now(kStatusTimeout);
                    break;
                }
            }
            tc_fence_after();
            ph ^= 1;
            // ---- O: column j of O^T -> O staging tile as two [64 tokens][64 d_v]
            // row-major boxes; a full chunk leaves by one TMA store, a partial one as
            // 16-byte rows of its L valid tokens.
            {
                uint16_t* ostage = reinterpret_cast<uint16_t*>(sO) + (j >> 6) * 4096 + (j & 63);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float x[32];
                    tmem_ld32(tmem + lane_off + kRO + 32 * hf, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ostage[(32 * hf + e) * 64] = f32_to_bf16(x[e]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync(kBarState, kStateThreads);
            if (L == kC) {
                if (stid == 0) {
                    tma_store_3d(&map_o, sO, 0, it.U.h, (int)c0);
                    tma_store_3d(&map_o, sO + 8192, 64, it.U.h, (int)c0);
                    bulk_commit_group();
                }
            } else {
                uint16_t* obase = static_cast<uint16_t*>(a.o) + (c0 * H + it.U.h) * kD;
                const int64_t tok_stride = (int64_t)H * kD;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int vid = stid + kStateThreads * k;  // token r, 16-byte column c16
                    const int r = vid >> 4, c16 = vid & 15;
                    if (r < L) {
                        const uint8_t* src = sO + (c16 >> 3) * 8192 + r * 128 + (c16 & 7) * 16;
                        *reinterpret_cast<uint4*>(obase + r * tok_stride + 8 * c16) =
                            *reinterpret_cast<const uint4*>(src);
                    }
                }
                group_sync(kBarState, kStateThreads);  // staging read before it is rewritten
            }
            drained = true;
        }
        if (stid == 0) bulk_wait_group0();  // O stores issued by this thread
        if (stid == 0 && !drained) {
            mma_commit(drain_s);
            mbar_wait(drain_s, 0, kWaitNs / 4);
        }
        // TMA loads the prep group never consumed (only after an abort)
        if (stid == kRefill && *abort_flag)
            for (int x = 0; x < 2; ++x)
                if ((issued >> x) & 1u) mbar_wait(&full[x], (issued_par >> x) & 1u, kWaitNs / 4);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [T_tot, H, 128] bf16 (tokens `ld` elements apart) viewed as a 3-D tensor
// (feature, head, token); boxes of
// 64 features x 1 head x 64 tokens, zero fill past T_tot on loads, clipped on
// stores. Loads use the 128-byte swizzle the MMA descriptors expect; the O
// store reads a plain row-major staging tile.
bool make_map(CUtensorMap* m, const void* ptr, int H, int64_t T, int64_t ld, bool swizzle) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)ld * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(const PrefillArgs& a) {
    return a.is_bf16 && a.dk == kD && a.dv == kD && a.chunk == kC && a.T_tot > 0 &&
           a.T_tot < ((int64_t)1 << 31) && encode_fn() != nullptr;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, a.Hk, a.T_tot, a.ld_q, true) || !make_map(&mk, a.k, a.Hk, a.T_tot, a.ld_k, true) ||
        !make_map(&mv, a.v, a.H, a.T_tot, a.ld_v, true) ||
        !make_map(&mo, a.o, a.H, a.T_tot, (int64_t)a.H * kD, false))
        return cudaErrorInvalidValue;
    auto kernel = a.undecayed ? prefill_tc_kernel<true> : prefill_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t units = (int64_t)a.N * a.H;
    const int grid = (int)(units < sms ? units : sms);
    TcParams p{a};
    kernel<<<grid, kThreads, kSmemAlloc, s>>>(p, mq, mk, mv, mo);
    return cudaGetLastError();
}

}  // namespace gdn
