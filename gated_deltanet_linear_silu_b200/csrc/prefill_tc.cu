// Chunked gated delta rule on the 5th-generation tensor cores (tcgen05):
// bf16 q/k/v, d_k = d_v = 128, chunk C = 64, fp32 state and accumulation.
//
// The recurrence is the decay-first rule of "Qwen3.5-MoE source walkthrough",
// 4.3; the chunk algebra (cumulative decay gamma, UT transform with a unit
// lower-triangular solve, inter-chunk state passing) is that of
// "Parallelizing Linear Transformers with the Delta Rule over Sequence Length"
// (Yang et al., 2024) with the gating of "Gated Delta Networks" (Yang, Kautz,
// Hatamizadeh, 2024). Per chunk (rows r = tokens, S = state [dk, dv], ^ the
// per-row L2 norm, rq / rk the norm factors of the q / k rows):
//   A = strict_tril(diag(beta) (K^ K^^T) o M),  T = (I+A)^-1
//   W = T diag(beta e^gamma) K^,   U~ = T diag(beta) V,   U = U~ - W S
//   O = diag(rq) [diag(e^gamma) Q S + P U],   P = (Q K^^T) o M
//   S <- e^{gamma_L} S + (diag(e^{gamma_L-gamma}) K^)^T U
// with M[r][j] = e^{gamma_r - gamma_j} for j <= r, else 0. The q norm (with the
// query scale) is a pure row factor of O, so it is applied to the output only.
// When |gamma| < 60 over the chunk (the common case) the decay factors too:
// M[r][j] = e^{gamma_r} e^{-gamma_j}, so P' = (Q K^^T) o (e^{-gamma_j} mask)
// and O = diag(rq e^gamma) [Q S + P' U] -- no per-element exponential, and
// Q enters the MMA unscaled; otherwise P keeps the exact masked exponentials
// and Q is scaled by e^gamma in place. K~ = diag(e^{gamma_L - gamma} rk) K
// never exists: its row factors scale U's columns in a second bf16 copy.
//
// B200 mapping. Every contraction is an M = 128 tcgen05.mma on transposed
// products (the 128-wide head dimension is the MMA's M), with fp32
// accumulators in tensor memory (TMEM, 512 columns):
//   [Q;K] K^T          -> R_G   (lanes 0-63: Q K^T, lanes 64-127: K K^T)
//   W^T  = K^T T1      -> R_W   (lanes = dk, columns = tokens)
//   U~^T = V^T T2      -> R_U[b]
//   U^T  = U~^T + S^T (-W^T)                 (accumulated in R_U[b])
//   O^T  = S^T Q^T + U^T P'^T                (R_O)
//   S^T += (U^T diag(e^{gamma_L - gamma} rk / E)) K   (R_S = S^T / E, fp32)
// R_S is the fp32 master state over a running scale E: a chunk's decay
// multiplies E, and R_S is rewritten (pre-decayed, E = 1) only when E would
// fall below 2^-30, so most chunks never rewrite the 64 KB state.
// S^T and U^T are the A operands of the state MMAs and stay in TMEM as packed
// bf16 (R_SB; R_U[b] holds U^T and its column-scaled copy); only B operands
// come from shared memory, all of them read in place as TMA left them except
// the small P, T1, T2 and -W^T tiles the epilogues write. The triangular solve runs on CUDA cores in fp32 in place
// over A: 16 x 16 diagonal blocks by substitution in registers, merged on
// tf32 mma.sync tiles.
//
// Warp roles (one persistent CTA of 16 warps per SM; units (sequence, head) in
// longest-first order, CTA c starting with unit c and taking the next from a
// work counter as it runs out; every role walks the same list of 64-token
// chunks):
//   warp 0        TMA producer: q, k, v tiles of a chunk into a 3-stage ring;
//                 takes the CTA's next unit from the work counter
//   warp 1        issues the state-independent MMAs (Gram, W^T, U~^T)
//   warp 2        issues the state MMAs (U, O, S); the last MMA of a chunk
//                 frees its stage for the producer
//   warp 3        gates: beta, the cumulative decay gamma and its factors
//   warps 4-7     Gram epilogue (P, A, k norms), solve, export of T1 and T2
//   warps 8-11    -W^T epilogue and q norms of a chunk (Q scaled in place when
//                 the decay does not factor), then the previous chunk's output,
//                 stored straight to HBM
//   warps 12-15   state epilogues: U^T and its scaled copy, S^T to bf16, the
//                 running scale, the final state
// The state chain of a chunk is MMA U -> U epilogue -> MMA S -> S^T to bf16;
// the next chunks' tiles, Gram, solve and W, and the output overlap with it. Roles hand off through mbarriers. Every hand-off wait is
// bounded: on timeout the kernel records the timeout status, all roles leave
// their loops, MMAs and TMA copies are drained (bounded), TMEM is freed and
// the kernel returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace {

using namespace tc;

constexpr int kC = 64;   // chunk
constexpr int kD = 128;  // head dim (dk = dv)
constexpr int kThreads = 512;
constexpr int kStages = 3;
constexpr int kWarpTma = 0, kWarpMmaPrep = 1, kWarpMmaState = 2, kWarpGate = 3;
constexpr int kWg1 = 4, kWg2 = 8, kWg3 = 12;          // first warp of each epilogue group
constexpr int kBarWg1 = 1, kBarWg2 = 2, kBarWg3 = 3;  // named barrier ids (128 threads)
constexpr uint64_t kDrainNs = kDefaultWaitNs / 4;

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t kBox = 8192;  // 64 rows x 128 B (64 bf16)
// stage: [Q box0][K box0][Q box1][K box1][V box0][V box1]; [Q;K] of a box is
// 128 consecutive rows (the Gram MMA's A operand).
constexpr uint32_t kQb0 = 0, kKb0 = kBox, kQb1 = 2 * kBox, kKb1 = 3 * kBox;
constexpr uint32_t kVb0 = 4 * kBox;
constexpr uint32_t kStageBytes = 6 * kBox;           // 48 KB
constexpr uint32_t kOffP = kStages * kStageBytes;    // P bf16 [64 r][64 j] (K-major), per stage
constexpr uint32_t kOffT1 = kOffP + kStages * kBox;  // T1 bf16 [64 r][64 j] (K-major)
constexpr uint32_t kOffT2 = kOffT1 + kBox;           // T2
constexpr uint32_t kOffWT = kOffT2 + kBox;           // -W^T bf16 [128 dk][64 tok] (MN-major)
constexpr int kLdA = 68;                             // padded fp32 row stride
constexpr uint32_t kOffA = kOffWT + 2 * kBox;        // A, then T, fp32 [64][kLdA]
constexpr uint32_t kOffVec = kOffA + 64 * kLdA * 4;  // per-stage vectors
constexpr uint32_t kVecBytes = 2176;
constexpr uint32_t kOffOf = kOffVec + kStages * kVecBytes;  // output row factors, 2 x 64 fp32
constexpr uint32_t kOffBar = kOffOf + 2 * 64 * 4;
constexpr uint32_t kOffMisc = kOffBar + 512;
constexpr int kRing = 16;                            // unit ring: [kRing] x (unit, ordinal tag)
constexpr uint32_t kOffRing = kOffMisc + 64;
constexpr uint32_t kSmemBytes = kOffRing + kRing * 8;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kOffP % 1024 == 0 && kOffT1 % 1024 == 0 && kOffWT % 1024 == 0, "swizzle alignment");

// Per-stage vector block (fp32 offsets, 64 per row vector): gamma, beta,
// e^{-gamma} (P's and A's column decay when it factors), e^{gamma'} (A's and
// W's row decay: gamma_r, or gamma_{r-1} in the read-before-decay order),
// e^{gamma} (the output's row decay when it factors), e^{gamma_L - gamma} (0
// past the chunk's end), the k norm factors rk, kf = e^{gamma_L - gamma} rk,
// then the factored-decay flag and e^{gamma_L}. The output row factors (q norm
// times decay) live apart, in a ring of two, because the output of a chunk is
// written after the next chunk's vectors are needed.
constexpr int kVGam = 0, kVBet = 64, kVCf = 128, kVEa = 192, kVEr = 256, kVEgl = 320, kVRk = 384;
constexpr int kVKf = 448, kVFlag = 512, kVEL = 513;
constexpr float kFactorLimit = 60.f;  // |gamma| bound of the factored decay
constexpr float kRescale = 9.3132257e-10f;  // 2^-30: least running state scale E

// TMEM columns (fp32, 128 lanes).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kRS = 0, kRSB = 128, kRO = 192, kRU = 256, kRG = 384, kRW = 448;

constexpr uint32_t kIdescG = idesc_bf16(128, 64, 0, 0);    // [Q;K] K^T
constexpr uint32_t kIdescW = idesc_bf16(128, 64, 1, 0);    // K^T T1, V^T T2
constexpr uint32_t kIdescSW = idesc_bf16(128, 64, 0, 1);   // S^T (-W^T)
constexpr uint32_t kIdescSQ = idesc_bf16(128, 64, 0, 0);   // S^T Q~^T, U^T P^T
constexpr uint32_t kIdescUK = idesc_bf16(128, 128, 0, 1);  // U^T K~

constexpr float kLog2e = 1.4426950408889634f;

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

// Scale the 128-byte row `row` of a swizzled bf16 tile in place by f; returns
// the sum of squares of the row's values before scaling.
__device__ __forceinline__ float scale_row_ss(uint8_t* tile, int row, float f) {
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
        uint4* p = reinterpret_cast<uint4*>(tile + sw128_off(row, c));
        uint4 u = *p;
        float x, y;
        unpack_bf16(u.x, x, y); ss = fmaf(x, x, fmaf(y, y, ss)); u.x = pack_bf16(x * f, y * f);
        unpack_bf16(u.y, x, y); ss = fmaf(x, x, fmaf(y, y, ss)); u.y = pack_bf16(x * f, y * f);
        unpack_bf16(u.z, x, y); ss = fmaf(x, x, fmaf(y, y, ss)); u.z = pack_bf16(x * f, y * f);
        unpack_bf16(u.w, x, y); ss = fmaf(x, x, fmaf(y, y, ss)); u.w = pack_bf16(x * f, y * f);
        *p = u;
    }
    return ss;
}

// Sum of squares of the 64 values of row `row` of a swizzled bf16 tile.
__device__ __forceinline__ float sumsq_row(const uint8_t* tile, int row) {
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile + sw128_off(row, c));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 v = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
            acc = __ffma2_rn(v, v, acc);
        }
    }
    return acc.x + acc.y;
}

// Warp-level m16n8k8 TF32 tensor-core product (fp32 accumulate) used by the
// merges of the triangular solve: d(16x8) += A(16x8) * B(8x8), both read from
// fp32 shared memory with row stride kLdA (B as k x n). The fp32 bit patterns
// go in as they are: the tensor core uses their tf32 part (the top 19 bits).
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const float* A, const float* B) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t a0 = __float_as_uint(A[g * kLdA + t]), a1 = __float_as_uint(A[(g + 8) * kLdA + t]);
    const uint32_t a2 = __float_as_uint(A[g * kLdA + t + 4]), a3 = __float_as_uint(A[(g + 8) * kLdA + t + 4]);
    const uint32_t b0 = __float_as_uint(B[t * kLdA + g]), b1 = __float_as_uint(B[(t + 4) * kLdA + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// d (16 x 8) += A (16 x 8nk) B (8nk x 8).
__device__ __forceinline__ void mma_tf32_16x8(float (&d)[4], const float* A, const float* B, int nk) {
    for (int ks = 0; ks < nk; ++ks) mma_tf32_16x8x8(d, A + 8 * ks, B + 8 * ks * kLdA);
}
// Store the 16x8 accumulator tile (times f) row-major with stride kLdA.
__device__ __forceinline__ void store_acc_16x8(float* D, const float (&d)[4], float f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2*>(D + g * kLdA + 2 * t) = make_float2(f * d[0], f * d[1]);
    *reinterpret_cast<float2*>(D + (g + 8) * kLdA + 2 * t) = make_float2(f * d[2], f * d[3]);
}
// D (16 x 16) = f * A (16 x 16) B (16 x 16), one warp; D must not overlap A or B.
__device__ __forceinline__ void mma_tf32_16x16(float* D, const float* A, const float* B, float f) {
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    mma_tf32_16x8(d0, A, B, 2);
    mma_tf32_16x8(d1, A, B + 8, 2);
    store_acc_16x8(D, d0, f);
    store_acc_16x8(D + 8, d1, f);
}

struct Unit {
    int n, h;
    int64_t start, end;
};

// Unit u = (sequence order[u / H], head u % H) with its bounds checked (the
// hT = h0 copies of units without tokens, and the status of bad ones).
__device__ __forceinline__ bool load_unit_checked(const PrefillArgs& a, int u, Unit& U) {
    U.h = u % a.H;
    U.n = a.order[u / a.H];
    if (U.n < 0 || U.n >= a.N) return false;
    U.start = a.cu[U.n];
    U.end = a.cu[U.n + 1];
    return U.start >= 0 && U.start <= U.end && U.end <= a.T_tot;
}

// The CTA's work list: the 64-token chunks of its units, in order. The first
// unit is u = blockIdx.x; each later one is taken from the work counter when
// the producer reaches it (units in longest-first order, the sequences with
// tokens first), so a CTA whose units are short takes more of them. The
// producer publishes the k-th unit of the CTA in slot k % kRing of a ring in
// shared memory (the unit, then the ordinal k as its tag); every other role
// reads the slot once the tag shows k. No role trails the producer by kRing
// units: the stage ring keeps them within a few chunks. Every role walks the
// same list.
struct Item {
    int u;
    int k;  // ordinal of the unit within this CTA
    Unit U;
    int64_t c0;
    int L;
    bool first, last;
};

struct UnitRing {
    volatile int* slot;  // [kRing][2]
    int* counter;        // work counter (the schedule zeroes it)
    int* status;
    volatile int* abort_flag;
    uint64_t wlim;
    bool producer;
};

// The k-th (k >= 1) unit of this CTA, or -1 past the last. A reader whose wait
// runs out (or sees another role's abort) records the timeout and gets -1.
// Scalar arguments: the one copy of the wait loop serves every call site.
__device__ __noinline__ int ring_unit(volatile int* slot, int* counter, int* status, volatile int* abort_flag,
                                      uint64_t wlim, bool producer, int k, int units) {
    volatile int* e = slot + 2 * (k % kRing);
    if (producer) {
        const int u = (int)gridDim.x + atomicAdd(counter, 1);
        const int v = u < units ? u : -1;
        e[0] = v;
        __threadfence_block();
        e[1] = k;
        return v;
    }
    if (e[1] != k) {
        const uint64_t t0 = globaltimer_ns();
        while (e[1] != k) {
            if (*abort_flag || globaltimer_ns() - t0 >= wlim) {
                if (!*abort_flag) {
                    *abort_flag = 1;
                    set_status(status, kStatusTimeout);
                }
                return -1;
            }
            __nanosleep(64);
        }
    }
    __threadfence_block();
    return e[0];
}

__device__ __forceinline__ void item_unit(const PrefillArgs& a, Item& it) {
    it.U.h = it.u % a.H;
    it.U.n = a.order[it.u / a.H];
    it.U.start = a.cu[it.U.n];
    it.U.end = a.cu[it.U.n + 1];
    it.c0 = it.U.start;
    it.first = true;
}
__device__ __forceinline__ void item_len(Item& it) {
    it.L = (int)((it.U.end - it.c0 < kC) ? it.U.end - it.c0 : kC);
    it.last = it.c0 + kC >= it.U.end;
}
__device__ __forceinline__ bool item_first(const PrefillArgs& a, int units, Item& it) {
    it.u = blockIdx.x;
    it.k = 0;
    if (it.u >= units) return false;
    item_unit(a, it);
    item_len(it);
    return true;
}
__device__ __forceinline__ bool item_next(const PrefillArgs& a, int units, Item& it, const UnitRing& ring) {
    it.c0 += kC;
    it.first = false;
    if (it.c0 >= it.U.end) {
        it.k += 1;
        it.u = ring_unit(ring.slot, ring.counter, ring.status, ring.abort_flag, ring.wlim, ring.producer, it.k,
                         units);
        if (it.u < 0) return false;
        item_unit(a, it);
    }
    item_len(it);
    return true;
}

// ---- Fused conv ("7.6 Qwen3.5: linear-attention hybrid", 7.6.2: depthwise causal
// Conv1d, kernel 4, padding 3, then SiLU). A producer lane owns one 16-byte column
// (8 channels) of a 64-channel box of the stage: channel ch of x, whose row p
// starts at xp + p * ld.

// Half the taps of channels ch .. ch+7, right-aligned into a 4-wide window: w2[j][p]
// holds tap j of the channel pair p times 1/2, so the sum is h = y/2 of
// y_t = sum_j w[j] x_{t-3+j} (zero taps for K < 4), SiLU's argument; scaling by a
// power of two commutes with the rounding, so h is exactly half the fp32 sum.
__device__ __forceinline__ void conv_load_taps(const PrefillArgs& a, int ch, float2 (&w2)[4][4]) {
    const uint16_t* w = static_cast<const uint16_t*>(a.conv_w);
    const int K = a.conv_K;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int jj = j - (4 - K);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float lo = 0.f, hi = 0.f;
            if (jj >= 0) {
                lo = 0.5f * bf16_to_f32(w[(int64_t)(ch + 2 * p) * K + jj]);
                hi = 0.5f * bf16_to_f32(w[(int64_t)(ch + 2 * p + 1) * K + jj]);
            }
            w2[j][p] = make_float2(lo, hi);
        }
    }
}

// Raw input of the lane's 8 channels at token p of conv sequence nseq (first token
// seq0): x from seq0 on; before it the sequence's conv state window (column
// K-1 + p - seq0), or zeros where there is none.
__device__ __forceinline__ void conv_fetch(const PrefillArgs& a, const uint16_t* xp, int ch, int nseq,
                                           int64_t seq0, int64_t p, float2 (&x)[4]) {
    if (p >= seq0) {
        const uint4 u = *reinterpret_cast<const uint4*>(xp + p * a.ld_q);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) unpack_bf16(w[q], x[q].x, x[q].y);
        return;
    }
    const int W = a.conv_K - 1;
    const int64_t col = W + (p - seq0);
    const uint16_t* st = static_cast<const uint16_t*>(a.conv_state);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float lo = 0.f, hi = 0.f;
        if (st && col >= 0) {
            lo = bf16_to_f32(st[((int64_t)nseq * a.ld_q + ch + 2 * q) * W + col]);
            hi = bf16_to_f32(st[((int64_t)nseq * a.ld_q + ch + 2 * q + 1) * W + col]);
        }
        x[q] = make_float2(lo, hi);
    }
}

// At the first chunk of a unit: the lane's taps and the raw rows c0-3 .. c0-1 before
// the chunk (from x inside a sequence split into segments, else the conv state).
__device__ __forceinline__ void conv_unit_start(const PrefillArgs& a, int n, int64_t c0, int ch,
                                                const uint16_t* xp, float2 (&w2)[4][4], float2 (&win)[3][4]) {
    conv_load_taps(a, ch, w2);
    const int nseq = n / a.conv_seg;
    const int64_t seq0 = a.conv_cu[nseq];
#pragma unroll
    for (int j = 0; j < 3; ++j) conv_fetch(a, xp, ch, nseq, seq0, c0 - 3 + j, win[j]);
}

// Conv + SiLU in place over the 64 raw rows of one 16-byte column of a swizzled
// bf16 box, with the arithmetic of the standalone conv (fp32 pairs; SiLU(y) =
// h + h tanh(h) with h = y/2 from the halved taps, one XU operation per element;
// bf16 rounding). win comes in with the three raw rows before the box's first
// row (oldest first) and leaves with its last three raw rows. Rows go in batches
// of four: all four loads before the first store, since a store to a swizzled
// address would otherwise hold back the next row's load (the compiler cannot
// tell the rows apart) and chain all 64 rows end to end.
__device__ __forceinline__ void conv_column(uint8_t* box, int c16, const float2 (&w2)[4][4],
                                            float2 (&win)[3][4]) {
#pragma unroll 1
    for (int r0 = 0; r0 < kC; r0 += 4) {
        uint8_t* rows = box + r0 * 128;
        const int sw = r0 & 4;  // the rows' swizzle phase
        uint4 raw[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) raw[b] = *reinterpret_cast<const uint4*>(rows + sw128_off(sw + b, c16) - sw * 128);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t wi[4] = {raw[b].x, raw[b].y, raw[b].z, raw[b].w};
            float2 xt[4];
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                unpack_bf16(wi[q], xt[q].x, xt[q].y);
                float2 acc = __fmul2_rn(w2[0][q], win[0][q]);
                acc = __ffma2_rn(w2[1][q], win[1][q], acc);
                acc = __ffma2_rn(w2[2][q], win[2][q], acc);
                acc = __ffma2_rn(w2[3][q], xt[q], acc);  // h = y / 2
                float2 t;
                asm("tanh.approx.f32 %0, %1;" : "=f"(t.x) : "f"(acc.x));
                asm("tanh.approx.f32 %0, %1;" : "=f"(t.y) : "f"(acc.y));
                const float2 s = __ffma2_rn(acc, t, acc);
                o[q] = pack_bf16(s.x, s.y);
            }
            *reinterpret_cast<uint4*>(rows + sw128_off(sw + b, c16) - sw * 128) = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                win[0][q] = win[1][q];
                win[1][q] = win[2][q];
                win[2][q] = xt[q];
            }
        }
    }
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

// Bounded wait that also gives up once another role has aborted (checked
// between sleeps of at most 0.2 ms). limit 0: only a phase already complete at
// the first (non-blocking) probe passes. One thread per role waits; the others
// of a warp group learn the outcome at a named barrier. Not inlined: one copy
// of the loop serves every wait of the kernel.
__device__ __noinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort_flag, uint64_t limit) {
    if (limit == 0) return mbar_test_wait(bar, parity);
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 200000u)) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit) return false;
    }
    return true;
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
    tma_load_3d(stage + kVb0 + kBox, mv, bar, 64, h, t);
}

// mbarriers (arrival count in parentheses; "commit" = tcgen05.commit).
struct Bars {
    uint64_t full[kStages];      // tiles of a stage landed              (TMA bytes)
    uint64_t conv_full[kStages];  // fused conv: tiles convolved          (warps 0 and 3, 1 each)
    uint64_t empty[kStages];     // tiles of a stage no longer read      (commit)
    uint64_t vfree[kStages];     // vector block of a stage no longer read (WG3, 1)
    uint64_t gready[kStages];    // gate vectors of a stage written      (gate warp, 1)
    uint64_t rk_ready[kStages];  // k norm factors of a stage written    (WG1, 1)
    uint64_t g_full;             // Gram MMA done                        (commit)
    uint64_t g_free;             // R_G read                             (WG1, 128)
    uint64_t t_ready;            // P, T1, T2 written                    (WG1, 1)
    uint64_t w_full;             // W^T / U~^T MMAs done                 (commit)
    uint64_t w_free;             // R_W read                             (WG2, 128)
    uint64_t wt_ready;           // -W^T, K~, Q~ written                 (WG2, 1)
    uint64_t wt_free;            // MMA U done reading -W^T              (commit)
    uint64_t u_full;             // MMA U done                           (commit)
    uint64_t ub_ready;           // U^T as bf16 in TMEM                  (WG3, 1)
    uint64_t s_full;             // MMA S and MMA O1 done                (commit)
    uint64_t sb_ready;           // S^T as bf16 in R_SB                  (WG3, 1)
    uint64_t sd_ready;           // R_S pre-decayed or initialised       (WG3, 1)
    uint64_t o_full[2];          // MMA O2 done, per U buffer            (commit)
    uint64_t o_free;             // R_O read                             (WG3, 128)
    uint64_t drain_prep, drain_state;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

// kUndecayed: each token reads the state before its own decay (row decay
// gamma_{r-1} in A and W). A template parameter, so the default order's code is
// not touched by the option. kConv: the tiles are raw rows of the layer input,
// convolved in shared memory by warp 0 (q, k) and the gate warp (v) before the
// Gram MMA reads them.
template <bool kUndecayed, bool kConv>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ TcParams P, const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
    extern __shared__ uint8_t smem_raw[];
    // Dependent launch (the sequence split's passes): the next kernel may start
    // launching; this one reads the schedule (and every input) only after the
    // previous kernel has finished. No-ops for an ordinary launch.
    pdl_launch_dependents();
    pdl_wait_previous();
    // 1024-byte alignment of the shared-window address (swizzle atoms, TMA).
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const PrefillArgs& a = P.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int group = H / a.Hk;  // value heads per q, k head
    const int total = a.N * H;                  // every unit (bounds checked by api.cu)
    const int units = a.counter[1] * H;         // units with tokens, first in order
    const uint64_t wlim = a.wait_ns;

    Bars& B = *reinterpret_cast<Bars*>(sm + kOffBar);
    uint32_t* tmem_base_p = reinterpret_cast<uint32_t*>(sm + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);
    // the unit ring; only the producer (warp 0, lane 0) takes units from the counter
    const UnitRing ring{reinterpret_cast<volatile int*>(sm + kOffRing), a.counter, a.status, abort_flag, wlim,
                        warp == kWarpTma && lane == 0};
    float* sA = reinterpret_cast<float*>(sm + kOffA);
    uint8_t* sT1 = sm + kOffT1;
    uint8_t* sT2 = sm + kOffT2;
    uint8_t* sWT = sm + kOffWT;
    auto stage = [&](int s) { return sm + s * kStageBytes; };
    auto vecp = [&](int s) { return reinterpret_cast<float*>(sm + kOffVec + s * kVecBytes); };

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&B.full[s], 1);
            mbar_init(&B.conv_full[s], 2);
            mbar_init(&B.empty[s], 1);
            mbar_init(&B.vfree[s], 1);
            mbar_init(&B.gready[s], 1);
            mbar_init(&B.rk_ready[s], 1);
        }
        mbar_init(&B.g_full, 1);
        mbar_init(&B.g_free, 128);
        mbar_init(&B.t_ready, 1);
        mbar_init(&B.w_full, 1);
        mbar_init(&B.w_free, 128);
        mbar_init(&B.wt_ready, 1);
        mbar_init(&B.wt_free, 1);
        mbar_init(&B.u_full, 1);
        mbar_init(&B.ub_ready, 1);
        mbar_init(&B.s_full, 1);
        mbar_init(&B.sb_ready, 1);
        mbar_init(&B.sd_ready, 1);
        mbar_init(&B.o_full[0], 1);
        mbar_init(&B.o_full[1], 1);
        mbar_init(&B.o_free, 128);
        mbar_init(&B.drain_prep, 1);
        mbar_init(&B.drain_state, 1);
        fence_mbar_init();
        *abort_flag = 0;
        for (int e = 0; e < kRing; ++e) ring.slot[2 * e + 1] = -1;
    }
    if (warp == 0) tmem_alloc(tmem_base_p, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_p;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lane quarter

    // The first failed wait of the kernel records the timeout; every role then
    // leaves its loop.
    auto fail = [&]() {
        if (!*abort_flag) {
            *abort_flag = 1;
            set_status(a.status, kStatusTimeout);
        }
    };

    if (warp == kWarpTma && kConv) {
        // ================================== producer + conv of the q, k tiles
        // Lane 0 keeps the raw rows of chunk i and of the chunks after it whose
        // stage is already free in flight; then the warp convolves chunk i in
        // place (a lane per 16-byte column of the Q0, K0, Q1, K1 boxes) and hands
        // the stage to the Gram MMA. The producer walk (lane 0) takes the units;
        // the conv walk reads them from the ring like every other role.
        if (lane == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
        }
        const UnitRing cring{ring.slot, ring.counter, ring.status, ring.abort_flag, ring.wlim, false};
        Item pit, cit;
        bool phave = lane == 0 && item_first(a, units, pit);
        int pi = 0;                              // next chunk to load
        uint32_t issued = 0, issued_par = 0;     // last load per stage, for the drain
        const int bi = lane >> 3, c16 = lane & 7;  // box (Q0, K0, Q1, K1) and column
        const bool is_k = (bi & 1) != 0;
        const int off = 64 * (bi >> 1) + 8 * c16;  // channel within the head
        float2 w2[4][4], win[3][4];
        bool have = item_first(a, units, cit);
        for (int i = 0; have; ++i, have = item_next(a, units, cit, cring)) {
            const int s = i % kStages, k = i / kStages;
            bool ok = true;
            if (lane == 0) {
                while (phave) {
                    const int ps = pi % kStages, pk = pi / kStages;
                    if (pi <= i) {  // chunk i itself: wait for its stage
                        if (!mbar_wait_or_abort(&B.empty[ps], (pk & 1) ^ 1, abort_flag, wlim)) {
                            ok = false;
                            break;
                        }
                    } else if (pi >= i + kStages || !mbar_test_wait(&B.empty[ps], (pk & 1) ^ 1)) {
                        break;
                    }
                    issue_tiles(stage(ps), &B.full[ps], &map_q, &map_k, &map_v, pit.U.h / group, pit.U.h,
                                pit.c0);
                    issued |= 1u << ps;
                    issued_par = (issued_par & ~(1u << ps)) | ((uint32_t)(pk & 1) << ps);
                    ++pi;
                    phave = item_next(a, units, pit, ring);
                }
                if (ok) ok = mbar_wait_or_abort(&B.full[s], k & 1, abort_flag, wlim);
            }
            if (!__shfl_sync(0xffffffffu, (int)ok, 0)) {
                if (lane == 0) fail();
                break;
            }
            mbar_test_wait(&B.full[s], k & 1);  // each lane's own acquire of the landed rows
            const int hk = cit.U.h / group;
            const uint16_t* xp = static_cast<const uint16_t*>(is_k ? a.k : a.q) + hk * kD + off;
            if (cit.first) conv_unit_start(a, cit.U.n, cit.c0, (is_k ? a.Hk * kD : 0) + hk * kD + off, xp, w2, win);
            conv_column(stage(s) + bi * kBox, c16, w2, win);
            fence_proxy_async();  // the tiles are read by the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.conv_full[s]);
        }
        // Every copy lands before the CTA exits, also those nobody consumed.
        if (lane == 0)
            for (int s = 0; s < kStages; ++s)
                if ((issued >> s) & 1u) mbar_wait(&B.full[s], (issued_par >> s) & 1u, kDrainNs);
        __syncwarp();
    } else if (warp == kWarpTma) {
        // ============================================================ producer
        if (lane == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
            uint32_t issued = 0, issued_par = 0;  // last load per stage, for the drain
            Item it;
            bool have = item_first(a, units, it);
            for (int i = 0; have; ++i, have = item_next(a, units, it, ring)) {
                const int s = i % kStages, k = i / kStages;
                if (!mbar_wait_or_abort(&B.empty[s], (k & 1) ^ 1, abort_flag, wlim)) {
                    fail();
                    break;
                }
                issue_tiles(stage(s), &B.full[s], &map_q, &map_k, &map_v, it.U.h / group, it.U.h, it.c0);
                issued |= 1u << s;
                issued_par = (issued_par & ~(1u << s)) | ((uint32_t)(k & 1) << s);
            }
            // Every copy lands before the CTA exits, also those nobody consumed
            // because another role gave up (the abort can come after this loop).
            for (int s = 0; s < kStages; ++s)
                if ((issued >> s) & 1u) mbar_wait(&B.full[s], (issued_par >> s) & 1u, kDrainNs);
        }
        __syncwarp();
    } else if (warp == kWarpMmaPrep) {
        // =========================================== state-independent MMAs
        if (lane == 0) {
            bool ok = true;
            Item git, wit;
            bool have_g = item_first(a, units, git);
            bool have_w = have_g;
            wit = git;
            int ig = 0;
            // Gram of chunk ig: [Q;K] K^T -> R_G, once R_G has been read
            auto gram = [&]() -> bool {
                const int s = ig % kStages, k = ig / kStages;
                if (!mbar_wait_or_abort(kConv ? &B.conv_full[s] : &B.full[s], k & 1, abort_flag, wlim))
                    return false;
                if (ig > 0 && !mbar_wait_or_abort(&B.g_free, (ig - 1) & 1, abort_flag, wlim)) return false;
                tc_fence_after();
                const uint8_t* st = stage(s);
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t qoff = (kk < 4 ? kQb0 : kQb1) + 32 * (kk & 3);
                    const uint32_t koff = (kk < 4 ? kKb0 : kKb1) + 32 * (kk & 3);
                    mma_bf16(tmem + kRG, sw128_desc(smem_u32(st + qoff), 16, 1024),
                             sw128_desc(smem_u32(st + koff), 16, 1024), kIdescG, kk > 0);
                }
                mma_commit(&B.g_full);
                ++ig;
                return true;
            };
            if (have_g) {
                ok = gram();
                have_g = item_next(a, units, git, ring);
            }
            // The next chunk's Gram goes out before this chunk's W, so the Gram
            // epilogue of chunk i + 1 can follow the solve of chunk i at once. With
            // the fused conv it goes early only if that chunk is convolved already
            // (else it follows W, which must not wait for the next chunk's conv).
            for (int i = 0; ok && have_w; ++i, have_w = item_next(a, units, wit, ring)) {
                if (kConv && have_g && ig == i) {  // chunk i's own Gram, deferred
                    if (!(ok = gram())) break;
                    have_g = item_next(a, units, git, ring);
                }
                if (have_g && (!kConv || mbar_test_wait(&B.conv_full[ig % kStages], (ig / kStages) & 1))) {
                    if (!(ok = gram())) break;
                    have_g = item_next(a, units, git, ring);
                }
                // W^T = K^T T1 -> R_W ; U~^T = V^T T2 -> R_U[i & 1]
                const int s = i % kStages, b = i & 1;
                if (!mbar_wait_or_abort(&B.t_ready, i & 1, abort_flag, wlim) ||
                    (i >= 1 && !mbar_wait_or_abort(&B.w_free, (i - 1) & 1, abort_flag, wlim)) ||
                    (i >= 2 && !mbar_wait_or_abort(&B.o_full[b], ((i >> 1) - 1) & 1, abort_flag, wlim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* st = stage(s);
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + kRW, sw128_desc(smem_u32(st + kKb0 + 2048 * kk), kKb1 - kKb0, 1024),
                             sw128_desc(smem_u32(sT1 + 32 * kk), 16, 1024), kIdescW, kk > 0);
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + kRU + 64 * b, sw128_desc(smem_u32(st + kVb0 + 2048 * kk), kBox, 1024),
                             sw128_desc(smem_u32(sT2 + 32 * kk), 16, 1024), kIdescW, kk > 0);
                mma_commit(&B.w_full);
            }
            if (!ok) fail();
            mma_commit(&B.drain_prep);  // every MMA of this thread is done before TMEM is freed
            mbar_wait(&B.drain_prep, 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp == kWarpMmaState) {
        // ========================================================= state MMAs
        if (lane == 0) {
            bool ok = true;
            Item it;
            bool have = item_first(a, units, it);
            for (int i = 0; have; ++i, have = item_next(a, units, it, ring)) {
                const int s = i % kStages, b = i & 1;
                const uint8_t* st = stage(s);
                if (!mbar_wait_or_abort(&B.wt_ready, i & 1, abort_flag, wlim) ||
                    !mbar_wait_or_abort(&B.sb_ready, i & 1, abort_flag, wlim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // U^T += S^T (-W^T)   (A = S^T from R_SB)
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ta(tmem + kRU + 64 * b, tmem + kRSB + 8 * kk,
                                sw128_desc(smem_u32(sWT + 2048 * kk), 8192, 1024), kIdescSW, 1);
                mma_commit(&B.wt_free);
                mma_commit(&B.u_full);
                if (!mbar_wait_or_abort(&B.ub_ready, i & 1, abort_flag, wlim) ||
                    !mbar_wait_or_abort(&B.sd_ready, i & 1, abort_flag, wlim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // S^T += (U^T diag(kf / E)) K   (A = the scaled U^T copy in R_U[b]): the
                // chain's second MMA goes first
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ta(tmem + kRS, tmem + kRU + 64 * b + 32 + 8 * kk,
                                sw128_desc(smem_u32(st + kKb0 + 2048 * kk), kKb1 - kKb0, 1024), kIdescUK, 1);
                // O^T = S^T Q^T (Q~ when the decay does not factor), once the previous
                // chunk's output has left R_O. s_full is committed after it: the S
                // epilogue overwrites R_SB, which this MMA reads.
                if (i >= 1 && !mbar_wait_or_abort(&B.o_free, (i - 1) & 1, abort_flag, wlim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t qo = (kk < 4 ? kQb0 : kQb1) + 32 * (kk & 3);
                    mma_bf16_ta(tmem + kRO, tmem + kRSB + 8 * kk, sw128_desc(smem_u32(st + qo), 16, 1024),
                                kIdescSQ, kk > 0);
                }
                mma_commit(&B.s_full);
                // O^T += U^T P^T   (P' when the decay factors)
                const uint8_t* sP = sm + kOffP + s * kBox;
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ta(tmem + kRO, tmem + kRU + 64 * b + 8 * kk,
                                sw128_desc(smem_u32(sP + 32 * kk), 16, 1024), kIdescSQ, 1);
                mma_commit(&B.o_full[b]);
                mma_commit(&B.empty[s]);  // the chunk's tiles and P are no longer read
            }
            if (!ok) fail();
            mma_commit(&B.drain_state);
            mbar_wait(&B.drain_state, 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp == kWarpGate) {
        // ============================================================== gates
        // (and, with the fused conv, the conv of the v tiles: lanes 0-15, a
        // 16-byte column of the V0, V1 boxes each)
        float2 vw2[4][4], vwin[3][4];
        Item it;
        bool have = item_first(a, units, it);
        for (int i = 0; have; ++i, have = item_next(a, units, it, ring)) {
            const int s = i % kStages, k = i / kStages;
            const int L = it.L;
            // gates of rows 2*lane, 2*lane+1 (g = beta = 0 past the chunk's end)
            const int r = 2 * lane;
            float g0 = 0.f, g1 = 0.f, b0 = 0.f, b1 = 0.f;
            const float* gp = a.g + (it.c0 + r) * H + it.U.h;
            const float* bp = a.beta + (it.c0 + r) * H + it.U.h;
            if (r < L) { g0 = gp[0]; b0 = bp[0]; }
            if (r + 1 < L) { g1 = gp[H]; b1 = bp[H]; }
            const bool ok = lane != 0 || mbar_wait_or_abort(&B.vfree[s], (k & 1) ^ 1, abort_flag, wlim);
            if (__any_sync(0xffffffffu, !ok)) {
                if (lane == 0) fail();
                break;
            }
            // gamma = inclusive prefix sum of g (scan of the row-pair sums)
            const float pair = g0 + g1;
            float x = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            const float ga = x - pair + g0, gb = x;               // gamma_r, gamma_{r+1}
            const float gprev = __shfl_up_sync(0xffffffffu, gb, 1);
            const float gm1 = lane == 0 ? 0.f : gprev;             // gamma_{r-1}
            const float gL = __shfl_sync(0xffffffffu, gb, 31);     // gamma of the last row
            // The decay factors into e^{gamma_r} e^{-gamma_j} (both within fp32, with
            // room for the products P' U) while |gamma| stays below kFactorLimit;
            // gamma_{-1} = 0 is in range by definition.
            float mag = fmaxf(fabsf(ga), fabsf(gb));
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) mag = fmaxf(mag, __shfl_xor_sync(0xffffffffu, mag, o));
            float* vec = vecp(s);
            *reinterpret_cast<float2*>(vec + kVGam + r) = make_float2(ga, gb);
            *reinterpret_cast<float2*>(vec + kVBet + r) = make_float2(b0, b1);
            *reinterpret_cast<float2*>(vec + kVCf + r) = make_float2(ex2(-ga * kLog2e), ex2(-gb * kLog2e));
            const float2 er = make_float2(expf(ga), expf(gb));
            *reinterpret_cast<float2*>(vec + kVEr + r) = er;
            *reinterpret_cast<float2*>(vec + kVEa + r) = kUndecayed ? make_float2(expf(gm1), er.x) : er;
            *reinterpret_cast<float2*>(vec + kVEgl + r) =
                make_float2(r < L ? expf(gL - ga) : 0.f, r + 1 < L ? expf(gL - gb) : 0.f);
            if (lane == 0) {
                vec[kVFlag] = mag < kFactorLimit ? 1.f : 0.f;
                vec[kVEL] = expf(gL);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.gready[s]);
            if constexpr (kConv) {
                const bool okc = lane != 0 || mbar_wait_or_abort(&B.full[s], k & 1, abort_flag, wlim);
                if (!__shfl_sync(0xffffffffu, (int)okc, 0)) {
                    if (lane == 0) fail();
                    break;
                }
                mbar_test_wait(&B.full[s], k & 1);
                if (a.conv_v && lane < 16) {
                    const int off = 64 * (lane >> 3) + 8 * (lane & 7);
                    const uint16_t* xp = static_cast<const uint16_t*>(a.v) + it.U.h * kD + off;
                    if (it.first) conv_unit_start(a, it.U.n, it.c0, 2 * a.Hk * kD + it.U.h * kD + off, xp, vw2, vwin);
                    conv_column(stage(s) + (4 + (lane >> 3)) * kBox, lane & 7, vw2, vwin);
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.conv_full[s]);
            }
        }
    } else if (warp < kWg2) {
        // ===================== WG1: Gram epilogue (P, A, k norms), solve, T export
        const int wq = warp & 3;           // TMEM lane quarter; diagonal block of the solve
        const int row = 32 * wq + lane;    // Gram row: q rows 0-63, k rows 64-127
        const int r = row & 63;
        const int rb = wq & 1;             // 32-row block of r
        const bool is_p = row < 64;
        const int gtid = tid - 32 * kWg1;  // 0..127
        Item it;
        bool have = item_first(a, units, it);
        for (int i = 0; have; ++i, have = item_next(a, units, it, ring)) {
            const int s = i % kStages, k = i / kStages;
            const int L = it.L;
            float* vec = vecp(s);
            {
                const bool ok = !(gtid == 0) || (mbar_wait_or_abort(&B.gready[s], k & 1, abort_flag, wlim) &&
                                mbar_wait_or_abort(&B.g_full, i & 1, abort_flag, wlim));
                if (group_any(kBarWg1, 128, !ok)) {
                    if (gtid == 0) fail();
                    break;
                }
            }
            tc_fence_after();
            // k norm factors from the diagonal of K K^T (column r of k row r), and
            // kf = e^{gamma_L - gamma} rk, the row factors of K in the state update
            if (!is_p) {
                float x[32];
                tmem_ld32(tmem + lane_off + kRG + 32 * rb, x);
                tmem_wait_ld();
                float d2 = 0.f;
#pragma unroll
                for (int e = 0; e < 32; ++e) d2 = (e == lane) ? x[e] : d2;
                float f = 0.f;
                if (r < L) f = a.qk_l2norm ? rsqrtf(d2 + a.eps) : 1.f;
                vec[kVRk + r] = f;
                vec[kVKf + r] = f * vec[kVEgl + r];
            }
            group_sync(kBarWg1, 128);
            if (gtid == 0) mbar_arrive(&B.rk_ready[s]);
            // P row r (q rows): P[r][j] = e^{gamma_r - gamma_j} rk_j (q_r . k_j), j <= r, or
            // with the factored decay P'[r][j] = e^{-gamma_j} rk_j (q_r . k_j).
            // A row r (k rows): A[r][j] = beta_r rk_r e^{gamma'_r - gamma_j} rk_j (k_r . k_j),
            // j < r; A's entries on and above the diagonal are never read.
            {
                const float* gam = vec + kVGam;
                const bool factored = vec[kVFlag] != 0.f;
                const float gr = (kUndecayed && !is_p) ? (r > 0 ? gam[r - 1] : 0.f) : gam[r];
                const float fr = is_p ? 1.f : vec[kVBet + r] * vec[kVRk + r];
                const float frf = is_p ? 1.f : fr * vec[kVEa + r];
                uint8_t* sP = sm + kOffP + s * kBox;
                // 16-column steps up to the end of the row's own 32-column block
#pragma unroll 1
                for (int j0 = 0; j0 < 32 * (rb + 1); j0 += 16) {
                    float x[16];
                    tmem_ld16(tmem + lane_off + kRG + j0, x);
                    tmem_wait_ld();
                    const float4* rk4 = reinterpret_cast<const float4*>(vec + kVRk + j0);
                    if (factored) {
                        const float4* cf4 = reinterpret_cast<const float4*>(vec + kVCf + j0);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 c = cf4[q4], kk = rk4[q4];
                            const float2 c01 = __fmul2_rn(make_float2(c.x, c.y), make_float2(kk.x, kk.y));
                            const float2 c23 = __fmul2_rn(make_float2(c.z, c.w), make_float2(kk.z, kk.w));
                            const float2 v01 = __fmul2_rn(__fmul2_rn(c01, make_float2(frf, frf)),
                                                          make_float2(x[4 * q4], x[4 * q4 + 1]));
                            const float2 v23 = __fmul2_rn(__fmul2_rn(c23, make_float2(frf, frf)),
                                                          make_float2(x[4 * q4 + 2], x[4 * q4 + 3]));
                            x[4 * q4] = v01.x; x[4 * q4 + 1] = v01.y; x[4 * q4 + 2] = v23.x; x[4 * q4 + 3] = v23.y;
                        }
                    } else {
                        const float4* g4 = reinterpret_cast<const float4*>(gam + j0);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 gj = g4[q4], kk = rk4[q4];
                            x[4 * q4] *= __expf(fminf(gr - gj.x, 0.f)) * (fr * kk.x);
                            x[4 * q4 + 1] *= __expf(fminf(gr - gj.y, 0.f)) * (fr * kk.y);
                            x[4 * q4 + 2] *= __expf(fminf(gr - gj.z, 0.f)) * (fr * kk.z);
                            x[4 * q4 + 3] *= __expf(fminf(gr - gj.w, 0.f)) * (fr * kk.w);
                        }
                    }
                    if (is_p) {
                        uint32_t w[8];
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            w[c] = pack_bf16(j0 + 2 * c <= r ? x[2 * c] : 0.f, j0 + 2 * c + 1 <= r ? x[2 * c + 1] : 0.f);
                        *reinterpret_cast<uint4*>(sP + sw128_off(r, j0 >> 3)) = make_uint4(w[0], w[1], w[2], w[3]);
                        *reinterpret_cast<uint4*>(sP + sw128_off(r, (j0 >> 3) + 1)) = make_uint4(w[4], w[5], w[6], w[7]);
                    } else {
                        float4* Ar = reinterpret_cast<float4*>(sA + r * kLdA + j0);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            Ar[q4] = make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
                    }
                }
                if (is_p && rb == 0) {  // P's block above the diagonal
#pragma unroll 1
                    for (int c = 4; c < 8; ++c) *reinterpret_cast<uint4*>(sP + sw128_off(r, c)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            tc_fence_before();
            mbar_arrive(&B.g_free);  // R_G read: the next chunk's Gram may go
            group_sync(kBarWg1, 128);

            // ---- solve T = (I + A)^-1 in place. 16 x 16 blocks (bi, bj) sit at rows
            // 16 bi, columns 16 bj; T's blocks above the diagonal are scratch.
            auto blk = [&](int bi, int bj) { return sA + 16 * bi * kLdA + 16 * bj; };
            // 1. Diagonal blocks: warp wq, lane c < 16 solves column c of block wq by
            //    forward substitution in registers (once x[m] is final,
            //    x[r] -= A[r][m] x[m] for r > m) and writes it over A.
            {
                const int o = 16 * wq;
                const int c = lane & 15;
                float xv[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) xv[rr] = (rr == c) ? 1.f : 0.f;
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
                    float4 av[16];
#pragma unroll
                    for (int rr = 4 * m4 + 1; rr < 16; ++rr)
                        av[rr] = *reinterpret_cast<const float4*>(sA + (o + rr) * kLdA + o + 4 * m4);
#pragma unroll
                    for (int mm = 0; mm < 4; ++mm) {
                        const int m = 4 * m4 + mm;
                        const float xm = xv[m];
#pragma unroll
                        for (int rr = m + 1; rr < 16; ++rr) {
                            const float am = mm == 0 ? av[rr].x : mm == 1 ? av[rr].y : mm == 2 ? av[rr].z : av[rr].w;
                            xv[rr] = fmaf(-am, xm, xv[rr]);
                        }
                    }
                }
                __syncwarp();
                if (lane < 16) {
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) sA[(o + rr) * kLdA + o + c] = xv[rr];
                }
            }
            group_sync(kBarWg1, 128);
            // 2a. T10 = -T11 (A10 T00) and T32 = -T33 (A32 T22) with scratch blocks (0,1)
            //     and (2,3); meanwhile Y'_{a,1} = A_{2+a,1} T11 into (a,3).
            if (wq < 2) {
                const int p = 2 * wq;
                float* Y = blk(p, p + 1);
                mma_tf32_16x16(Y, blk(p + 1, p), blk(p, p), 1.f);
                __syncwarp();
                mma_tf32_16x16(blk(p + 1, p), blk(p + 1, p + 1), Y, -1.f);
            } else {
                const int aa = wq - 2;
                mma_tf32_16x16(blk(aa, 3), blk(2 + aa, 1), blk(1, 1), 1.f);
            }
            group_sync(kBarWg1, 128);
            // 2b. Y'_{a,0} = A_{2+a,0} T00 + A_{2+a,1} T10 into (a,2), one 16 x 8 half
            //     per warp (a = wq >> 1, half = wq & 1).
            {
                const int aa = wq >> 1, nh = wq & 1;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tf32_16x8(d, blk(2 + aa, 0), blk(0, 0) + 8 * nh, 4);
                store_acc_16x8(blk(aa, 2) + 8 * nh, d, 1.f);
            }
            group_sync(kBarWg1, 128);
            // 2c. T_{2+a,b} = -sum_{m<=a} T_{2+a,2+m} Y'_{m,b}, over A_{2+a,b}
            //     (warp: a = wq >> 1, b = wq & 1).
            {
                const int aa = wq >> 1, bb = wq & 1;
                float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tf32_16x8(d0, blk(2 + aa, 2), blk(0, 2 + bb), 2 * (aa + 1));
                mma_tf32_16x8(d1, blk(2 + aa, 2), blk(0, 2 + bb) + 8, 2 * (aa + 1));
                store_acc_16x8(blk(2 + aa, bb), d0, -1.f);
                store_acc_16x8(blk(2 + aa, bb) + 8, d1, -1.f);
            }
            // T1 and T2 are read by the previous chunk's W MMA until it completes
            {
                const bool ok = !(gtid == 0) || (i == 0 || mbar_wait_or_abort(&B.w_full, (i - 1) & 1, abort_flag, wlim));
                if (group_any(kBarWg1, 128, !ok)) {  // also orders 2c before the export
                    if (gtid == 0) fail();
                    break;
                }
            }
            // 3. Export T1[r][j] = T[r][j] beta_j e^{gamma'_j} rk_j and T2[r][j] = T[r][j] beta_j
            //    as bf16, the K-major B operands of W^T = K^T T1 and U~^T = V^T T2 (T is
            //    lower triangular with a unit diagonal; its upper part is scratch).
            {
                const int rr = gtid & 63, hf = gtid >> 6;
                const float* Trow = sA + rr * kLdA;
#pragma unroll 1
                for (int j = 32 * hf; j < 32 * hf + 32; j += 4) {
                    // T's upper part holds finite scratch: read it and select zeros
                    float4 t = *reinterpret_cast<const float4*>(Trow + j);
                    t.x = j <= rr ? t.x : 0.f;
                    t.y = j + 1 <= rr ? t.y : 0.f;
                    t.z = j + 2 <= rr ? t.z : 0.f;
                    t.w = j + 3 <= rr ? t.w : 0.f;
                    const float4 bb = *reinterpret_cast<const float4*>(vec + kVBet + j);
                    const float4 ee = *reinterpret_cast<const float4*>(vec + kVEa + j);
                    const float4 kk = *reinterpret_cast<const float4*>(vec + kVRk + j);
                    const float2 u01 = __fmul2_rn(make_float2(t.x, t.y), make_float2(bb.x, bb.y));
                    const float2 u23 = __fmul2_rn(make_float2(t.z, t.w), make_float2(bb.z, bb.w));
                    const float2 t01 = __fmul2_rn(u01, __fmul2_rn(make_float2(ee.x, ee.y), make_float2(kk.x, kk.y)));
                    const float2 t23 = __fmul2_rn(u23, __fmul2_rn(make_float2(ee.z, ee.w), make_float2(kk.z, kk.w)));
                    const uint32_t off = sw128_off(rr, j >> 3) + (j & 7) * 2;
                    *reinterpret_cast<uint2*>(sT1 + off) = make_uint2(pack_bf16(t01.x, t01.y), pack_bf16(t23.x, t23.y));
                    *reinterpret_cast<uint2*>(sT2 + off) = make_uint2(pack_bf16(u01.x, u01.y), pack_bf16(u23.x, u23.y));
                }
            }
            fence_proxy_async();  // P, T1, T2 are read by the tensor cores
            group_sync(kBarWg1, 128);
            if (gtid == 0) mbar_arrive(&B.t_ready);
        }
    } else if (warp < kWg3) {
        // ===== WG2: -W^T epilogue and q norms of chunk i, then the output of chunk
        // i - 1 (the order in which they become ready)
        const int row = 32 * (warp & 3) + lane;     // TMEM lane: dk index; dv index of O
        const int gtid = tid - 32 * kWg2;
        const int qr = gtid >> 1, qbox = gtid & 1;  // q row and 64-column box of this thread
        Item it, prev;
        bool have = item_first(a, units, it), have_prev = false;
        for (int i = 0; have || have_prev; ++i) {
            if (have) {
                const int s = i % kStages, k = i / kStages;
                const int L = it.L;
                float* vec = vecp(s);
                uint8_t* qtile = stage(s) + (qbox ? kQb1 : kQb0);
                {
                    const bool ok = !(gtid == 0) || mbar_wait_or_abort(&B.w_full, i & 1, abort_flag, wlim);
                    if (group_any(kBarWg2, 128, !ok)) {
                        if (gtid == 0) fail();
                        break;
                    }
                }
                tc_fence_after();
                float x0[32], x1[32];
                tmem_ld32(tmem + lane_off + kRW, x0);
                tmem_ld32(tmem + lane_off + kRW + 32, x1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&B.w_free);
                {
                    // -W^T is read by the previous chunk's MMA U until it completes
                    const bool ok = !(gtid == 0) ||
                                    ((i == 0 || mbar_wait_or_abort(&B.wt_free, (i - 1) & 1, abort_flag, wlim)) &&
                                     mbar_wait_or_abort(&B.gready[s], k & 1, abort_flag, wlim));
                    if (group_any(kBarWg2, 128, !ok)) {
                        if (gtid == 0) fail();
                        break;
                    }
                }
                store_half_row(sWT, row, 0, x0, -1.f);
                store_half_row(sWT, row, 1, x1, -1.f);
                // Without the factored decay MMA O reads Q~ = diag(e^gamma) Q: scale in
                // place (the Gram MMA has read the raw Q). The q norm comes from the raw
                // values.
                const bool factored = vec[kVFlag] != 0.f;
                float ss = 0.f;
                if (!factored) ss = scale_row_ss(qtile, qr, vec[kVEr + qr]);
                fence_proxy_async();
                group_sync(kBarWg2, 128);
                if (gtid == 0) mbar_arrive(&B.wt_ready);
                if (factored) ss = sumsq_row(qtile, qr);
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                if (qbox == 0) {
                    float f = 0.f;
                    if (qr < L) f = a.qk_l2norm ? a.scale * rsqrtf(ss + a.eps) : a.scale;
                    reinterpret_cast<float*>(sm + kOffOf)[64 * (i & 1) + qr] = factored ? f * vec[kVEr + qr] : f;
                }
                // the output factors are read by every thread of the group below
            }
            if (have_prev) {
                // ---- O of chunk i - 1: column `row` of O^T times the output row factors
                // (q norm, and the decay when it factors), stored straight to HBM (for
                // each token the 128 threads write its 256 contiguous bytes).
                const int ip = i - 1, b = ip & 1;
                const int L = prev.L;
                {
                    const bool ok = !(gtid == 0) || mbar_wait_or_abort(&B.o_full[b], (ip >> 1) & 1, abort_flag, wlim);
                    if (group_any(kBarWg2, 128, !ok)) {
                        if (gtid == 0) fail();
                        break;
                    }
                }
                tc_fence_after();
                const float* of = reinterpret_cast<const float*>(sm + kOffOf) + 64 * (ip & 1);
                uint16_t* op = static_cast<uint16_t*>(a.o) + (prev.c0 * H + prev.U.h) * kD + row;
                const int ts = H * kD;  // elements between tokens
                float x0[32], x1[32];
                tmem_ld32(tmem + lane_off + kRO, x0);
                tmem_ld32(tmem + lane_off + kRO + 32, x1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&B.o_free);  // R_O read: the next chunk's MMA O may go
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // 16 tokens at a time
                    const float* x = (q < 2 ? x0 : x1) + 16 * (q & 1);
                    const float4* of4 = reinterpret_cast<const float4*>(of + 16 * q);
                    uint16_t y[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 f = of4[q4];
                        y[4 * q4] = f32_to_bf16(x[4 * q4] * f.x);
                        y[4 * q4 + 1] = f32_to_bf16(x[4 * q4 + 1] * f.y);
                        y[4 * q4 + 2] = f32_to_bf16(x[4 * q4 + 2] * f.z);
                        y[4 * q4 + 3] = f32_to_bf16(x[4 * q4 + 3] * f.w);
                    }
                    if (16 * q + 16 <= L) {  // uniform: no per-element guard on full steps
#pragma unroll
                        for (int e = 0; e < 16; ++e) op[e * ts] = y[e];
                    } else {  // the chunk's last tokens (a partial chunk only)
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (16 * q + e < L) op[e * ts] = y[e];
                    }
                    op += 16 * ts;
                }
            }
            group_sync(kBarWg2, 128);  // the output factors of chunk i are written
            have_prev = have;
            if (have) {
                prev = it;
                have = item_next(a, units, it, ring);
            }
        }
    } else {
        // ========================================== WG3: the state epilogues
        const int j = tid - 32 * kWg3;  // 0..127 = TMEM lane = dv index
        // Units with no tokens on this CTA's stride still need hT = h0.
        for (int e = blockIdx.x; e < total; e += gridDim.x) {
            Unit U;
            if (!load_unit_checked(a, e, U)) {
                if (j == 0) set_status(a.status, kStatusBadSeqlens);
                continue;
            }
            if (U.end > U.start || !a.hT) continue;
            const int64_t base = ((int64_t)U.n * H + U.h) * kD * kD;
            for (int x = j; x < kD * kD; x += 128) a.hT[base + x] = a.h0 ? a.h0[base + x] : 0.f;
        }
        // R_S holds S^T / E: the decay of a chunk multiplies E instead of R_S (its
        // update is scaled by 1 / E through the U^T copy of MMA S), and R_S is
        // rewritten with E folded in only when E would fall below kRescale.
        float E = 1.f;
        Item it;
        bool have = item_first(a, units, it);
        for (int i = 0; have; ++i, have = item_next(a, units, it, ring)) {
            const int s = i % kStages, k = i / kStages, b = i & 1;
            const int64_t sbase = ((int64_t)it.U.n * H + it.U.h) * kD * kD;
            if (it.first) {
                // Initial state: S^T as the bf16 A operand in R_SB (thread = dv lane j),
                // and in R_S either as is (E = e^{gamma_L}) or pre-decayed (E = 1).
                {
                    const bool ok = !(j == 0) || mbar_wait_or_abort(&B.gready[s], k & 1, abort_flag, wlim);
                    if (group_any(kBarWg3, 128, !ok)) {
                        if (j == 0) fail();
                        break;
                    }
                }
                const float eL = vecp(s)[kVEL];
                const bool fold = eL >= kRescale;
                E = fold ? eL : 1.f;
                const float* h0p = a.h0 ? a.h0 + sbase + j : nullptr;  // column j of S
#pragma unroll 1
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
#pragma unroll
                    for (int c = 0; c < 16; ++c) w[c] = pack_bf16(v[2 * c], v[2 * c + 1]);
                    tmem_st16(tmem + lane_off + kRSB + 16 * cc, w);
                    if (!fold) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] *= eL;
                    }
                    tmem_st32(tmem + lane_off + kRS + 32 * cc, v);
                }
                tmem_wait_st();
                tc_fence_before();
                group_sync(kBarWg3, 128);
                if (j == 0) {
                    mbar_arrive(&B.sb_ready);
                    mbar_arrive(&B.sd_ready);
                }
            }
            // ---- U^T (64 tokens of dv row j) as packed bf16 in columns 0-31 of R_U[b]
            // (A operand of MMA O2) and U^T diag(kf / E) in columns 32-63 (A operand of
            // MMA S: the state update's K~ = diag(kf) K with K read raw, over E)
            {
                const bool ok = !(j == 0) || (mbar_wait_or_abort(&B.u_full, i & 1, abort_flag, wlim) &&
                                              mbar_wait_or_abort(&B.rk_ready[s], k & 1, abort_flag, wlim));
                if (group_any(kBarWg3, 128, !ok)) {
                    if (j == 0) fail();
                    break;
                }
            }
            tc_fence_after();
            {
                float x0[32], x1[32];
                tmem_ld32(tmem + lane_off + kRU + 64 * b, x0);
                tmem_ld32(tmem + lane_off + kRU + 64 * b + 32, x1);
                tmem_wait_ld();
                {
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) w[c] = pack_bf16(x0[2 * c], x0[2 * c + 1]);
                    tmem_st16(tmem + lane_off + kRU + 64 * b, w);
                }
                {
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) w[c] = pack_bf16(x1[2 * c], x1[2 * c + 1]);
                    tmem_st16(tmem + lane_off + kRU + 64 * b + 16, w);
                }
                const float4* kf4 = reinterpret_cast<const float4*>(vecp(s) + kVKf);
                const float2 inv = make_float2(1.f / E, 1.f / E);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float(&x)[32] = hf ? x1 : x0;
                    uint32_t w[16];
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 f = kf4[8 * hf + q4];
                        const float2 f01 = __fmul2_rn(make_float2(f.x, f.y), inv);
                        const float2 f23 = __fmul2_rn(make_float2(f.z, f.w), inv);
                        const float2 v01 = __fmul2_rn(make_float2(x[4 * q4], x[4 * q4 + 1]), f01);
                        const float2 v23 = __fmul2_rn(make_float2(x[4 * q4 + 2], x[4 * q4 + 3]), f23);
                        w[2 * q4] = pack_bf16(v01.x, v01.y);
                        w[2 * q4 + 1] = pack_bf16(v23.x, v23.y);
                    }
                    tmem_st16(tmem + lane_off + kRU + 64 * b + 32 + 16 * hf, w);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            group_sync(kBarWg3, 128);
            if (j == 0) {
                mbar_arrive(&B.ub_ready);
                mbar_arrive(&B.vfree[s]);  // the chunk's gate vectors have been read
            }
            // ---- new state S = E R_S: bf16 S^T for the next chunk's MMAs (the chain),
            // and, when E times the next chunk's decay would fall below kRescale, R_S
            // rewritten pre-decayed with E = 1; the final state at the end of a sequence.
            {
                const bool ok = !(j == 0) || mbar_wait_or_abort(&B.s_full, i & 1, abort_flag, wlim);
                if (group_any(kBarWg3, 128, !ok)) {
                    if (j == 0) fail();
                    break;
                }
            }
            tc_fence_after();
            if (!it.last) {
                // the next chunk's decay (its gates are in the next stage's vector block)
                const int s1 = (i + 1) % kStages, k1 = (i + 1) / kStages;
                {
                    const bool ok = !(j == 0) || mbar_wait_or_abort(&B.gready[s1], k1 & 1, abort_flag, wlim);
                    if (group_any(kBarWg3, 128, !ok)) {
                        if (j == 0) fail();
                        break;
                    }
                }
                const float prod = E * vecp(s1)[kVEL];
                const bool fold = prod >= kRescale;
                const float2 e2 = make_float2(E, E), p2 = make_float2(prod, prod);
#pragma unroll 1
                for (int cc = 0; cc < 4; cc += 2) {  // two loads in flight per wait
                    float v[32], u[32];
                    tmem_ld32(tmem + lane_off + kRS + 32 * cc, v);
                    tmem_ld32(tmem + lane_off + kRS + 32 * cc + 32, u);
                    tmem_wait_ld();
                    uint32_t w[32];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float2 a2 = __fmul2_rn(make_float2(v[2 * c], v[2 * c + 1]), e2);
                        const float2 b2 = __fmul2_rn(make_float2(u[2 * c], u[2 * c + 1]), e2);
                        w[c] = pack_bf16(a2.x, a2.y);
                        w[16 + c] = pack_bf16(b2.x, b2.y);
                    }
                    tmem_st32(tmem + lane_off + kRSB + 16 * cc, w);
                    if (!fold) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 a2 = __fmul2_rn(make_float2(v[e], v[e + 1]), p2);
                            const float2 b2 = __fmul2_rn(make_float2(u[e], u[e + 1]), p2);
                            v[e] = a2.x; v[e + 1] = a2.y; u[e] = b2.x; u[e + 1] = b2.y;
                        }
                        tmem_st32(tmem + lane_off + kRS + 32 * cc, v);
                        tmem_st32(tmem + lane_off + kRS + 32 * cc + 32, u);
                    }
                }
                tmem_wait_st();
                E = fold ? prod : 1.f;
                tc_fence_before();
                group_sync(kBarWg3, 128);
                if (j == 0) {
                    mbar_arrive(&B.sb_ready);
                    mbar_arrive(&B.sd_ready);
                }
            } else if (a.hT) {
                float* hTp = a.hT + sbase + j;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    float v[32];
                    tmem_ld32(tmem + lane_off + kRS + 32 * cc, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) hTp[(32 * cc + e) * kD] = E * v[e];
                }
            }
        }
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
// (feature, head, token); boxes of 64 features x 1 head x 64 tokens with the
// 128-byte swizzle the MMA descriptors expect, zero fill past T_tot.
bool make_map(CUtensorMap* m, const void* ptr, int H, int64_t T, int64_t ld) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)ld * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(const PrefillArgs& a) {
    return a.is_bf16 && a.dk == kD && a.dv == kD && a.chunk == kC && a.T_tot > 0 &&
           a.T_tot < ((int64_t)1 << 31) && encode_fn() != nullptr;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s, bool pdl) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.Hk, a.T_tot, a.ld_q) || !make_map(&mk, a.k, a.Hk, a.T_tot, a.ld_k) ||
        !make_map(&mv, a.v, a.H, a.T_tot, a.ld_v))
        return cudaErrorInvalidValue;
    auto kernel = a.conv_w ? (a.undecayed ? prefill_tc_kernel<true, true> : prefill_tc_kernel<false, true>)
                           : (a.undecayed ? prefill_tc_kernel<true, false> : prefill_tc_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t units = (int64_t)a.N * a.H;
    const int grid = (int)(units < sms ? units : sms);
    TcParams p{a};
    if (pdl) return launch_pdl(kernel, dim3(grid), dim3(kThreads), kSmemAlloc, s, p, mq, mk, mv);
    kernel<<<grid, kThreads, kSmemAlloc, s>>>(p, mq, mk, mv);
    return cudaGetLastError();
}

}  // namespace gdn
