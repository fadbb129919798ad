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
//   [Q;K] K^T          -> TMEM  R_A   (128 lanes = 64 q rows + 64 k rows, 64 cols)
//   W^T  = K^T T1^T    -> TMEM  R_W   (lanes = dk, cols = tokens)
//   U~^T = V^T T2^T    -> TMEM  R_U   (lanes = dv, cols = tokens)
//   U^T  = U~^T + S^T (-W^T)         (accumulated in R_U)
//   O^T  = S^T Q~^T + U^T P^T        (R_O, lanes = dv, cols = tokens)
//   S^T <- e^{gamma_L} S^T + U^T K~  (R_S, fp32 master state, lanes = dv, cols = dk)
// The algorithmic 11.5 MFLOP per (chunk, head) are exactly the MMAs issued.
// The L2 norms, scale and decays are applied as per-row factors in the
// epilogues, so the MMAs read the raw bf16 input tiles that TMA brings in
// (128-byte swizzle). The solve for T runs on CUDA cores in fp32.
//
// This version runs the phases of a chunk in lock-step across one 256-thread
// CTA per SM (two warps per TMEM lane quarter, each taking half of the
// columns); thread 0 issues TMA and MMAs. The
// next chunk's tiles are prefetched by TMA during the current chunk.
// Every wait is bounded: on timeout the kernel records GDN timeout status,
// drains its TMA copies, frees TMEM and returns.
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
constexpr int kThreads = 256;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t kBox = 8192;                   // 64 rows x 128 B (64 bf16)
constexpr uint32_t kQb0 = 0, kKb0 = kBox, kQb1 = 2 * kBox, kKb1 = 3 * kBox;
constexpr uint32_t kVb0 = 4 * kBox, kVb1 = 5 * kBox;
constexpr uint32_t kStageBytes = 6 * kBox;        // 48 KB: Q, K, V tiles
constexpr uint32_t kOffSA = 2 * kStageBytes;      // S^T bf16, 2 x [128 dv][64 dk] K-major
constexpr uint32_t kOffWT = kOffSA + 32768;       // -W^T bf16 [128 dk][64 tok] MN-major
constexpr uint32_t kOffUT = kOffWT + 16384;       // U^T bf16 [128 dv][64 tok] K-major
constexpr uint32_t kOffP = kOffUT + 16384;        // P bf16 [64 r][64 j] K-major
constexpr uint32_t kOffT1 = kOffP + 8192;         // T1^T bf16 [64 m][64 r] MN-major
constexpr uint32_t kOffT2 = kOffT1 + 8192;        // T2^T bf16
constexpr int kLdA = 68;                          // padded fp32 row stride (272 B)
constexpr uint32_t kOffA = kOffT2 + 8192;         // A fp32 [64][kLdA] (later also Y)
constexpr uint32_t kOffTf = kOffA + 64 * kLdA * 4;  // T fp32 [64][kLdA]
constexpr uint32_t kOffVec = kOffTf + 64 * kLdA * 4;  // gamma, beta, rq, rk: 4 x 64 fp32
constexpr uint32_t kOffBar = kOffVec + 1024;      // mbarriers
constexpr uint32_t kOffMisc = kOffBar + 64;       // tmem base, abort flag, scan carry
constexpr uint32_t kSmemBytes = kOffMisc + 64;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment

// TMEM columns (fp32, 128 lanes).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kRS = 0, kRU = 128, kRO = 192, kRA = 256, kRW = 320;

constexpr uint32_t kIdescA = idesc_bf16(128, 64, 0, 0);    // [Q;K] K^T
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
__device__ __forceinline__ void unpack_bf16(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

// Write 64 fp32 values as one 128-byte bf16 row of a 128B-swizzled tile.
__device__ __forceinline__ void store_row64(uint8_t* tile, int row, const float (&v)[64]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = pack_bf16(v[8 * c + 0], v[8 * c + 1]);
        u.y = pack_bf16(v[8 * c + 2], v[8 * c + 3]);
        u.z = pack_bf16(v[8 * c + 4], v[8 * c + 5]);
        u.w = pack_bf16(v[8 * c + 6], v[8 * c + 7]);
        *reinterpret_cast<uint4*>(tile + sw128_off(row, c)) = u;
    }
}

// Same, with every value multiplied by f.
__device__ __forceinline__ void store_row64_scaled(uint8_t* tile, int row, const float (&v)[64],
                                                   float f) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = pack_bf16(v[8 * c + 0] * f, v[8 * c + 1] * f);
        u.y = pack_bf16(v[8 * c + 2] * f, v[8 * c + 3] * f);
        u.z = pack_bf16(v[8 * c + 4] * f, v[8 * c + 5] * f);
        u.w = pack_bf16(v[8 * c + 6] * f, v[8 * c + 7] * f);
        *reinterpret_cast<uint4*>(tile + sw128_off(row, c)) = u;
    }
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

// Sum of squares of a 128-byte bf16 row (order of chunks irrelevant).
__device__ __forceinline__ float row_sumsq(const uint8_t* tile, int row) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile + sw128_off(row, c));
        float a, b;
        unpack_bf16(u.x, a, b); s = fmaf(a, a, s); s = fmaf(b, b, s);
        unpack_bf16(u.y, a, b); s = fmaf(a, a, s); s = fmaf(b, b, s);
        unpack_bf16(u.z, a, b); s = fmaf(a, a, s); s = fmaf(b, b, s);
        unpack_bf16(u.w, a, b); s = fmaf(a, a, s); s = fmaf(b, b, s);
    }
    return s;
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
                                            const CUtensorMap* mk, const CUtensorMap* mv, int h,
                                            int64_t c0) {
    mbar_arrive_expect_tx(bar, kStageBytes);
    const int t = (int)c0;
    tma_load_3d(stage + kQb0, mq, bar, 0, h, t);
    tma_load_3d(stage + kQb1, mq, bar, 64, h, t);
    tma_load_3d(stage + kKb0, mk, bar, 0, h, t);
    tma_load_3d(stage + kKb1, mk, bar, 64, h, t);
    tma_load_3d(stage + kVb0, mv, bar, 0, h, t);
    tma_load_3d(stage + kVb1, mv, bar, 64, h, t);
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ TcParams P, const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the shared-window address (swizzle atoms, TMA).
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const PrefillArgs& a = P.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Two warps share each TMEM lane quarter and split the columns in halves.
    const int quarter = warp & 3, half = warp >> 2;
    const int row = 32 * quarter + lane;  // TMEM lane owned by this thread
    const int H = a.H;
    const int64_t total = (int64_t)a.N * H;

    uint8_t* sSA = sm + kOffSA;
    uint8_t* sWT = sm + kOffWT;
    uint8_t* sUT = sm + kOffUT;
    uint8_t* sP = sm + kOffP;
    uint8_t* sT1 = sm + kOffT1;
    uint8_t* sT2 = sm + kOffT2;
    float* sA = reinterpret_cast<float*>(sm + kOffA);
    float* sT = reinterpret_cast<float*>(sm + kOffTf);
    float* gam = reinterpret_cast<float*>(sm + kOffVec);
    float* bet = gam + 64;
    float* rq = gam + 128;
    float* rk = gam + 192;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kOffBar);  // [2]
    uint64_t* mbar = full + 2;
    uint32_t* tmem_base_p = reinterpret_cast<uint32_t*>(sm + kOffMisc);
    int* abort_flag = reinterpret_cast<int*>(sm + kOffMisc + 4);
    float* carry = reinterpret_cast<float*>(sm + kOffMisc + 8);

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(mbar, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
    }
    if (warp == 0) tmem_alloc(tmem_base_p, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_p;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;  // this warp's TMEM lane quarter

    uint32_t full_phase = 0;  // bit s: expected parity of full[s]
    uint32_t mma_phase = 0;
    int cur = 0;              // stage of the chunk being processed
    uint32_t inflight = 0;    // bit s: TMA issued into stage s, not yet consumed
    auto stage = [&](int i) { return sm + i * kStageBytes; };
    bool aborted = false;

    // Bounded wait by every thread; all threads agree on the outcome.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait(bar, parity, kWaitNs);
        const int bad = __syncthreads_or(!ok);
        if (bad && tid == 0) {
            *abort_flag = 1;
            set_status(a.status, kStatusTimeout);
        }
        return !bad;
    };

    int64_t u = next_nonempty(a, blockIdx.x, total);
    // Units with no tokens on this CTA's stride still need hT = h0.
    for (int64_t e = blockIdx.x; e < total; e += gridDim.x) {
        Unit U;
        if (!load_unit(a, e, U)) {
            if (tid == 0) set_status(a.status, kStatusBadSeqlens);
            continue;
        }
        if (U.end > U.start || !a.hT) continue;
        const int64_t base = ((int64_t)U.n * H + U.h) * kD * kD;
        for (int i = tid; i < kD * kD; i += kThreads) a.hT[base + i] = a.h0 ? a.h0[base + i] : 0.f;
    }
    // Gates of the next chunk, prefetched one chunk ahead (threads 0..63, row = tid).
    float g_next = 0.f, b_next = 0.f;
    if (u < total) {
        Unit U;
        load_unit(a, u, U);
        if (tid == 0) {
            issue_tiles(stage(0), &full[0], &map_q, &map_k, &map_v, U.h, U.start);
            inflight |= 1u;
        }
        if (tid < 64 && U.start + tid < U.end) {
            g_next = a.g[(U.start + tid) * H + U.h];
            b_next = a.beta[(U.start + tid) * H + U.h];
        }
    }

    while (u < total && !aborted) {
        Unit U;
        load_unit(a, u, U);
        const int64_t sbase = ((int64_t)U.n * H + U.h) * kD * kD;

        // ---- initial state: R_S (fp32) and S^T (bf16 A operand). Thread (row j =
        // dv index, half) owns dk columns [64*half, 64*half + 64).
        {
            const int j = row;
            float v[64];
#pragma unroll
            for (int e = 0; e < 64; ++e)
                v[e] = a.h0 ? a.h0[sbase + (int64_t)(64 * half + e) * kD + j] : 0.f;
            float w0[32], w1[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) { w0[e] = v[e]; w1[e] = v[32 + e]; }
            tmem_st32(tmem + lane_off + kRS + 64 * half, w0);
            tmem_st32(tmem + lane_off + kRS + 64 * half + 32, w1);
            store_row64(sSA + half * 16384, j, v);
            tmem_wait_st();
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        for (int64_t c0 = U.start; c0 < U.end && !aborted; c0 += kC) {
            const int L = (U.end - c0 < kC) ? (int)(U.end - c0) : kC;
            const bool last = c0 + kC >= U.end;
            uint8_t* st = stage(cur);

            // ---- prefetch the next chunk (this unit or the next one): tiles into
            // the other stage by TMA, gates into registers
            const float g_cur = g_next, b_cur = b_next;
            {
                int64_t nu = u, nc0 = c0 + kC, nend = U.end;
                int nh = U.h;
                if (last) {
                    nu = next_nonempty(a, u + gridDim.x, total);
                    if (nu < total) {
                        Unit N2;
                        load_unit(a, nu, N2);
                        nc0 = N2.start;
                        nend = N2.end;
                        nh = N2.h;
                    }
                }
                if (nu < total) {
                    if (tid == 0) {
                        issue_tiles(stage(cur ^ 1), &full[cur ^ 1], &map_q, &map_k, &map_v, nh, nc0);
                        inflight |= 1u << (cur ^ 1);
                    }
                    g_next = 0.f;
                    b_next = 0.f;
                    if (tid < 64 && nc0 + tid < nend) {
                        g_next = a.g[(nc0 + tid) * H + nh];
                        b_next = a.beta[(nc0 + tid) * H + nh];
                    }
                }
            }
            if (!wait_all(&full[cur], (full_phase >> cur) & 1u)) { aborted = true; break; }
            full_phase ^= 1u << cur;
            inflight &= ~(1u << cur);

            // ---- per-row scalars: gates, cumulative decay, L2 norms
            if (tid < 64) {
                const int r = tid;
                float g = 0.f, b = 0.f, fq = 0.f;
                if (r < L) {
                    g = g_cur;
                    b = b_cur;
                    const float ss = row_sumsq(st + kQb0, r) + row_sumsq(st + kQb1, r);
                    fq = (a.qk_l2norm ? 1.f / sqrtf(ss + a.eps) : 1.f) * a.scale;
                }
                float x = g;  // inclusive scan over the 64 rows (two warps)
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                if (tid == 31) *carry = x;
                bet[r] = b;
                rq[r] = fq;
                gam[r] = x;  // warp 1 adds warp 0's total below
            } else if (tid < 128) {
                const int r = tid - 64;
                float fk = 0.f;
                if (r < L) {
                    const float ss = row_sumsq(st + kKb0, r) + row_sumsq(st + kKb1, r);
                    fk = a.qk_l2norm ? 1.f / sqrtf(ss + a.eps) : 1.f;
                }
                rk[r] = fk;
            }
            __syncthreads();
            if (tid >= 32 && tid < 64) gam[tid] += *carry;
            __syncthreads();
            const float gL = gam[63];

            // ---- MMA_a: [Q;K] K^T -> R_A
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t qo = (k < 4 ? kQb0 : kQb1) + 32 * (k & 3);
                    const uint32_t ko = (k < 4 ? kKb0 : kKb1) + 32 * (k & 3);
                    mma_bf16(tmem + kRA, sw128_desc(smem_u32(st + qo), 16, 1024),
                             sw128_desc(smem_u32(st + ko), 16, 1024), kIdescA, k > 0);
                }
                mma_commit(mbar);
            }
            if (!wait_all(mbar, mma_phase)) { aborted = true; break; }
            mma_phase ^= 1;
            tc_fence_after();

            // ---- epilogue a: P rows (lanes < 64) and A rows (lanes >= 64); each
            // thread takes 32 of the 64 columns. Branch-free: every element is
            // computed (exponent clamped at 0 so the masked-out upper triangle
            // cannot overflow), then selected.
            {
                float x[32];
                tmem_ld32(tmem + lane_off + kRA + 32 * half, x);
                tmem_wait_ld();
                const int j0 = 32 * half;
                if (row < 64) {
                    const int r = row;
                    const float gr = gam[r], fr = rq[r];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = j0 + e;
                        const float ex = __expf(fminf(gr - gam[j], 0.f));
                        const float val = ex * (fr * rk[j]) * x[e];
                        x[e] = (j <= r) ? val : 0.f;
                    }
                    store_half_row(sP, r, half, x, 1.f);
                } else {
                    const int r = row - 64;
                    const float gr = gam[r], fr = bet[r] * rk[r];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = j0 + e;
                        const float ex = __expf(fminf(gr - gam[j], 0.f));
                        const float val = ex * (fr * rk[j]) * x[e];
                        x[e] = (j < r) ? val : 0.f;
                    }
                    float4* Ar = reinterpret_cast<float4*>(sA + r * kLdA + j0);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        Ar[q4] = make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();

            // ---- solve T = (I + A)^-1 by blocks: 16x16 diagonal inverses by forward
            // substitution (one column per thread, tid < 64), merged to 32x32
            // (T_10 = -T_11 A_10 T_00), then to 64x64 below. Meanwhile tid 64..191
            // turn Q into Q~ and tid 192..255 clear the upper-right 32x32 block.
            if (tid < 64) {
                const int o = 16 * (tid >> 4), c = tid & 15;
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
                const bool left = ((tid >> 4) & 1) == 0;  // block 0 or 2: clear its right neighbour
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    sT[(o + r) * kLdA + o + c] = x[r];
                    if (left) sT[(o + r) * kLdA + o + 16 + c] = 0.f;
                }
            } else if (tid < 192) {
                const int rr = tid - 64, r = rr & 63;
                scale_row(st + ((rr >> 6) ? kQb1 : kQb0), r, expf(gam[r]) * rq[r]);
            } else {
                for (int e = tid - 192; e < 32 * 32; e += 64) sT[(e >> 5) * kLdA + 32 + (e & 31)] = 0.f;
            }
            __syncthreads();
            {
                // 16 -> 32: for the pairs of diagonal blocks at offset o = 0 and 32,
                // Y = A_10 T_00 then T_10 = -T_11 Y; thread -> 1 row x 2 columns.
                const int o = 32 * (tid >> 7), idx = tid & 127;
                const int r = idx >> 3, cc = 2 * (idx & 7);
                float y0 = 0.f, y1 = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float2 t2 = *reinterpret_cast<const float2*>(sT + (o + m) * kLdA + o + cc);
                    const float av = sA[(o + 16 + r) * kLdA + o + m];
                    y0 = fmaf(av, t2.x, y0);
                    y1 = fmaf(av, t2.y, y1);
                }
                __syncthreads();  // A_10 blocks fully read
                *reinterpret_cast<float2*>(sA + (o + 16 + r) * kLdA + o + cc) = make_float2(y0, y1);
                __syncthreads();
                float z0 = 0.f, z1 = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float2 y2 = *reinterpret_cast<const float2*>(sA + (o + 16 + m) * kLdA + o + cc);
                    const float tv = sT[(o + 16 + r) * kLdA + o + 16 + m];
                    z0 = fmaf(tv, y2.x, z0);
                    z1 = fmaf(tv, y2.y, z1);
                }
                *reinterpret_cast<float2*>(sT + (o + 16 + r) * kLdA + o + cc) = make_float2(-z0, -z1);
            }
            __syncthreads();
            {
                // Y = A_10 T_00 ; thread -> 2 rows x 2 columns of the 32x32 block
                const int r0 = 2 * (tid >> 4), c0b = 2 * (tid & 15);
                float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll 8
                for (int m = 0; m < 32; ++m) {
                    const float2 t2 = *reinterpret_cast<const float2*>(sT + m * kLdA + c0b);
                    const float a0 = sA[(32 + r0) * kLdA + m], a1 = sA[(33 + r0) * kLdA + m];
                    y00 = fmaf(a0, t2.x, y00); y01 = fmaf(a0, t2.y, y01);
                    y10 = fmaf(a1, t2.x, y10); y11 = fmaf(a1, t2.y, y11);
                }
                __syncthreads();  // everyone done reading A_10
                *reinterpret_cast<float2*>(sA + (32 + r0) * kLdA + c0b) = make_float2(y00, y01);
                *reinterpret_cast<float2*>(sA + (33 + r0) * kLdA + c0b) = make_float2(y10, y11);
                __syncthreads();
                // T_10 = -T_11 Y  (Y now in A's lower-left block)
                float z00 = 0.f, z01 = 0.f, z10 = 0.f, z11 = 0.f;
#pragma unroll 8
                for (int m = 0; m < 32; ++m) {
                    const float2 y2 = *reinterpret_cast<const float2*>(sA + (32 + m) * kLdA + c0b);
                    const float t0 = sT[(32 + r0) * kLdA + 32 + m], t1 = sT[(33 + r0) * kLdA + 32 + m];
                    z00 = fmaf(t0, y2.x, z00); z01 = fmaf(t0, y2.y, z01);
                    z10 = fmaf(t1, y2.x, z10); z11 = fmaf(t1, y2.y, z11);
                }
                *reinterpret_cast<float2*>(sT + (32 + r0) * kLdA + c0b) = make_float2(-z00, -z01);
                *reinterpret_cast<float2*>(sT + (33 + r0) * kLdA + c0b) = make_float2(-z10, -z11);
            }
            __syncthreads();
            // T1^T, T2^T rows (row m = column m of T) as bf16 MN-major B operands
            if (tid < 128) {
                const int j = tid & 63;
                float x[64];
#pragma unroll
                for (int r = 0; r < 64; ++r) x[r] = sT[r * kLdA + j];
                if (tid < 64) store_row64_scaled(sT1, j, x, bet[j] * expf(gam[j]) * rk[j]);
                else store_row64_scaled(sT2, j, x, bet[j]);
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();

            // ---- MMA_w: W^T = K^T T1^T -> R_W ;  MMA_b: U~^T = V^T T2^T -> R_U
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    mma_bf16(tmem + kRW, sw128_desc(smem_u32(st + kKb0 + 2048 * k), kKb1 - kKb0, 1024),
                             sw128_desc(smem_u32(sT1 + 2048 * k), 8192, 1024), kIdescMN, k > 0);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    mma_bf16(tmem + kRU, sw128_desc(smem_u32(st + kVb0 + 2048 * k), kVb1 - kVb0, 1024),
                             sw128_desc(smem_u32(sT2 + 2048 * k), 8192, 1024), kIdescMN, k > 0);
                }
                mma_commit(mbar);
            }
            if (!wait_all(mbar, mma_phase)) { aborted = true; break; }
            mma_phase ^= 1;
            tc_fence_after();

            // ---- epilogue w: -W^T rows (lane = dk i, 32 columns each); K -> K~ in place
            {
                float x[32];
                tmem_ld32(tmem + lane_off + kRW + 32 * half, x);
                tmem_wait_ld();
                store_half_row(sWT, row, half, x, -1.f);
                if (tid < 128) {
                    const int r = tid & 63;
                    scale_row(st + (tid < 64 ? kKb0 : kKb1), r, expf(gL - gam[r]) * rk[r]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();

            // ---- MMA1: U^T += S^T (-W^T) (R_U) ; O^T = S^T Q~^T (R_O)
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t sa = sw128_desc(smem_u32(sSA + (k >> 2) * 16384 + 32 * (k & 3)), 16, 1024);
                    mma_bf16(tmem + kRU, sa, sw128_desc(smem_u32(sWT + 2048 * k), 8192, 1024), kIdescSW, 1);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t sa = sw128_desc(smem_u32(sSA + (k >> 2) * 16384 + 32 * (k & 3)), 16, 1024);
                    const uint32_t qo = (k < 4 ? kQb0 : kQb1) + 32 * (k & 3);
                    mma_bf16(tmem + kRO, sa, sw128_desc(smem_u32(st + qo), 16, 1024), kIdescSQ, k > 0);
                }
                mma_commit(mbar);
            }
            // R_S <- e^{gamma_L} R_S while MMA1 runs (MMA1 does not touch R_S)
            {
                const float eL = expf(gL);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float v[32];
                    tmem_ld32(tmem + lane_off + kRS + 64 * half + 32 * cc, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] *= eL;
                    tmem_st32(tmem + lane_off + kRS + 64 * half + 32 * cc, v);
                }
                tmem_wait_st();
            }
            if (!wait_all(mbar, mma_phase)) { aborted = true; break; }
            mma_phase ^= 1;
            tc_fence_after();

            // ---- epilogue U: U^T rows (lane = dv j, 32 tokens each) as bf16 A operand
            {
                float x[32];
                tmem_ld32(tmem + lane_off + kRU + 32 * half, x);
                tmem_wait_ld();
                store_half_row(sUT, row, half, x, 1.f);
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();

            // ---- MMA2: O^T += U^T P^T (R_O) ; S^T += U^T K~ (R_S)
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + kRO, sw128_desc(smem_u32(sUT + 32 * k), 16, 1024),
                             sw128_desc(smem_u32(sP + 32 * k), 16, 1024), kIdescSQ, 1);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + kRS, sw128_desc(smem_u32(sUT + 32 * k), 16, 1024),
                             sw128_desc(smem_u32(st + kKb0 + 2048 * k), kKb1 - kKb0, 1024), kIdescUK, 1);
                mma_commit(mbar);
            }
            if (!wait_all(mbar, mma_phase)) { aborted = true; break; }
            mma_phase ^= 1;
            tc_fence_after();

            // ---- epilogue S and O
            {
                const int j = row;
                float v[64];
                tmem_ld64(tmem + lane_off + kRS + 64 * half, v);
                tmem_wait_ld();
                store_row64(sSA + half * 16384, j, v);
                if (last && a.hT) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) a.hT[sbase + (int64_t)(64 * half + e) * kD + j] = v[e];
                }
                // O^T column j, tokens [32*half, 32*half+32) -> O tile [64 tokens][128]
                // bf16 staged in this stage's V region (V is dead after MMA_b), then
                // written out as coalesced 16-byte rows, only the L valid tokens.
                float x[32];
                tmem_ld32(tmem + lane_off + kRO + 32 * half, x);
                tmem_wait_ld();
                uint16_t* ostage = reinterpret_cast<uint16_t*>(st + kVb0);
#pragma unroll
                for (int e = 0; e < 32; ++e) ostage[(32 * half + e) * kD + j] = f32_to_bf16(x[e]);
            }
            __syncthreads();
            {
                const uint4* src = reinterpret_cast<const uint4*>(st + kVb0);
                uint16_t* o = static_cast<uint16_t*>(a.o);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int vid = tid + kThreads * i;  // 16-byte vector id
                    const int r = vid >> 4, c16 = vid & 15;
                    if (r < L)
                        *reinterpret_cast<uint4*>(o + ((c0 + r) * H + U.h) * kD + 8 * c16) = src[vid];
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
            cur ^= 1;
        }
        u = next_nonempty(a, u + gridDim.x, total);
    }

    // ---- drain TMA copies still in flight (bounded), free TMEM
    if (tid == 0) {
        for (int s = 0; s < 2; ++s)
            if ((inflight >> s) & 1u) mbar_wait(&full[s], (full_phase >> s) & 1u, kWaitNs);
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

// [T_tot, H, 128] bf16 viewed as a 3-D tensor (feature, head, token); boxes of
// 64 features x 1 head x 64 tokens, 128-byte swizzle, zero fill past T_tot.
bool make_map(CUtensorMap* m, const void* ptr, int H, int64_t T) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
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

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.H, a.T_tot) || !make_map(&mk, a.k, a.H, a.T_tot) ||
        !make_map(&mv, a.v, a.H, a.T_tot))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t units = (int64_t)a.N * a.H;
    const int grid = (int)(units < sms ? units : sms);
    TcParams p{a};
    prefill_tc_kernel<<<grid, kThreads, kSmemAlloc, s>>>(p, mq, mk, mv);
    return cudaGetLastError();
}

}  // namespace gdn
