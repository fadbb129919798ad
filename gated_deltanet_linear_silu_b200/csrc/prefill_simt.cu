// Chunked gated delta rule, fp32 on CUDA cores (any supported head dims).
//
// The recurrence ("Qwen3.5-MoE source walkthrough", 4.3) is regrouped in
// chunks of C tokens, the WY/UT form of "Parallelizing Linear Transformers
// with the Delta Rule over Sequence Length" (Yang et al., 2024) with the
// gating of "Gated Delta Networks" (Yang, Kautz, Hatamizadeh, 2024), written
// for the decay-first rule. For a chunk r = 0..L-1 with start state S
// [dk, dv] and gamma_r = g_0 + ... + g_r:
//   A[r][j] = beta_r e^{gamma_r - gamma_j} k_r.k_j  (j < r),  T = (I + A)^{-1}
//   W = T diag(beta e^gamma) K,   U~ = T diag(beta) V,   U = U~ - W S
//   O = diag(e^gamma) Q S + (Q K^T o M) U,   M[r][j] = e^{gamma_r - gamma_j} (j <= r)
//   S <- e^{gamma_{L-1}} S + (diag(e^{gamma_{L-1} - gamma}) K)^T U
// Only exponentials of non-positive differences are formed, so strong decay
// underflows to zero instead of overflowing. Padding a partial chunk with
// zero rows (k = q = v = 0, beta = g = 0) is exact.
//
// One CTA (256 threads) owns one (sequence, head, d_v tile) at a time and
// walks its chunks in order with the state tile resident in shared memory.
// The grid is persistent; units are taken from a counter in longest-sequence
// -first order. This kernel is the fp32 path (tolerance 1e-4 configurations)
// and the path for head dims other than 128.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct Layout {
    int C, dk, DVT, ldk, ldv, ldc, lds;
    size_t q, k, w, v, u, s, am, tm, p, gam, bet, total_floats;
};

__host__ __device__ inline Layout make_layout(int C, int dk, int DVT) {
    Layout L;
    L.C = C; L.dk = dk; L.DVT = DVT;
    L.ldk = dk + 1; L.ldv = DVT + 1; L.ldc = C + 1; L.lds = DVT + 1;  // odd strides: no bank conflicts
    size_t o = 0;
    L.q = o;  o += (size_t)C * L.ldk;
    L.k = o;  o += (size_t)C * L.ldk;
    L.w = o;  o += (size_t)C * L.ldk;
    L.v = o;  o += (size_t)C * L.ldv;
    L.u = o;  o += (size_t)C * L.ldv;
    L.s = o;  o += (size_t)dk * L.lds;
    L.am = o; o += (size_t)C * L.ldc;
    L.tm = o; o += (size_t)C * L.ldc;
    L.p = o;  o += (size_t)C * L.ldc;
    L.gam = o; o += C;
    L.bet = o; o += C;
    L.total_floats = o;
    return L;
}

// acc[i][0..1] += sum_k A[(m0+i)*sam + k*sak] * B[k*sbk + n*sbn], n in {nA, nB}.
__device__ __forceinline__ void mac4x2(float (&acc)[4][2], const float* A, int sam, int sak,
                                       const float* B, int sbk, int sbn, int Kd, int m0, int nA,
                                       int nB, bool okA, bool okB) {
    const float* a0 = A + (size_t)m0 * sam;
    for (int k = 0; k < Kd; ++k) {
        const float b0 = okA ? B[k * sbk + nA * sbn] : 0.f;
        const float b1 = okB ? B[k * sbk + nB * sbn] : 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float av = a0[i * sam + k * sak];
            acc[i][0] = fmaf(av, b0, acc[i][0]);
            acc[i][1] = fmaf(av, b1, acc[i][1]);
        }
    }
}

// out(m, n) = sum_k A(m, k) B(k, n) for m < M (multiple of 4), n < N; each warp
// takes 4 x 64 tiles; epi(m, n, value) consumes the result.
template <class Epi>
__device__ __forceinline__ void gemm(int M, int N, int Kd, const float* A, int sam, int sak,
                                     const float* B, int sbk, int sbn, Epi epi) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = M >> 2, nt = (N + 63) >> 6;
    for (int tile = warp; tile < mt * nt; tile += kWarps) {
        const int m0 = (tile % mt) * 4;
        const int nA = (tile / mt) * 64 + lane, nB = nA + 32;
        const bool okA = nA < N, okB = nB < N;
        float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
        mac4x2(acc, A, sam, sak, B, sbk, sbn, Kd, m0, nA, nB, okA, okB);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (okA) epi(m0 + i, nA, acc[i][0]);
            if (okB) epi(m0 + i, nB, acc[i][1]);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) prefill_simt_kernel(PrefillArgs a, int DVT, int n_vt) {
    extern __shared__ float sm[];
    __shared__ int s_unit;
    const int C = a.chunk, dk = a.dk, dv = a.dv, H = a.H;
    const Layout Lo = make_layout(C, dk, DVT);
    float* Qs = sm + Lo.q;
    float* Ks = sm + Lo.k;
    float* Ws = sm + Lo.w;
    float* Vs = sm + Lo.v;
    float* Us = sm + Lo.u;
    float* Ss = sm + Lo.s;
    float* Am = sm + Lo.am;
    float* Tm = sm + Lo.tm;
    float* Pm = sm + Lo.p;
    float* gam = sm + Lo.gam;
    float* bet = sm + Lo.bet;
    const int ldk = Lo.ldk, ldv = Lo.ldv, ldc = Lo.ldc, lds = Lo.lds;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const T* q = static_cast<const T*>(a.q);
    const T* k = static_cast<const T*>(a.k);
    const T* v = static_cast<const T*>(a.v);
    T* o = static_cast<T*>(a.o);
    const int64_t total_units = (int64_t)a.N * H * n_vt;

    for (;;) {
        if (tid == 0) s_unit = atomicAdd(a.counter, 1);
        __syncthreads();
        const int64_t unit = s_unit;
        __syncthreads();
        if (unit >= total_units) break;
        const int vt = (int)(unit % n_vt);
        const int h = (int)((unit / n_vt) % H);
        const int hk = h / (H / a.Hk);  // the q, k head this value head reads
        const int n = a.order[unit / ((int64_t)n_vt * H)];
        const int64_t start = a.cu[n], end = a.cu[n + 1];
        if (!(n >= 0 && n < a.N && start >= 0 && start <= end && end <= a.T_tot)) {
            if (tid == 0) set_status(a.status, kStatusBadSeqlens);
            continue;
        }
        const int j0 = vt * DVT;  // first value column of this tile

        // Initial state tile.
        for (int e = tid; e < dk * DVT; e += kThreads) {
            const int i = e / DVT, j = e % DVT;
            Ss[i * lds + j] = a.h0 ? a.h0[(((int64_t)n * H + h) * dk + i) * dv + j0 + j] : 0.f;
        }

        for (int64_t c0 = start; c0 < end; c0 += C) {
            const int L = (end - c0 < C) ? (int)(end - c0) : C;
            __syncthreads();  // previous chunk finished with every buffer
            // 1. Load the chunk (rows >= L are zero).
            for (int e = tid; e < C * dk; e += kThreads) {
                const int r = e / dk, i = e % dk;
                float qv = 0.f, kv = 0.f;
                if (r < L) {
                    qv = Elem<T>::load(q, (c0 + r) * a.ld_q + hk * dk + i);
                    kv = Elem<T>::load(k, (c0 + r) * a.ld_k + hk * dk + i);
                }
                Qs[r * ldk + i] = qv;
                Ks[r * ldk + i] = kv;
            }
            for (int e = tid; e < C * DVT; e += kThreads) {
                const int r = e / DVT, j = e % DVT;
                Vs[r * ldv + j] = r < L ? Elem<T>::load(v, (c0 + r) * a.ld_v + h * dv + j0 + j) : 0.f;
            }
            if (tid < C) {
                gam[tid] = tid < L ? a.g[(c0 + tid) * H + h] : 0.f;
                bet[tid] = tid < L ? a.beta[(c0 + tid) * H + h] : 0.f;
            }
            __syncthreads();
            // 2. L2 norm of q and k rows, q scale; cumulative decay.
            for (int r = warp; r < L; r += kWarps) {
                float sq = 0.f, sk = 0.f;
                for (int i = lane; i < dk; i += 32) {
                    sq += Qs[r * ldk + i] * Qs[r * ldk + i];
                    sk += Ks[r * ldk + i] * Ks[r * ldk + i];
                }
                sq = warp_sum(sq);
                sk = warp_sum(sk);
                const float iq = (a.qk_l2norm ? 1.f / sqrtf(sq + a.eps) : 1.f) * a.scale;
                const float ik = a.qk_l2norm ? 1.f / sqrtf(sk + a.eps) : 1.f;
                for (int i = lane; i < dk; i += 32) {
                    Qs[r * ldk + i] *= iq;
                    Ks[r * ldk + i] *= ik;
                }
            }
            if (tid == 0) {
                float acc = 0.f;
                for (int r = 0; r < C; ++r) {
                    acc += gam[r];
                    gam[r] = acc;
                }
            }
            __syncthreads();
            // 3. A = strict_tril(beta_r e^{grow_r - gamma_j} K K^T);  P = tril(e^{..} Q K^T).
            // The row decay grow_r is gamma_r, or gamma_{r-1} (gamma_{-1} = 0) when
            // token r reads the state before its own decay.
            const bool und = a.undecayed != 0;
            gemm(C, C, dk, Ks, ldk, 1, Ks, 1, ldk, [&](int r, int j, float x) {
                const float gr = und ? (r > 0 ? gam[r - 1] : 0.f) : gam[r];
                Am[r * ldc + j] = j < r ? bet[r] * expf(gr - gam[j]) * x : 0.f;
            });
            gemm(C, C, dk, Qs, ldk, 1, Ks, 1, ldk, [&](int r, int j, float x) {
                Pm[r * ldc + j] = j <= r ? expf(gam[r] - gam[j]) * x : 0.f;
            });
            __syncthreads();
            // 4. T = (I + A)^{-1} by forward substitution, LPC lanes per column.
            {
                const int LPC = kThreads / C;
                const int j = tid / LPC, part = tid % LPC;
                for (int r = part; r < C; r += LPC) Tm[r * ldc + j] = (r == j) ? 1.f : 0.f;
                __syncwarp();
                for (int r = 1; r < C; ++r) {
                    float s = 0.f;
                    if (r > j)
                        for (int m = j + part; m < r; m += LPC) s = fmaf(Am[r * ldc + m], Tm[m * ldc + j], s);
                    s = group_sum(s, LPC);
                    if (r > j && part == 0) Tm[r * ldc + j] = -s;
                    __syncwarp();
                }
            }
            __syncthreads();
            // 5. T1 = T diag(beta e^grow) (into Am), T2 = T diag(beta) (in place).
            for (int e = tid; e < C * C; e += kThreads) {
                const int r = e / C, m = e % C;
                const float t = Tm[r * ldc + m];
                const float gm = und ? (m > 0 ? gam[m - 1] : 0.f) : gam[m];
                Am[r * ldc + m] = t * bet[m] * expf(gm);
                Tm[r * ldc + m] = t * bet[m];
            }
            __syncthreads();
            // 6. W = T1 K,  U~ = T2 V.
            gemm(C, dk, C, Am, ldc, 1, Ks, ldk, 1, [&](int r, int i, float x) { Ws[r * ldk + i] = x; });
            gemm(C, DVT, C, Tm, ldc, 1, Vs, ldv, 1, [&](int r, int j, float x) { Us[r * ldv + j] = x; });
            __syncthreads();
            // 7. U = U~ - W S.
            gemm(C, DVT, dk, Ws, ldk, 1, Ss, lds, 1, [&](int r, int j, float x) { Us[r * ldv + j] -= x; });
            __syncthreads();
            // 8. O = diag(e^gamma) Q S + P U  -> global.
            {
                const int mt = C >> 2, nt = (DVT + 63) >> 6;
                for (int tile = warp; tile < mt * nt; tile += kWarps) {
                    const int m0 = (tile % mt) * 4;
                    const int nA = (tile / mt) * 64 + lane, nB = nA + 32;
                    const bool okA = nA < DVT, okB = nB < DVT;
                    float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
                    mac4x2(acc, Qs, ldk, 1, Ss, lds, 1, dk, m0, nA, nB, okA, okB);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float e = expf(gam[m0 + i]);
                        acc[i][0] *= e;
                        acc[i][1] *= e;
                    }
                    mac4x2(acc, Pm, ldc, 1, Us, ldv, 1, C, m0, nA, nB, okA, okB);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = m0 + i;
                        if (r >= L) continue;
                        const int64_t base = ((c0 + r) * H + h) * dv + j0;
                        if (okA) Elem<T>::store(o, base + nA, acc[i][0]);
                        if (okB) Elem<T>::store(o, base + nB, acc[i][1]);
                    }
                }
            }
            // 9. K~ = diag(e^{gamma_{L-1} - gamma}) K (K is not read by step 8).
            const float gL = gam[L - 1];
            for (int e = tid; e < L * dk; e += kThreads) {
                const int m = e / dk, i = e % dk;
                Ks[m * ldk + i] *= expf(gL - gam[m]);
            }
            __syncthreads();
            // 10. S <- e^{gamma_{L-1}} S + K~^T U.
            const float eL = expf(gL);
            gemm(dk, DVT, C, Ks, 1, ldk, Us, ldv, 1, [&](int i, int j, float x) {
                Ss[i * lds + j] = fmaf(eL, Ss[i * lds + j], x);
            });
        }
        __syncthreads();
        if (a.hT)
            for (int e = tid; e < dk * DVT; e += kThreads) {
                const int i = e / DVT, j = e % DVT;
                a.hT[(((int64_t)n * H + h) * dk + i) * dv + j0 + j] = Ss[i * lds + j];
            }
        __syncthreads();
    }
}

int sm_count() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <typename T>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t s) {
    const int n_vt = a.dv <= 64 ? 1 : 2;
    const int DVT = a.dv / n_vt;
    const Layout Lo = make_layout(a.chunk, a.dk, DVT);
    const size_t smem = Lo.total_floats * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefill_simt_kernel<T>, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int64_t units = (int64_t)a.N * a.H * n_vt;
    const int64_t cap = (int64_t)sm_count() * per_sm;
    const int64_t grid = units < cap ? units : cap;
    if (grid <= 0) return cudaSuccess;
    prefill_simt_kernel<T><<<(unsigned)grid, kThreads, smem, s>>>(a, DVT, n_vt);
    return cudaGetLastError();
}

}  // namespace

size_t prefill_simt_smem_bytes(int chunk, int dk, int dv) {
    const int n_vt = dv <= 64 ? 1 : 2;
    return make_layout(chunk, dk, dv / n_vt).total_floats * sizeof(float);
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s) {
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
