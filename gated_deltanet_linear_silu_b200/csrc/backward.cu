// Backward of the gated delta rule (fp32 CUDA cores), one CTA per (sequence,
// value head), token by token.
//
// Forward rule ("Qwen3.5-MoE source walkthrough", 4.3), state S [dk, dv]:
//   k^ = L2(k_t), q^ = scale L2(q_t);  S' = a S (a = e^{g_t});  m = S'^T k^;
//   delta = beta (v - m);  S_t = S' + k^ delta^T;  o_t = S_t^T q^.
// Reverse-mode step for token t, with dS the gradient of S_t on entry:
//   dS += q^ do^T;            dq^ = S_t do = S' do + k^ (delta . do)
//   ddelta = dS^T k^;         dk^ = dS delta;   dv = beta ddelta;
//   dbeta = ddelta . (v - m); dm = -beta ddelta; dk^ += S' dm;
//   dS' = dS + k^ dm^T;       dg = <dS', S'>;   dS <- a dS'  (gradient of S_{t-1}),
// then through the L2 norms: dk = (dk^ - k^ (k^ . dk^)) / |k|_eps and
// dq = scale (dq~ - q~ (q~ . dq~)) / |q|_eps with q~ = q / |q|_eps, dq~ = dq^.
//
// The reverse sweep needs S_{t-1} for every token: a forward pass stores the
// state every ck tokens (checkpoints in the workspace), then for each block of
// ck tokens, last block first, the states before each token are recomputed
// into a per-CTA workspace buffer and the block is swept backwards.
//
// Layout: thread (rg, cg) holds rows [rg*RPT, rg*RPT+RPT) x columns [4cg, 4cg+4)
// of S_{t-1} and of dS in registers; sums over rows go through `red`
// [RG][dv], sums over columns through `redr` [dk][dv/4 + 1] (the extra column
// keeps the threads that add up one row each on distinct banks), and the
// per-thread terms of dg through `gps` [threads].
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

template <typename T, int RPT>
__global__ void __launch_bounds__(256) backward_kernel(BackwardArgs a) {
    extern __shared__ float sm[];
    const int dk = a.dk, dv = a.dv, cols4 = dv >> 2, RG = dk / RPT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = tid % cols4, rg = tid / cols4;
    const int i0 = rg * RPT, j0 = 4 * cg;
    const int H = a.H, Hk = a.Hk, G = H / Hk;
    const int64_t unit = blockIdx.x;
    const int n = (int)(unit / H), h = (int)(unit % H), hk = h / G;
    const int64_t DD = (int64_t)dk * dv;

    float* qn = sm;              // [dk] q / |q|_eps
    float* kh = qn + dk;         // [dk] k^
    float* rr = kh + dk;         // [dk] S' do / a
    float* dkh = rr + dk;        // [dk]
    float* dqh = dkh + dk;       // [dk]
    float* vv = dqh + dk;        // [dv]
    float* dov = vv + dv;        // [dv]
    float* mm = dov + dv;        // [dv] m
    float* dl = mm + dv;         // [dv] delta
    float* dmm = dl + dv;        // [dv] dm
    float* dbt = dmm + dv;       // [dv] ddelta (v - m)
    float* red = dbt + dv;       // [RG][dv]
    const int ldr = cols4 + 1;
    float* redr = red + RG * dv; // [dk][ldr]
    float* scal = redr + dk * ldr;  // [16]: a, beta, |q|, |k|, delta.do, k^.dk^, q~.dq~, -,
                                    //       g, beta as loaded
    float* gps = scal + 16;         // [threads]

    const int64_t start = a.cu[n], end = a.cu[n + 1];
    const int ck = a.ck;  // tokens between checkpoints: kCk, or 1 (every state kept)
    const int64_t ck_base = 2 * (int64_t)n + (start + ck - 1) / ck;  // first checkpoint slot
    const int64_t nch = (end - start + ck - 1) / ck;
    if (!(start >= 0 && start <= end && end <= a.T_tot && ck_base + nch <= a.ck_slots)) {
        if (tid == 0) set_status(a.status, kStatusBadSeqlens);
        return;
    }
    const T* q = static_cast<const T*>(a.q);
    const T* k = static_cast<const T*>(a.k);
    const T* v = static_cast<const T*>(a.v);
    float* buf = ck > 1 ? a.ws_buf + unit * ck * DD : nullptr;
    auto ckpt = [&](int64_t c) { return a.ws_ckpt + ((ck_base + c) * H + h) * DD; };
    auto load_tile = [&](const float* base, float4 (&x)[RPT]) {
#pragma unroll
        for (int r = 0; r < RPT; ++r) x[r] = *reinterpret_cast<const float4*>(base + (int64_t)(i0 + r) * dv + j0);
    };
    auto store_tile = [&](float* base, const float4 (&x)[RPT]) {
#pragma unroll
        for (int r = 0; r < RPT; ++r) *reinterpret_cast<float4*>(base + (int64_t)(i0 + r) * dv + j0) = x[r];
    };
    // Token t's k^ (and q~, do when `full`), v, a, beta into shared memory. A
    // thread holds at most one element of each vector (the CTA has at least
    // max(dk, dv) threads), and the next token's elements are requested into
    // registers while the current token is worked on: the guess is t + 1 in the
    // forward passes and t - 1 in the reverse sweep; a wrong guess (once per
    // block of ck tokens) just loads again.
    struct Pref {
        float k, q, v, d, g, b;
        int64_t t;
        bool full;
    } pf{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, -1, false};
    auto issue = [&](int64_t t, bool full) {
        pf.t = t;
        pf.full = full;
        if (t < start || t >= end) return;
        if (tid < dk) {
            pf.k = Elem<T>::load(k, (t * Hk + hk) * dk + tid);
            if (full) pf.q = Elem<T>::load(q, (t * Hk + hk) * dk + tid);
        }
        if (tid < dv) {
            pf.v = Elem<T>::load(v, (t * H + h) * dv + tid);
            if (full) pf.d = a.dO[(t * H + h) * dv + tid];
        }
        if (tid == 0) {
            pf.g = a.g[t * H + h];
            pf.b = a.beta[t * H + h];
        }
    };
    auto load_token = [&](int64_t t, bool full, int64_t t_next, bool full_next) {
        if (pf.t != t || pf.full != full) issue(t, full);
        __syncthreads();  // the previous token's values are no longer read
        if (tid == 0) {
            scal[8] = pf.g;
            scal[9] = pf.b;
        }
        if (tid < dk) {
            kh[tid] = pf.k;
            if (full) qn[tid] = pf.q;
        }
        if (tid < dv) {
            vv[tid] = pf.v;
            if (full) dov[tid] = pf.d;
        }
        issue(t_next, full_next);
        __syncthreads();
        if (warp == 0) {
            float sk = 0.f, sq = 0.f;
            for (int i = lane; i < dk; i += 32) {
                sk += kh[i] * kh[i];
                if (full) sq += qn[i] * qn[i];
            }
            sk = warp_sum(sk);
            sq = warp_sum(sq);
            if (lane == 0) {
                scal[0] = expf(scal[8]);
                scal[1] = scal[9];
                scal[2] = a.qk_l2norm ? sqrtf(sq + a.eps) : 1.f;
                scal[3] = a.qk_l2norm ? sqrtf(sk + a.eps) : 1.f;
            }
        }
        __syncthreads();
        const float inv_k = 1.f / scal[3], inv_q = 1.f / scal[2];
        for (int i = tid; i < dk; i += blockDim.x) {
            kh[i] *= inv_k;
            if (full) qn[i] *= inv_q;
        }
        __syncthreads();
    };
    // Partial sums over this thread's rows (x . kh per column) into red.
    auto col_partial = [&](const float4 (&x)[RPT]) {
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float kv = kh[i0 + r];
            p.x = fmaf(x[r].x, kv, p.x); p.y = fmaf(x[r].y, kv, p.y);
            p.z = fmaf(x[r].z, kv, p.z); p.w = fmaf(x[r].w, kv, p.w);
        }
        *reinterpret_cast<float4*>(red + rg * dv + j0) = p;
    };
    // Partial sums over this thread's columns (x . w per row) into redr.
    auto row_partial = [&](const float4 (&x)[RPT], const float* w) {
        const float4 w4 = *reinterpret_cast<const float4*>(w + j0);
#pragma unroll
        for (int r = 0; r < RPT; ++r)
            redr[(i0 + r) * ldr + cg] = x[r].x * w4.x + x[r].y * w4.y + x[r].z * w4.z + x[r].w * w4.w;
    };
    auto col_total = [&](int j) {
        float s = 0.f;
        for (int g2 = 0; g2 < RG; ++g2) s += red[g2 * dv + j];
        return s;
    };
    auto row_total = [&](int i) {
        float s = 0.f;
        for (int c = 0; c < cols4; ++c) s += redr[i * ldr + c];
        return s;
    };
    // One forward token on the register tile S (the state before token t).
    auto forward_step = [&](int64_t t, float4 (&S)[RPT]) {
        load_token(t, false, t + 1, false);
        col_partial(S);
        __syncthreads();
        const float al = scal[0], be = scal[1];
        for (int j = tid; j < dv; j += blockDim.x) dl[j] = be * (vv[j] - al * col_total(j));
        __syncthreads();
        const float4 d4 = *reinterpret_cast<const float4*>(dl + j0);
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float kv = kh[i0 + r];
            S[r].x = fmaf(al, S[r].x, kv * d4.x); S[r].y = fmaf(al, S[r].y, kv * d4.y);
            S[r].z = fmaf(al, S[r].z, kv * d4.z); S[r].w = fmaf(al, S[r].w, kv * d4.w);
        }
    };

    // ---- forward: checkpoints every ck tokens
    float4 S[RPT];
    if (a.h0) load_tile(a.h0 + unit * DD, S);
    else
#pragma unroll
        for (int r = 0; r < RPT; ++r) S[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t t = start; t < end; ++t) {
        if ((t - start) % ck == 0) store_tile(ckpt((t - start) / ck), S);
        forward_step(t, S);
    }

    // ---- backward, last block first
    float4 dS[RPT];
    if (a.dhT) load_tile(a.dhT + unit * DD, dS);
    else
#pragma unroll
        for (int r = 0; r < RPT; ++r) dS[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t c = nch - 1; c >= 0; --c) {
        const int64_t c0 = start + c * ck, c1 = (c0 + ck < end) ? c0 + ck : end;
        if (ck > 1) {  // recompute the block's states into buf
            load_tile(ckpt(c), S);
            for (int64_t t = c0; t < c1; ++t) {
                store_tile(buf + (t - c0) * DD, S);  // the state before token t
                if (t + 1 < c1) forward_step(t, S);
            }
        }
        for (int64_t t = c1 - 1; t >= c0; --t) {
            __syncthreads();  // buf writes (and the previous token's reads) are done
            float4 Sp[RPT];
            load_tile(ck > 1 ? buf + (t - c0) * DD : ckpt(c), Sp);  // the state before token t
            load_token(t, true, t - 1, true);
            const float al = scal[0], be = scal[1];
            // A: m = a Sp^T k^, delta; r = Sp do
            col_partial(Sp);
            row_partial(Sp, dov);
            __syncthreads();
            for (int j = tid; j < dv; j += blockDim.x) {
                const float m = al * col_total(j);
                mm[j] = m;
                dl[j] = be * (vv[j] - m);
            }
            for (int i = tid; i < dk; i += blockDim.x) rr[i] = row_total(i);
            __syncthreads();
            // B: dS += q^ do^T; ddelta = dS^T k^; dk^ = dS delta
            const float sc = a.scale;
            {
                const float4 o4 = *reinterpret_cast<const float4*>(dov + j0);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float qv = sc * qn[i0 + r];
                    dS[r].x = fmaf(qv, o4.x, dS[r].x); dS[r].y = fmaf(qv, o4.y, dS[r].y);
                    dS[r].z = fmaf(qv, o4.z, dS[r].z); dS[r].w = fmaf(qv, o4.w, dS[r].w);
                }
            }
            col_partial(dS);
            row_partial(dS, dl);
            __syncthreads();
            for (int j = tid; j < dv; j += blockDim.x) {
                const float dd = col_total(j);
                a.dv_out[(t * H + h) * dv + j] = be * dd;
                dmm[j] = -be * dd;
                dbt[j] = dd * (vv[j] - mm[j]);
            }
            for (int i = tid; i < dk; i += blockDim.x) dkh[i] = row_total(i);
            __syncthreads();
            // C: dk^ += a Sp dm; dS' = dS + k^ dm^T; dg = a <dS', Sp>; dS <- a dS'
            row_partial(Sp, dmm);
            float gp = 0.f;
            {
                const float4 m4 = *reinterpret_cast<const float4*>(dmm + j0);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float kv = kh[i0 + r];
                    float4 x = dS[r];
                    x.x = fmaf(kv, m4.x, x.x); x.y = fmaf(kv, m4.y, x.y);
                    x.z = fmaf(kv, m4.z, x.z); x.w = fmaf(kv, m4.w, x.w);
                    gp += x.x * Sp[r].x + x.y * Sp[r].y + x.z * Sp[r].z + x.w * Sp[r].w;
                    dS[r] = make_float4(al * x.x, al * x.y, al * x.z, al * x.w);
                }
            }
            // (the CTA may end in a partial warp, so no shuffles outside warp 0)
            gps[tid] = gp;
            __syncthreads();
            for (int i = tid; i < dk; i += blockDim.x) dkh[i] += al * row_total(i);
            if (warp == 0) {
                float dd = 0.f, db = 0.f, gsum = 0.f;
                for (int j = lane; j < dv; j += 32) {
                    dd += dl[j] * dov[j];
                    db += dbt[j];
                }
                for (int x = lane; x < (int)blockDim.x; x += 32) gsum += gps[x];
                dd = warp_sum(dd);
                db = warp_sum(db);
                gsum = warp_sum(gsum);
                if (lane == 0) {
                    scal[4] = dd;
                    a.dbeta[t * H + h] = db;
                    a.dg[t * H + h] = al * gsum;
                }
            }
            __syncthreads();
            // dq^ = a r + k^ (delta . do); norm products
            for (int i = tid; i < dk; i += blockDim.x) dqh[i] = al * rr[i] + kh[i] * scal[4];
            __syncthreads();
            if (warp == 0) {
                float sk = 0.f, sq = 0.f;
                for (int i = lane; i < dk; i += 32) {
                    sk += kh[i] * dkh[i];
                    sq += qn[i] * dqh[i];
                }
                sk = warp_sum(sk);
                sq = warp_sum(sq);
                if (lane == 0) {
                    scal[5] = sk;
                    scal[6] = sq;
                }
            }
            __syncthreads();
            const float nq = scal[2], nk = scal[3], sk = scal[5], sq = scal[6];
            for (int i = tid; i < dk; i += blockDim.x) {
                const float gk = a.qk_l2norm ? (dkh[i] - kh[i] * sk) / nk : dkh[i];
                const float gq = sc * (a.qk_l2norm ? (dqh[i] - qn[i] * sq) / nq : dqh[i]);
                const int64_t o = (t * Hk + hk) * dk + i;
                if (G > 1) {
                    atomicAdd(a.dk_out + o, gk);
                    atomicAdd(a.dq_out + o, gq);
                } else {
                    a.dk_out[o] = gk;
                    a.dq_out[o] = gq;
                }
            }
        }
    }
    if (a.dh0) store_tile(a.dh0 + unit * DD, dS);
}

template <typename T, int RPT>
cudaError_t launch_rpt(const BackwardArgs& a, cudaStream_t s) {
    const int cols4 = a.dv / 4, RG = a.dk / RPT;
    const int threads = cols4 * RG;
    const size_t smem = sizeof(float) * (5 * a.dk + 6 * a.dv + RG * a.dv + a.dk * (cols4 + 1) + 16 + threads);
    backward_kernel<T, RPT><<<(unsigned)((int64_t)a.N * a.H), threads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const BackwardArgs& a, cudaStream_t s) {
    // rows per thread: the smallest power of two (<= 16, dividing dk) that keeps
    // the CTA at <= 256 threads
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

size_t backward_workspace_floats(int N, int64_t T_tot, int H, int dk, int dv, int ck) {
    const int64_t slots = 2 * (int64_t)N + (T_tot + ck - 1) / ck + 1;
    return (size_t)(slots * H + (ck > 1 ? (int64_t)N * H * ck : 0)) * dk * dv;
}

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s) {
    if ((int64_t)a.N * a.H == 0) return cudaSuccess;
    if (a.H != a.Hk) {  // q, k gradients of a shared head are sums over its value heads
        cudaError_t e = cudaMemsetAsync(a.dq_out, 0, sizeof(float) * a.T_tot * a.Hk * a.dk, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.dk_out, 0, sizeof(float) * a.T_tot * a.Hk * a.dk, s);
        if (e != cudaSuccess) return e;
    }
    return a.is_bf16 ? launch_t<uint16_t>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
