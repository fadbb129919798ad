/*
 * CPU oracle for the Gated DeltaNet token mixer -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 restatement of what the mixer computes, written from the
 * pages' definitions. Only the tests, the smoke check and the benchmark's CPU
 * baseline may call it; the product library never does, and the two share no
 * code, headers or tables.
 *
 * Sources (page title, section):
 *   [R] "Qwen3.5-MoE ... source walkthrough", section 4.3 "Qwen3_5MoeGatedDeltaNet":
 *       the recurrent (single-token) gated delta rule -- decay the state by
 *       exp(g_t), read kv_mem = sum over the key axis of S * k_t, form the
 *       correction delta = (v_t - kv_mem) * beta_t, add the outer product
 *       k_t^T delta, read the output as sum over the key axis of S * q_t.
 *       The state is [d_k, d_v]: the reductions run over the key axis.
 *   [C] "7.6 Qwen3.5: linear-attention hybrid", 7.6.2: a depthwise causal
 *       Conv1d of kernel 4 with padding 3 over conv_dim = 2*key_dim + value_dim
 *       channels, then L2 normalisation of q and k per head.
 *   [S] Same page as [R], section 8.2: the prefill keeps the last K conv inputs
 *       as the conv state (left-padded when the sequence is shorter than K),
 *       and the recurrent state is carried from call to call.
 *   [U] "7.6 Qwen3.5: linear-attention hybrid", 7.6.2, the recurrence as that
 *       page writes it: S_t = alpha_t S_{t-1} + k_t [beta_t (v_t - S_{t-1}^T k_t)]^T,
 *       i.e. the memory is read from the state before the decay. Selected by
 *       `undecayed`; [R]'s decay-first order is the default.
 * Readings where the pages are silent:
 *   SiLU follows the conv; L2(x) = x / sqrt(sum x^2 + eps); `scale` multiplies
 *   the normalised q; the conv state exposes the K-1 most recent inputs
 *   (the K-th is never read again); sequences never mix across cu_seqlens.
 *
 * Pins: tests/test_oracle_pins.py checks every function here against closed
 * forms, exact-retrieval identities, explicit unrolled matrix products on tiny
 * inputs, a library conv1d, linearity, a contraction bound and the fp64
 * chunkwise evaluator below.  Absolute parity against the pages is unpinned:
 * they print no worked numeric example of the mixer.
 *
 * Built with -DGDN_ORACLE_PIN_CHECK (a separate library that only the
 * pin-sensitivity test loads), gdn_oracle_recurrence_planted can plant one of
 * four deliberate mistakes in the recurrence, to show that the pins catch
 * each. The oracle library proper is built without that flag and has no such
 * code.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

/* bf16 -> double: the bf16 bits are the top half of an IEEE float. */
static double load_elem(const void *base, int dtype, int64_t i) {
    if (dtype == OR_F64) return ((const double *)base)[i];
    if (dtype == OR_F32) return (double)((const float *)base)[i];
    uint32_t u = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Thread pool over independent work items                                   */
/* ------------------------------------------------------------------------ */

typedef void (*item_fn)(void *ctx, int64_t item);
typedef struct {
    item_fn fn;
    void *ctx;
    int64_t n_items;
    int64_t next;
    pthread_mutex_t mu;
} pool_t;

static void *pool_worker(void *arg) {
    pool_t *p = (pool_t *)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        int64_t i = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (i >= p->n_items) return NULL;
        p->fn(p->ctx, i);
    }
}

static void run_items(item_fn fn, void *ctx, int64_t n_items, int n_threads) {
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_items) n_threads = (int)(n_items > 0 ? n_items : 1);
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n_items = n_items;
    p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    int started = 0;
    for (int t = 1; t < n_threads; ++t)
        if (pthread_create(&th[started], NULL, pool_worker, &p) == 0) ++started;
    pool_worker(&p); /* the calling thread works too */
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&p.mu);
}

/* ------------------------------------------------------------------------ */
/* Recurrence [R]: one (sequence, head) at a time, token by token.            */
/* ------------------------------------------------------------------------ */

typedef struct {
    const void *q, *k, *v;
    int dtype;
    const void *g, *beta;
    int gate_dtype;
    const int64_t *cu;
    int H, Hk, dk, dv; /* H value heads; q, k have Hk heads, each shared by H / Hk value heads */
    double scale;
    int qk_l2norm;
    double eps;
    int undecayed; /* 1: read kv_mem from the state before the decay ([U]) */
    const void *h0;
    int h0_dtype;
    double *hT, *o;
#ifdef GDN_ORACLE_PIN_CHECK
    int planted; /* the deliberate mistake to plant (1..4), 0 for none */
#endif
} rec_ctx;

#ifdef GDN_ORACLE_PIN_CHECK
#define PLANTED(n) (c->planted == (n))
#else
#define PLANTED(n) 0
#endif

/* Normalise x (length d) in place: x / sqrt(sum x^2 + eps). */
static void l2_normalise(double *x, int d, double eps) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < d; ++i) x[i] *= inv;
}

static void rec_item(void *vctx, int64_t item) {
    const rec_ctx *c = (const rec_ctx *)vctx;
    const int H = c->H, Hk = c->Hk, dk = c->dk, dv = c->dv;
    const int64_t n = item / H;
    const int h = (int)(item % H);
    const int hk = h / (H / Hk); /* the key head this value head reads */
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double)); /* S[i][j], i: key, j: value */
    double *q = (double *)malloc(sizeof(double) * dk);
    double *k = (double *)malloc(sizeof(double) * dk);
    double *m = (double *)malloc(sizeof(double) * dv);
    double *delta = (double *)malloc(sizeof(double) * dv);
    const int64_t sbase = (n * H + h) * (int64_t)dk * dv;
    if (c->h0)
        for (int64_t e = 0; e < (int64_t)dk * dv; ++e) S[e] = load_elem(c->h0, c->h0_dtype, sbase + e);

    for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        const int64_t qk_base = (t * Hk + hk) * (int64_t)dk;
        const int64_t v_base = (t * H + h) * (int64_t)dv;
        for (int i = 0; i < dk; ++i) {
            q[i] = load_elem(c->q, c->dtype, qk_base + i);
            k[i] = load_elem(c->k, c->dtype, qk_base + i);
        }
        if (c->qk_l2norm) {
            l2_normalise(q, dk, c->eps);
            l2_normalise(k, dk, c->eps);
        }
        for (int i = 0; i < dk; ++i) q[i] *= c->scale;
        const double g = load_elem(c->g, c->gate_dtype, t * H + h);
        const double beta = load_elem(c->beta, c->gate_dtype, t * H + h);
        const double alpha = exp(g);

        /* [U]: kv_mem_j = sum_i S_{t-1}[i][j] k_i, before the decay.
         * (planted mistake 1: the same read in the default rule) */
        if (c->undecayed || PLANTED(1))
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * k[i];
                m[j] = acc;
            }

        /* S <- S * exp(g_t) */
        if (!PLANTED(3)) /* planted mistake 3: no decay */
            for (int64_t e = 0; e < (int64_t)dk * dv; ++e) S[e] *= alpha;

        /* [R]: kv_mem_j = sum_i S[i][j] k_i  (reduction over the key axis) */
        if (!c->undecayed && !PLANTED(1))
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) {
                    /* planted mistake 2: transposed state read */
                    const double s = (PLANTED(2) && dk == dv) ? S[j * dv + i] : S[i * dv + j];
                    acc += s * k[i];
                }
                m[j] = acc;
            }

        /* delta_j = (v_j - kv_mem_j) * beta_t */
        for (int j = 0; j < dv; ++j) {
            const double vj = load_elem(c->v, c->dtype, v_base + j);
            /* planted mistake 4: wrong sign of the memory */
            delta[j] = PLANTED(4) ? (vj + m[j]) * beta : (vj - m[j]) * beta;
        }

        /* S[i][j] += k_i * delta_j  (outer product k^T delta) */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] += k[i] * delta[j];

        /* o_j = sum_i S[i][j] q_i */
        if (c->o)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * q[i];
                c->o[v_base + j] = acc;
            }
    }
    if (c->hT) memcpy(c->hT + sbase, S, sizeof(double) * (size_t)dk * dv);
    free(S);
    free(q);
    free(k);
    free(m);
    free(delta);
}

/*
 * Gated delta rule over packed sequences, token by token in fp64.
 *   q,k [T_tot,Hk,dk], v [T_tot,H,dv] (dtype), g,beta [T_tot,H] (gate_dtype),
 *   cu_seqlens [N+1], h0 [N,H,dk,dv] (h0_dtype) or NULL for zeros,
 *   hT [N,H,dk,dv] double or NULL, o [T_tot,H,dv] double or NULL.
 * Value head h reads q and k of head h / (H / Hk) (grouped value heads: the
 * config's linear_num_value_heads may exceed linear_num_key_heads; H == Hk is
 * the plain layer). undecayed = 1 selects the [U] order (read, then decay).
 * Returns 0, or -1 on a bad argument.
 */
static int recurrence_impl(const void *q, const void *k, const void *v, int dtype,
                           const void *g, const void *beta, int gate_dtype,
                           const int64_t *cu_seqlens, int N, int H, int Hk, int dk, int dv,
                           double scale, int qk_l2norm, double eps, int undecayed,
                           const void *h0, int h0_dtype, double *hT, double *o, int n_threads,
                           int planted) {
    if (N < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || dk <= 0 || dv <= 0 || !cu_seqlens) return -1;
    rec_ctx c = {q, k, v, dtype, g, beta, gate_dtype, cu_seqlens, H, Hk, dk, dv, scale,
                 qk_l2norm, eps, undecayed, h0, h0_dtype, hT, o
#ifdef GDN_ORACLE_PIN_CHECK
                 , planted
#endif
    };
    (void)planted;
    run_items(rec_item, &c, (int64_t)N * H, n_threads);
    return 0;
}

int gdn_oracle_recurrence(const void *q, const void *k, const void *v, int dtype,
                          const void *g, const void *beta, int gate_dtype,
                          const int64_t *cu_seqlens, int N, int H, int Hk, int dk, int dv,
                          double scale, int qk_l2norm, double eps, int undecayed,
                          const void *h0, int h0_dtype, double *hT, double *o, int n_threads) {
    return recurrence_impl(q, k, v, dtype, g, beta, gate_dtype, cu_seqlens, N, H, Hk, dk, dv, scale,
                           qk_l2norm, eps, undecayed, h0, h0_dtype, hT, o, n_threads, 0);
}

#ifdef GDN_ORACLE_PIN_CHECK
/* gdn_oracle_recurrence with planted mistake `planted` (1..4; pin check only). */
int gdn_oracle_recurrence_planted(const void *q, const void *k, const void *v, int dtype,
                                  const void *g, const void *beta, int gate_dtype,
                                  const int64_t *cu_seqlens, int N, int H, int Hk, int dk, int dv,
                                  double scale, int qk_l2norm, double eps, int undecayed,
                                  const void *h0, int h0_dtype, double *hT, double *o,
                                  int n_threads, int planted) {
    if (planted < 1 || planted > 4) return -1;
    return recurrence_impl(q, k, v, dtype, g, beta, gate_dtype, cu_seqlens, N, H, Hk, dk, dv, scale,
                           qk_l2norm, eps, undecayed, h0, h0_dtype, hT, o, n_threads, planted);
}
#endif

/* ------------------------------------------------------------------------ */
/* Conv stage [C]: causal depthwise conv, SiLU, per-head L2 norm of q and k.  */
/* ------------------------------------------------------------------------ */

typedef struct {
    const void *x;
    int dtype;
    const void *w;
    int w_dtype;
    const int64_t *cu;
    int C, K;
    const void *state_in;
    int state_dtype;
    double *state_out;
    int apply_silu, qk_l2norm, n_qk, head_dim;
    double eps;
    double *y;
} conv_ctx;

/* Input of sequence n at relative position p (p < 0 reaches into the conv
 * state, whose column s holds relative position s - (K-1)). */
static double conv_input(const conv_ctx *c, int64_t n, int64_t p, int ch) {
    if (p >= 0) return load_elem(c->x, c->dtype, (c->cu[n] + p) * c->C + ch);
    const int64_t s = (c->K - 1) + p;
    if (!c->state_in || s < 0) return 0.0;
    return load_elem(c->state_in, c->state_dtype, (n * c->C + ch) * (int64_t)(c->K - 1) + s);
}

static void conv_item(void *vctx, int64_t n) {
    const conv_ctx *c = (const conv_ctx *)vctx;
    const int C = c->C, K = c->K;
    const int64_t T = c->cu[n + 1] - c->cu[n];
    for (int64_t t = 0; t < T; ++t) {
        double *yrow = c->y + (c->cu[n] + t) * C;
        for (int ch = 0; ch < C; ++ch) {
            /* PyTorch Conv1d cross-correlation with padding K-1, first T outputs:
             * y[t] = sum_j w[j] * x[t - (K-1) + j] */
            double acc = 0.0;
            for (int j = 0; j < K; ++j)
                acc += load_elem(c->w, c->w_dtype, (int64_t)ch * K + j) *
                       conv_input(c, n, t - (K - 1) + j, ch);
            if (c->apply_silu) acc = acc / (1.0 + exp(-acc)); /* SiLU(z) = z * sigmoid(z) */
            yrow[ch] = acc;
        }
        if (c->qk_l2norm)
            for (int base = 0; base + c->head_dim <= c->n_qk; base += c->head_dim)
                l2_normalise(yrow + base, c->head_dim, c->eps);
    }
    if (c->state_out)
        for (int ch = 0; ch < C; ++ch)
            for (int s = 0; s < K - 1; ++s)
                c->state_out[(n * C + ch) * (int64_t)(K - 1) + s] =
                    conv_input(c, n, T - (K - 1) + s, ch);
}

/*
 * Conv stage over packed sequences.
 *   x [T_tot,C] (dtype), w [C,K] (w_dtype), cu_seqlens [N+1],
 *   state_in [N,C,K-1] (state_dtype) or NULL for zeros, state_out [N,C,K-1]
 *   double or NULL, y [T_tot,C] double.
 * The first n_qk channels (q then k) are L2-normalised in groups of head_dim
 * when qk_l2norm is set. Returns 0, or -1 on a bad argument.
 */
int gdn_oracle_conv_silu(const void *x, int dtype, const void *w, int w_dtype,
                         const int64_t *cu_seqlens, int N, int C, int K,
                         const void *state_in, int state_dtype, double *state_out,
                         int apply_silu, int qk_l2norm, int n_qk, int head_dim, double eps,
                         double *y, int n_threads) {
    if (N < 0 || C <= 0 || K < 1 || !cu_seqlens || !y) return -1;
    if (qk_l2norm && (head_dim <= 0 || n_qk % head_dim != 0 || n_qk > C)) return -1;
    conv_ctx c = {x, dtype, w, w_dtype, cu_seqlens, C, K, state_in, state_dtype, state_out,
                  apply_silu, qk_l2norm, n_qk, head_dim, eps, y};
    run_items(conv_item, &c, N, n_threads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* fp64 chunkwise evaluator: an independent regrouping of [R] used only to   */
/* check that the chunk algebra (cumulative decay, UT transform with a unit  */
/* lower-triangular solve, inter-chunk state passing) is exact. Published    */
/* methods: "Parallelizing Linear Transformers with the Delta Rule over       */
/* Sequence Length" (Yang et al., 2024) and "Gated Delta Networks" (Yang,     */
/* Kautz, Hatamizadeh, 2024), restated here for the decay-first form.         */
/* ------------------------------------------------------------------------ */

typedef struct {
    rec_ctx r;
    int chunk;
} chunk_ctx;

static void chunk_item(void *vctx, int64_t item) {
    const chunk_ctx *cc = (const chunk_ctx *)vctx;
    const rec_ctx *c = &cc->r;
    const int H = c->H, Hk = c->Hk, dk = c->dk, dv = c->dv, Cs = cc->chunk;
    const int64_t n = item / H;
    const int h = (int)(item % H);
    const int hk = h / (H / Hk);
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *Q = (double *)malloc(sizeof(double) * Cs * dk);
    double *Kc = (double *)malloc(sizeof(double) * Cs * dk);
    double *V = (double *)malloc(sizeof(double) * Cs * dv);
    double *gam = (double *)malloc(sizeof(double) * Cs);
    double *grow = (double *)malloc(sizeof(double) * Cs);
    double *bet = (double *)malloc(sizeof(double) * Cs);
    double *A = (double *)malloc(sizeof(double) * Cs * Cs);
    double *Tm = (double *)malloc(sizeof(double) * Cs * Cs);
    double *W = (double *)malloc(sizeof(double) * Cs * dk);
    double *U = (double *)malloc(sizeof(double) * Cs * dv);
    double *Sn = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    const int64_t sbase = (n * H + h) * (int64_t)dk * dv;
    if (c->h0)
        for (int64_t e = 0; e < (int64_t)dk * dv; ++e) S[e] = load_elem(c->h0, c->h0_dtype, sbase + e);

    for (int64_t t0 = c->cu[n]; t0 < c->cu[n + 1]; t0 += Cs) {
        const int L = (int)((c->cu[n + 1] - t0) < Cs ? (c->cu[n + 1] - t0) : Cs);
        double acc_g = 0.0;
        for (int r = 0; r < L; ++r) {
            const int64_t t = t0 + r;
            for (int i = 0; i < dk; ++i) {
                Q[r * dk + i] = load_elem(c->q, c->dtype, (t * Hk + hk) * (int64_t)dk + i);
                Kc[r * dk + i] = load_elem(c->k, c->dtype, (t * Hk + hk) * (int64_t)dk + i);
            }
            if (c->qk_l2norm) {
                l2_normalise(Q + r * dk, dk, c->eps);
                l2_normalise(Kc + r * dk, dk, c->eps);
            }
            for (int i = 0; i < dk; ++i) Q[r * dk + i] *= c->scale;
            for (int j = 0; j < dv; ++j) V[r * dv + j] = load_elem(c->v, c->dtype, (t * H + h) * (int64_t)dv + j);
            acc_g += load_elem(c->g, c->gate_dtype, t * H + h);
            gam[r] = acc_g; /* gamma_r = sum_{i<=r} g_i */
            bet[r] = load_elem(c->beta, c->gate_dtype, t * H + h);
        }
        /* Decay of the row whose delta is being solved for: token r reads the
         * state after gamma_r of decay ([R]), or before its own decay, i.e. after
         * gamma_{r-1} = gamma_r - g_r ([U]; gamma_{-1} = 0). */
        for (int r = 0; r < L; ++r) grow[r] = c->undecayed ? (r > 0 ? gam[r - 1] : 0.0) : gam[r];
        /* A[r][j] = beta_r exp(grow_r - gamma_j) k_r.k_j for j < r */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double a = 0.0;
                if (j < r) {
                    double dot = 0.0;
                    for (int i = 0; i < dk; ++i) dot += Kc[r * dk + i] * Kc[j * dk + i];
                    a = bet[r] * exp(grow[r] - gam[j]) * dot;
                }
                A[r * Cs + j] = a;
            }
        /* Tm = (I + A)^{-1}, unit lower triangular, by forward substitution */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double s = (r == j) ? 1.0 : 0.0;
                if (j < r)
                    for (int m = j; m < r; ++m) s -= A[r * Cs + m] * Tm[m * Cs + j];
                Tm[r * Cs + j] = (j <= r) ? s : 0.0;
            }
        /* W = Tm diag(beta e^grow) K ; U = Tm diag(beta) V - W S */
        for (int r = 0; r < L; ++r) {
            for (int i = 0; i < dk; ++i) {
                double s = 0.0;
                for (int m = 0; m <= r; ++m) s += Tm[r * Cs + m] * bet[m] * exp(grow[m]) * Kc[m * dk + i];
                W[r * dk + i] = s;
            }
            for (int j = 0; j < dv; ++j) {
                double s = 0.0;
                for (int m = 0; m <= r; ++m) s += Tm[r * Cs + m] * bet[m] * V[m * dv + j];
                for (int i = 0; i < dk; ++i) s -= W[r * dk + i] * S[i * dv + j];
                U[r * dv + j] = s;
            }
        }
        /* O_r = e^{gamma_r} q_r S + sum_{m<=r} e^{gamma_r - gamma_m} (q_r.k_m) u_m */
        if (c->o)
            for (int r = 0; r < L; ++r)
                for (int j = 0; j < dv; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < dk; ++i) s += Q[r * dk + i] * S[i * dv + j];
                    s *= exp(gam[r]);
                    for (int m = 0; m <= r; ++m) {
                        double dot = 0.0;
                        for (int i = 0; i < dk; ++i) dot += Q[r * dk + i] * Kc[m * dk + i];
                        s += exp(gam[r] - gam[m]) * dot * U[m * dv + j];
                    }
                    c->o[((t0 + r) * H + h) * (int64_t)dv + j] = s;
                }
        /* S <- e^{gamma_L} S + sum_m e^{gamma_L - gamma_m} k_m u_m^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double s = exp(gam[L - 1]) * S[i * dv + j];
                for (int m = 0; m < L; ++m) s += exp(gam[L - 1] - gam[m]) * Kc[m * dk + i] * U[m * dv + j];
                Sn[i * dv + j] = s;
            }
        memcpy(S, Sn, sizeof(double) * (size_t)dk * dv);
    }
    if (c->hT) memcpy(c->hT + sbase, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(Q); free(Kc); free(V); free(gam); free(grow); free(bet); free(A); free(Tm);
    free(W); free(U); free(Sn);
}

int gdn_oracle_chunked(const void *q, const void *k, const void *v, int dtype,
                       const void *g, const void *beta, int gate_dtype,
                       const int64_t *cu_seqlens, int N, int H, int Hk, int dk, int dv,
                       double scale, int qk_l2norm, double eps, int undecayed,
                       const void *h0, int h0_dtype, double *hT, double *o,
                       int chunk, int n_threads) {
    if (N < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || dk <= 0 || dv <= 0 || chunk <= 0 || !cu_seqlens)
        return -1;
    chunk_ctx c = {{q, k, v, dtype, g, beta, gate_dtype, cu_seqlens, H, Hk, dk, dv, scale, qk_l2norm,
                    eps, undecayed, h0, h0_dtype, hT, o
#ifdef GDN_ORACLE_PIN_CHECK
                    , 0
#endif
                   },
                   chunk};
    run_items(chunk_item, &c, (int64_t)N * H, n_threads);
    return 0;
}
