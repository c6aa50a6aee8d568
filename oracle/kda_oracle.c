/*
 * kda_oracle.c -- plain, slow, fp64 CPU oracle for the Kimi Delta Attention (KDA)
 * gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The CUDA product path
 * never links, imports or calls it, and it shares no code, header, table or
 * helper with that path.
 *
 * What it follows (sources are the web pages the method is described on):
 *   [rec]    K3 article summaries (xhh.club tag page), item "KDA recurrence form":
 *            linear attention -> DeltaNet -> Gated DeltaNet lineage, per-channel
 *            decay, erase-then-write state update, one 128x128 state per head,
 *            per-head RMSNorm and a full-rank sigmoid output gate.
 *   [chunk]  same page, item "chunkwise parallel algorithm": recurrence between
 *            chunks, matrix products inside a chunk, the per-step log-decay is
 *            bounded below by -5; chunkwise and recurrent forms compute the same
 *            thing (training/prefill use the first, decode the second).
 *   [hybrid] same page, item "3:1 hybrid": full-rank sigmoid gate.
 *   [sys]    same page, item "training and inference systems": context
 *            parallelism decomposes into an associative prefix scan over segment
 *            transitions (not a plain sum of per-segment states).
 *   [self]   K3 paper walkthrough (nlpx.cn), section 6 "terminology and
 *            self-test": the -5 bound on the log-decay, KCP segment transitions.
 *
 * The pages give the method in words only.  The symbolic form used here is the
 * plainest reading of [rec]:
 *     l_t   = max(log_alpha_t, -5)                (per key channel)
 *     S'    = Diag(exp(l_t)) S_{t-1}              (per-channel decay)
 *     u_t   = beta_t (v_t - S'^T k_t)             (erase: what the state already
 *                                                  stores under key k_t)
 *     S_t   = S' + k_t u_t^T                       (= (I - b k k^T) D S + b k v^T)
 *     o_t   = scale * S_t^T q_t                    (read with the updated state)
 * S is dk x dv, row index = key channel.  Inputs are token-major, head-minor:
 * q,k,log_alpha [T,H,dk], v [T,H,dv], beta [T,H], states [N,H,dk,dv].
 *
 * Everything is fp64.  Inputs arrive as float32 arrays (bf16 values are exactly
 * representable in float32) and are widened exactly.
 *
 * Functions with no independent pin are marked in their comments; all the
 * functions below are pinned by tests/test_oracle_pins.py.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* thread pool over independent (sequence, head) units                       */
/* ------------------------------------------------------------------------ */

typedef void (*unit_fn)(void* ctx, int64_t unit);

typedef struct {
    unit_fn fn;
    void* ctx;
    int64_t n_units;
    int64_t next;
    pthread_mutex_t mu;
} pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        int64_t u = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (u >= p->n_units) break;
        p->fn(p->ctx, u);
    }
    return NULL;
}

OR_API int oracle_available_cores(void) {
    cpu_set_t set;
    CPU_ZERO(&set);
    if (sched_getaffinity(0, sizeof(set), &set) == 0) {
        int c = CPU_COUNT(&set);
        if (c > 0) return c;
    }
    return 1;
}

/* Runs fn over [0, n_units) on n_threads threads (<= 0: all available cores).
 * Returns the number of threads actually used. */
static int run_units(unit_fn fn, void* ctx, int64_t n_units, int n_threads) {
    if (n_threads <= 0) n_threads = oracle_available_cores();
    if (n_threads > n_units) n_threads = (int)(n_units > 0 ? n_units : 1);
    pool_t p;
    p.fn = fn; p.ctx = ctx; p.n_units = n_units; p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    if (n_threads <= 1) {
        pool_worker(&p);
    } else {
        pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
        for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
        for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&p.mu);
    return n_threads;
}

/* ------------------------------------------------------------------------ */
/* token-by-token recurrence                                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    const float *q, *k, *v, *log_alpha, *beta;
    const double* init_state;
    const int64_t* cu;
    int N, H, dk, dv, h_begin, h_end;
    double scale, la_floor;
    int erase;
    double* o;
    double* final_state;
} rec_ctx;

/* One (sequence n, head h) unit: walks the tokens of sequence n in order.
 * erase = 1 is KDA itself.  erase = 0 drops the -beta k k^T term (the write
 * becomes S += beta k v^T): gated linear attention, used only by the
 * reduction tests of the linear-attention lineage named in [rec]. */
static void rec_unit(void* vctx, int64_t unit) {
    const rec_ctx* c = (const rec_ctx*)vctx;
    const int nh = c->h_end - c->h_begin;
    const int n = (int)(unit / nh);
    const int h = c->h_begin + (int)(unit % nh);
    const int dk = c->dk, dv = c->dv, H = c->H;

    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* alpha = (double*)malloc(sizeof(double) * (size_t)dk);
    double* u = (double*)malloc(sizeof(double) * (size_t)dv);
    const size_t st_off = ((size_t)n * H + h) * (size_t)dk * dv;
    if (c->init_state)
        memcpy(S, c->init_state + st_off, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        const float* qt = c->q + ((size_t)t * H + h) * dk;
        const float* kt = c->k + ((size_t)t * H + h) * dk;
        const float* vt = c->v + ((size_t)t * H + h) * dv;
        const float* lt = c->log_alpha + ((size_t)t * H + h) * dk;
        const double bt = (double)c->beta[(size_t)t * H + h];

        /* per-channel decay, log-decay clamped below ([chunk], [self]) */
        for (int i = 0; i < dk; ++i) {
            double l = (double)lt[i];
            if (l < c->la_floor) l = c->la_floor;
            alpha[i] = exp(l);
        }
        /* S' = Diag(alpha) S */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= alpha[i];
        /* u = beta (v - S'^T k)   (erase form)  or  u = beta v  (no erase) */
        for (int j = 0; j < dv; ++j) {
            double sk = 0.0;
            if (c->erase)
                for (int i = 0; i < dk; ++i) sk += S[(size_t)i * dv + j] * (double)kt[i];
            u[j] = bt * ((double)vt[j] - sk);
        }
        /* S = S' + k u^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += (double)kt[i] * u[j];
        /* o = scale * S^T q */
        double* ot = c->o + ((size_t)t * H + h) * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * (double)qt[i];
            ot[j] = c->scale * acc;
        }
    }
    if (c->final_state) memcpy(c->final_state + st_off, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(alpha); free(u);
}

/* Token-by-token recurrence over N packed sequences (cu_seqlens [N+1]).
 * Only heads [h_begin, h_end) are computed; the other heads' outputs are left
 * untouched.  Returns the number of threads used, or -1 on bad arguments. */
OR_API int oracle_kda_recurrent(const float* q, const float* k, const float* v,
                                const float* log_alpha, const float* beta,
                                const double* init_state, const int64_t* cu_seqlens,
                                int N, int H, int dk, int dv, int h_begin, int h_end,
                                double scale, double la_floor, int erase,
                                double* o, double* final_state, int n_threads) {
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || h_begin < 0 || h_end > H || h_begin >= h_end)
        return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    rec_ctx c = {q, k, v, log_alpha, beta, init_state, cu_seqlens, N, H, dk, dv,
                 h_begin, h_end, scale, la_floor, erase, o, final_state};
    return run_units(rec_unit, &c, (int64_t)N * (h_end - h_begin), n_threads);
}

/* ------------------------------------------------------------------------ */
/* backward of the token-by-token recurrence (reverse-mode, fp64)            */
/* ------------------------------------------------------------------------ */
/*
 * The pages give no backward pass.  This is the exact gradient of the forward
 * definition above, taken step by step in reverse: given dL/do_t and dL/dS_T
 * it returns dL/dq, dL/dk, dL/dv, dL/dbeta, dL/dlog_alpha and dL/dS_0.  The
 * clamp l = max(log_alpha, floor) passes the gradient where log_alpha >= floor
 * (equality included) and blocks it below.  Per token, with r = v - S'^T k,
 * u = beta r and G = dL/dS_t (accumulated from later tokens):
 *     G     += scale q do^T                      dq  = scale S_t do
 *     dk     = G u                               du  = G^T k
 *     dbeta  = du . r                            dr  = beta du,  dv = dr
 *     dS'    = G - k dr^T                        dk -= S' dr
 *     dl     = alpha o rowsum(dS' o S_{t-1})     G  <- Diag(alpha) dS'
 * The forward states S_{t-1} are kept for the whole sequence (test sizes only).
 * Pinned by central finite differences of the forward (test_oracle_pins.py).
 */
typedef struct {
    const float *q, *k, *v, *log_alpha, *beta;
    const double* init_state;
    const double *d_o, *d_final;
    const int64_t* cu;
    int N, H, dk, dv;
    double scale, la_floor;
    double *dq, *dk_out, *dv_out, *dbeta, *dla, *d_init;
} bwd_ctx;

static void bwd_unit(void* vctx, int64_t unit) {
    const bwd_ctx* c = (const bwd_ctx*)vctx;
    const int n = (int)(unit / c->H), h = (int)(unit % c->H);
    const int dk = c->dk, dv = c->dv, H = c->H;
    const int64_t t0 = c->cu[n], L = c->cu[n + 1] - c->cu[n];
    const size_t SZ = (size_t)dk * dv;
    const size_t st_off = ((size_t)n * H + h) * SZ;
    /* forward: the state before every token, u and r of every token */
    double* Sb = malloc(sizeof(double) * SZ * (size_t)(L + 1));
    double* R = malloc(sizeof(double) * (size_t)dv * (size_t)(L > 0 ? L : 1));
    double* alpha = malloc(sizeof(double) * (size_t)dk * (size_t)(L > 0 ? L : 1));
    if (c->init_state) memcpy(Sb, c->init_state + st_off, sizeof(double) * SZ);
    else memset(Sb, 0, sizeof(double) * SZ);
    for (int64_t tt = 0; tt < L; ++tt) {
        const int64_t t = t0 + tt;
        const float* kt = c->k + ((size_t)t * H + h) * dk;
        const float* vt = c->v + ((size_t)t * H + h) * dv;
        const float* lt = c->log_alpha + ((size_t)t * H + h) * dk;
        const double bt = (double)c->beta[(size_t)t * H + h];
        const double* Sp = Sb + SZ * (size_t)tt;
        double* Sn = Sb + SZ * (size_t)(tt + 1);
        double* al = alpha + (size_t)dk * tt;
        double* r = R + (size_t)dv * tt;
        for (int i = 0; i < dk; ++i) {
            double l = (double)lt[i];
            if (l < c->la_floor) l = c->la_floor;
            al[i] = exp(l);
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) Sn[(size_t)i * dv + j] = al[i] * Sp[(size_t)i * dv + j];
        for (int j = 0; j < dv; ++j) {
            double sk = 0.0;
            for (int i = 0; i < dk; ++i) sk += Sn[(size_t)i * dv + j] * (double)kt[i];
            r[j] = (double)vt[j] - sk;
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) Sn[(size_t)i * dv + j] += (double)kt[i] * bt * r[j];
    }
    /* reverse sweep */
    double* G = malloc(sizeof(double) * SZ);
    double* dSp = malloc(sizeof(double) * SZ);
    double* du = malloc(sizeof(double) * (size_t)dv);
    double* dr = malloc(sizeof(double) * (size_t)dv);
    if (c->d_final) memcpy(G, c->d_final + st_off, sizeof(double) * SZ);
    else memset(G, 0, sizeof(double) * SZ);
    for (int64_t tt = L - 1; tt >= 0; --tt) {
        const int64_t t = t0 + tt;
        const size_t ti = (size_t)t * H + h;
        const float* qt = c->q + ti * dk;
        const float* kt = c->k + ti * dk;
        const float* lt = c->log_alpha + ti * dk;
        const double bt = (double)c->beta[ti];
        const double* dot = c->d_o + ti * dv;
        const double* Sprev = Sb + SZ * (size_t)tt;      /* S_{t-1} */
        const double* St = Sb + SZ * (size_t)(tt + 1);   /* S_t */
        const double* al = alpha + (size_t)dk * tt;
        const double* r = R + (size_t)dv * tt;
        /* o_t = scale S_t^T q_t */
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) acc += St[(size_t)i * dv + j] * dot[j];
            c->dq[ti * dk + i] = c->scale * acc;
            for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += c->scale * (double)qt[i] * dot[j];
        }
        /* S_t = S' + k u^T */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += G[(size_t)i * dv + j] * (double)kt[i];
            du[j] = acc;
        }
        double db = 0.0;
        for (int j = 0; j < dv; ++j) {
            db += du[j] * r[j];
            dr[j] = bt * du[j];
            c->dv_out[ti * dv + j] = dr[j];
        }
        c->dbeta[ti] = db;
        for (int i = 0; i < dk; ++i) {
            double acc_u = 0.0, acc_r = 0.0;
            for (int j = 0; j < dv; ++j) {
                const double sp = al[i] * Sprev[(size_t)i * dv + j];   /* S' */
                acc_u += G[(size_t)i * dv + j] * bt * r[j];
                acc_r += sp * dr[j];
            }
            c->dk_out[ti * dk + i] = acc_u - acc_r;
        }
        /* S' = Diag(alpha) S_{t-1};  dS' = G - k dr^T */
        for (int i = 0; i < dk; ++i) {
            double da = 0.0;
            for (int j = 0; j < dv; ++j) {
                const double g = G[(size_t)i * dv + j] - (double)kt[i] * dr[j];
                dSp[(size_t)i * dv + j] = g;
                da += g * Sprev[(size_t)i * dv + j];
            }
            const double pass = ((double)lt[i] >= c->la_floor) ? 1.0 : 0.0;
            c->dla[ti * dk + i] = pass * al[i] * da;
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] = al[i] * dSp[(size_t)i * dv + j];
    }
    if (c->d_init) memcpy(c->d_init + st_off, G, sizeof(double) * SZ);
    free(Sb); free(R); free(alpha); free(G); free(dSp); free(du); free(dr);
}

/* Backward of oracle_kda_recurrent (erase form) over N packed sequences.
 * d_o [T,H,dv]; d_final [N,H,dk,dv] or NULL (zero).  Outputs (fp64): dq, dk
 * [T,H,dk], dv [T,H,dv], dbeta [T,H], dlog_alpha [T,H,dk], d_init [N,H,dk,dv]
 * or NULL.  Returns the number of threads used, or -1 on bad arguments. */
OR_API int oracle_kda_recurrent_bwd(const float* q, const float* k, const float* v,
                                    const float* log_alpha, const float* beta,
                                    const double* init_state, const int64_t* cu_seqlens,
                                    const double* d_o, const double* d_final,
                                    int N, int H, int dk, int dv, double scale, double la_floor,
                                    double* dq, double* dk_out, double* dv_out, double* dbeta,
                                    double* dlog_alpha, double* d_init, int n_threads) {
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    bwd_ctx c = {q, k, v, log_alpha, beta, init_state, d_o, d_final, cu_seqlens, N, H, dk, dv,
                 scale, la_floor, dq, dk_out, dv_out, dbeta, dlog_alpha, d_init};
    return run_units(bwd_unit, &c, (int64_t)N * H, n_threads);
}

/* ------------------------------------------------------------------------ */
/* naive chunkwise form (fp64), the same result reached by matrix products   */
/* inside each chunk and a recurrence between chunks ([chunk]).              */
/* ------------------------------------------------------------------------ */
/*
 * Per chunk of L <= C tokens starting from state S0 (g = in-chunk cumulative
 * sum of the clamped log-decays, Gam_t = exp(g_t), a dk-vector per token):
 *   A[t][s] = sum_c k_tc k_sc exp(g_tc - g_sc)            s < t
 *   P[t][s] = sum_c q_tc k_sc exp(g_tc - g_sc)            s <= t
 *   T       = (I + Diag(beta) A)^(-1) Diag(beta)           (forward substitution)
 *   W       = T (K o Gam),   Ut = T V
 *   U       = Ut - W S0
 *   O       = scale * ((Q o Gam) S0 + P U)
 *   S_L     = Diag(Gam_L) S0 + (K o Gam_L / Gam)^T U
 * Exponent differences are formed directly in fp64 (no reference points).
 */
typedef struct {
    const float *q, *k, *v, *log_alpha, *beta;
    const double* init_state;
    const int64_t* cu;
    int N, H, dk, dv, C;
    double scale, la_floor;
    double* o;
    double* final_state;
} chunk_ctx;

static void chunk_unit(void* vctx, int64_t unit) {
    const chunk_ctx* c = (const chunk_ctx*)vctx;
    const int n = (int)(unit / c->H), h = (int)(unit % c->H);
    const int dk = c->dk, dv = c->dv, H = c->H, C = c->C;
    double* S = calloc((size_t)dk * dv, sizeof(double));
    double* g = malloc(sizeof(double) * (size_t)C * dk);
    double* A = malloc(sizeof(double) * (size_t)C * C);
    double* P = malloc(sizeof(double) * (size_t)C * C);
    double* Tm = malloc(sizeof(double) * (size_t)C * C);
    double* W = malloc(sizeof(double) * (size_t)C * dk);
    double* Ut = malloc(sizeof(double) * (size_t)C * dv);
    double* U = malloc(sizeof(double) * (size_t)C * dv);
    double* Snew = malloc(sizeof(double) * (size_t)dk * dv);
    const size_t st_off = ((size_t)n * H + h) * (size_t)dk * dv;
    if (c->init_state) memcpy(S, c->init_state + st_off, sizeof(double) * (size_t)dk * dv);

#define QV(t, i) ((double)c->q[((size_t)(t) * H + h) * dk + (i)])
#define KV(t, i) ((double)c->k[((size_t)(t) * H + h) * dk + (i)])
#define VV(t, j) ((double)c->v[((size_t)(t) * H + h) * dv + (j)])
#define BV(t) ((double)c->beta[(size_t)(t) * H + h])

    for (int64_t t0 = c->cu[n]; t0 < c->cu[n + 1]; t0 += C) {
        const int L = (int)((c->cu[n + 1] - t0) < C ? (c->cu[n + 1] - t0) : C);
        /* g: in-chunk cumulative log-decay */
        for (int i = 0; i < dk; ++i) {
            double run = 0.0;
            for (int t = 0; t < L; ++t) {
                double l = (double)c->log_alpha[((size_t)(t0 + t) * H + h) * dk + i];
                if (l < c->la_floor) l = c->la_floor;
                run += l;
                g[(size_t)t * dk + i] = run;
            }
        }
        /* A, P */
        for (int t = 0; t < L; ++t)
            for (int s = 0; s < L; ++s) {
                double a = 0.0, p = 0.0;
                if (s <= t)
                    for (int i = 0; i < dk; ++i) {
                        double e = exp(g[(size_t)t * dk + i] - g[(size_t)s * dk + i]);
                        a += KV(t0 + t, i) * KV(t0 + s, i) * e;
                        p += QV(t0 + t, i) * KV(t0 + s, i) * e;
                    }
                A[(size_t)t * C + s] = (s < t) ? a : 0.0;
                P[(size_t)t * C + s] = p;
            }
        /* T = (I + Diag(beta) A)^(-1) Diag(beta): row t of X = (I+N)^(-1) is
           e_t - sum_{s<t} N[t][s] X[s], N = Diag(beta) A; then T = X Diag(beta). */
        for (int t = 0; t < L; ++t) {
            for (int s = 0; s < L; ++s) Tm[(size_t)t * C + s] = (s == t) ? 1.0 : 0.0;
            for (int r = 0; r < t; ++r) {
                double nr = BV(t0 + t) * A[(size_t)t * C + r];
                if (nr != 0.0)
                    for (int s = 0; s <= r; ++s) Tm[(size_t)t * C + s] -= nr * Tm[(size_t)r * C + s];
            }
        }
        for (int t = 0; t < L; ++t)
            for (int s = 0; s < L; ++s) Tm[(size_t)t * C + s] *= BV(t0 + s);
        /* W = T (K o Gam), Ut = T V */
        for (int t = 0; t < L; ++t) {
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int s = 0; s < L; ++s)
                    acc += Tm[(size_t)t * C + s] * KV(t0 + s, i) * exp(g[(size_t)s * dk + i]);
                W[(size_t)t * dk + i] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int s = 0; s < L; ++s) acc += Tm[(size_t)t * C + s] * VV(t0 + s, j);
                Ut[(size_t)t * dv + j] = acc;
            }
        }
        /* U = Ut - W S0 */
        for (int t = 0; t < L; ++t)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += W[(size_t)t * dk + i] * S[(size_t)i * dv + j];
                U[(size_t)t * dv + j] = Ut[(size_t)t * dv + j] - acc;
            }
        /* O = scale ((Q o Gam) S0 + P U) */
        for (int t = 0; t < L; ++t)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i)
                    acc += QV(t0 + t, i) * exp(g[(size_t)t * dk + i]) * S[(size_t)i * dv + j];
                for (int s = 0; s <= t; ++s) acc += P[(size_t)t * C + s] * U[(size_t)s * dv + j];
                c->o[((size_t)(t0 + t) * H + h) * dv + j] = c->scale * acc;
            }
        /* S_L = Diag(Gam_L) S0 + (K o Gam_L/Gam)^T U */
        for (int i = 0; i < dk; ++i) {
            const double gl = g[(size_t)(L - 1) * dk + i];
            for (int j = 0; j < dv; ++j) {
                double acc = exp(gl) * S[(size_t)i * dv + j];
                for (int s = 0; s < L; ++s)
                    acc += KV(t0 + s, i) * exp(gl - g[(size_t)s * dk + i]) * U[(size_t)s * dv + j];
                Snew[(size_t)i * dv + j] = acc;
            }
        }
        memcpy(S, Snew, sizeof(double) * (size_t)dk * dv);
    }
#undef QV
#undef KV
#undef VV
#undef BV
    if (c->final_state) memcpy(c->final_state + st_off, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(g); free(A); free(P); free(Tm); free(W); free(Ut); free(U); free(Snew);
}

/* Naive chunkwise form with chunk size C (chunks restart at each sequence). */
OR_API int oracle_kda_chunkwise(const float* q, const float* k, const float* v,
                                const float* log_alpha, const float* beta,
                                const double* init_state, const int64_t* cu_seqlens,
                                int N, int H, int dk, int dv, int C, double scale,
                                double la_floor, double* o, double* final_state,
                                int n_threads) {
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || C <= 0) return -1;
    chunk_ctx c = {q, k, v, log_alpha, beta, init_state, cu_seqlens, N, H, dk, dv, C,
                   scale, la_floor, o, final_state};
    return run_units(chunk_unit, &c, (int64_t)N * H, n_threads);
}

/* ------------------------------------------------------------------------ */
/* segment transition (affine map of the state over a whole segment)        */
/* ------------------------------------------------------------------------ */
/*
 * For one head and one segment of L tokens (one chunk of size L in the form
 * above), the state map is affine:  S_out = M S_in + Bm, with
 *     M  = Diag(Gam_L) - (K o Gam_L/Gam)^T W      (dk x dk)
 *     Bm = (K o Gam_L/Gam)^T Ut                   (dk x dv)
 * These are the segment transitions that context parallelism composes by an
 * associative prefix scan ([sys], [self]).  Inputs are one head's arrays:
 * q unused; k,log_alpha [L,dk], v [L,dv], beta [L].
 */
OR_API int oracle_kda_segment_transition(const float* k, const float* v,
                                         const float* log_alpha, const float* beta,
                                         int L, int dk, int dv, double la_floor,
                                         double* M, double* Bm) {
    if (L <= 0 || dk <= 0 || dv <= 0) return -1;
    double* g = malloc(sizeof(double) * (size_t)L * dk);
    double* A = calloc((size_t)L * L, sizeof(double));
    double* Tm = calloc((size_t)L * L, sizeof(double));
    double* W = malloc(sizeof(double) * (size_t)L * dk);
    double* Ut = malloc(sizeof(double) * (size_t)L * dv);
    for (int i = 0; i < dk; ++i) {
        double run = 0.0;
        for (int t = 0; t < L; ++t) {
            double l = (double)log_alpha[(size_t)t * dk + i];
            if (l < la_floor) l = la_floor;
            run += l;
            g[(size_t)t * dk + i] = run;
        }
    }
    for (int t = 0; t < L; ++t)
        for (int s = 0; s < t; ++s) {
            double a = 0.0;
            for (int i = 0; i < dk; ++i)
                a += (double)k[(size_t)t * dk + i] * (double)k[(size_t)s * dk + i] *
                     exp(g[(size_t)t * dk + i] - g[(size_t)s * dk + i]);
            A[(size_t)t * L + s] = a;
        }
    for (int t = 0; t < L; ++t) {
        Tm[(size_t)t * L + t] = 1.0;
        for (int r = 0; r < t; ++r) {
            double nr = (double)beta[t] * A[(size_t)t * L + r];
            for (int s = 0; s <= r; ++s) Tm[(size_t)t * L + s] -= nr * Tm[(size_t)r * L + s];
        }
    }
    for (int t = 0; t < L; ++t)
        for (int s = 0; s < L; ++s) Tm[(size_t)t * L + s] *= (double)beta[s];
    for (int t = 0; t < L; ++t) {
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int s = 0; s < L; ++s)
                acc += Tm[(size_t)t * L + s] * (double)k[(size_t)s * dk + i] * exp(g[(size_t)s * dk + i]);
            W[(size_t)t * dk + i] = acc;
        }
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int s = 0; s < L; ++s) acc += Tm[(size_t)t * L + s] * (double)v[(size_t)s * dv + j];
            Ut[(size_t)t * dv + j] = acc;
        }
    }
    for (int i = 0; i < dk; ++i) {
        const double gl = g[(size_t)(L - 1) * dk + i];
        for (int i2 = 0; i2 < dk; ++i2) {
            double acc = (i == i2) ? exp(gl) : 0.0;
            for (int s = 0; s < L; ++s)
                acc -= (double)k[(size_t)s * dk + i] * exp(gl - g[(size_t)s * dk + i]) * W[(size_t)s * dk + i2];
            M[(size_t)i * dk + i2] = acc;
        }
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int s = 0; s < L; ++s)
                acc += (double)k[(size_t)s * dk + i] * exp(gl - g[(size_t)s * dk + i]) * Ut[(size_t)s * dv + j];
            Bm[(size_t)i * dv + j] = acc;
        }
    }
    free(g); free(A); free(Tm); free(W); free(Ut);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* per-head RMSNorm + full-rank sigmoid output gate ([rec], [hybrid])        */
/* ------------------------------------------------------------------------ */
/*
 * For each row r (one token of one head, dv values):
 *     y_rj = o_rj / sqrt(mean_j o_rj^2 + eps) * w_j * sigmoid(g_rj)
 * w is a per-channel [dv] weight shared by all heads (NULL = ones).  The pages
 * name the norm and the gate but not eps, the weight or their order; this is
 * the reading used throughout (norm, then weight, then gate).
 */
OR_API int oracle_gate_norm(const double* o, const float* g, const float* w, double eps,
                            int64_t rows, int dv, double* y) {
    if (rows < 0 || dv <= 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const double* orow = o + (size_t)r * dv;
        double ms = 0.0;
        for (int j = 0; j < dv; ++j) ms += orow[j] * orow[j];
        ms /= (double)dv;
        const double inv = 1.0 / sqrt(ms + eps);
        for (int j = 0; j < dv; ++j) {
            const double gj = (double)g[(size_t)r * dv + j];
            const double sig = 1.0 / (1.0 + exp(-gj));
            const double wj = w ? (double)w[j] : 1.0;
            y[(size_t)r * dv + j] = orow[j] * inv * wj * sig;
        }
    }
    return 0;
}
