/*
 * Gated delta-rule oracle: plain fp64 token-by-token recurrence on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (state S has shape d_v x d_k, row i = value channel,
 * column j = key channel):
 *
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * with alpha_t = exp(g_t).  g_t is a scalar per head or a vector over the key
 * channels.  Sources:
 *   - "Decoding Hybrid Linear Attention Architectures", section 3, items 2
 *     (delta rule), 3 (gated delta rule, scalar gate) and 6 (Gated Delta
 *     Attention, per-channel gate), plus the single-step pseudocode under
 *     item 6, which fixes the order: decay, then erase along k_t, then write.
 *   - "Linear Attention Variants (RetNet, GLA, DeltaNet, Based)", section
 *     "DeltaNet: Error-Correcting Writes": the update written as
 *     S + beta v k^T - beta (S k) k^T, i.e. read what k_t maps to, subtract
 *     it, write the new value.  That is the form coded below.
 *   - "Decoding Hybrid Linear Attention Architectures", section 5 (the
 *     gates are accumulated in log space): the gate enters as g = log alpha.
 *
 * Readings where the pages are loose (each also listed in the design notes):
 *   - the output reads the state after the write (o_t = S_t q_t);
 *   - no 1/sqrt(d_k) query scale (no page applies one);
 *   - for a per-channel gate the decay scales the key axis of S and comes
 *     before the erase (pseudocode order under section 3 item 6).
 *
 * Inputs q, k, v are either fp32 or bf16 (raw 16-bit patterns); bf16 is
 * widened exactly (bit shift) and all arithmetic is in double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };
enum { OR_GATE_SCALAR = 0, OR_GATE_PER_CHANNEL = 1 };

/* Exact widening of one input element to double. */
static double load_elem(const void *base, size_t idx, int dtype) {
    if (dtype == OR_F64) return ((const double *)base)[idx];
    if (dtype == OR_F32) return (double)((const float *)base)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    const void *q, *k, *v;
    int in_dtype;
    const float *g;
    int gate_kind;
    const float *beta;
    const double *g64, *beta64; /* fp64 gates (take the place of g, beta when set) */
    const double *S0; /* may be NULL: zero initial state */
    double *o;
    double *S_T;      /* may be NULL */
    int B, T, H, dk, dv;
    int next;         /* shared work counter over (b, h) */
    pthread_mutex_t lock;
} job_t;

static double gate_at(const job_t *J, size_t idx) {
    return J->g64 ? J->g64[idx] : (double)J->g[idx];
}

/*
 * One (b, h) pair: the recurrence over t = 0..T-1.
 * Layouts: q,k [B,T,H,dk]; v,o [B,T,H,dv]; g [B,T,H] or [B,T,H,dk];
 * beta [B,T,H]; S0,S_T [B,H,dv,dk].
 */
static void run_head(job_t *J, int b, int h) {
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *kk = (double *)malloc(sizeof(double) * dk);
    double *qq = (double *)malloc(sizeof(double) * dk);
    double *alpha = (double *)malloc(sizeof(double) * dk);
    double *p = (double *)malloc(sizeof(double) * dv);
    const size_t sidx = ((size_t)b * H + h) * (size_t)dv * dk;
    if (J->S0)
        memcpy(S, J->S0 + sidx, sizeof(double) * (size_t)dv * dk);
    else
        memset(S, 0, sizeof(double) * (size_t)dv * dk);

    for (int t = 0; t < T; ++t) {
        const size_t tok = ((size_t)b * T + t) * H + h;
        for (int j = 0; j < dk; ++j) {
            kk[j] = load_elem(J->k, tok * dk + j, J->in_dtype);
            qq[j] = load_elem(J->q, tok * dk + j, J->in_dtype);
        }
        if (J->gate_kind == OR_GATE_PER_CHANNEL) {
            for (int j = 0; j < dk; ++j) alpha[j] = exp(gate_at(J, tok * dk + j));
        } else {
            const double a = exp(gate_at(J, tok));
            for (int j = 0; j < dk; ++j) alpha[j] = a;
        }
        const double beta = J->beta64 ? J->beta64[tok] : (double)J->beta[tok];

        /* 1. decay: S <- S Diag(alpha)  (scales the key axis) */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) S[(size_t)i * dk + j] *= alpha[j];

        /* 2. read what k_t currently maps to: p = S k */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kk[j];
            p[i] = acc;
        }

        /* 3. erase-and-write: S <- S + beta (v - p) k^T */
        for (int i = 0; i < dv; ++i) {
            const double vi = load_elem(J->v, tok * dv + i, J->in_dtype);
            const double c = beta * (vi - p[i]);
            for (int j = 0; j < dk; ++j) S[(size_t)i * dk + j] += c * kk[j];
        }

        /* 4. read-out after the write: o = S q */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qq[j];
            J->o[tok * dv + i] = acc;
        }
    }
    if (J->S_T) memcpy(J->S_T + sidx, S, sizeof(double) * (size_t)dv * dk);
    free(S);
    free(kk);
    free(qq);
    free(alpha);
    free(p);
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int w = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (w >= J->B * J->H) break;
        run_head(J, w / J->H, w % J->H);
    }
    return NULL;
}

/*
 * Forward over a whole sequence.  Returns 0 on success, -1 on a bad
 * argument.  nthreads <= 0 means one thread per online core.
 */
static int run_job(job_t *Jp, int nthreads);

int oracle_gdr_fwd(const void *q, const void *k, const void *v, int in_dtype,
                   const float *g, int gate_kind, const float *beta,
                   const double *S0, double *o, double *S_T, int B, int T,
                   int H, int dk, int dv, int nthreads) {
    if (!q || !k || !v || !g || !beta || !o) return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (in_dtype != OR_F32 && in_dtype != OR_BF16) return -1;
    if (gate_kind != OR_GATE_SCALAR && gate_kind != OR_GATE_PER_CHANNEL) return -1;
    job_t J;
    J.q = q; J.k = k; J.v = v; J.in_dtype = in_dtype;
    J.g = g; J.gate_kind = gate_kind; J.beta = beta;
    J.g64 = NULL; J.beta64 = NULL;
    J.S0 = S0; J.o = o; J.S_T = S_T;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    return run_job(&J, nthreads);
}

/*
 * The same forward with every input in fp64 (q, k, v, g = log alpha, beta):
 * for inputs that are themselves computed in fp64, such as the output of the
 * prologue (normalised q, k and gates mapped from their logits).
 */
int oracle_gdr_fwd_f64(const double *q, const double *k, const double *v,
                       const double *g, int gate_kind, const double *beta,
                       const double *S0, double *o, double *S_T, int B, int T,
                       int H, int dk, int dv, int nthreads) {
    if (!q || !k || !v || !g || !beta || !o) return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (gate_kind != OR_GATE_SCALAR && gate_kind != OR_GATE_PER_CHANNEL) return -1;
    job_t J;
    J.q = q; J.k = k; J.v = v; J.in_dtype = OR_F64;
    J.g = NULL; J.gate_kind = gate_kind; J.beta = NULL;
    J.g64 = g; J.beta64 = beta;
    J.S0 = S0; J.o = o; J.S_T = S_T;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    return run_job(&J, nthreads);
}

/* Runs every (b, h) of the job on nthreads threads (<= 0: one). */
static int run_job(job_t *Jp, int nthreads) {
    job_t J = *Jp;
    const int B = J.B, H = J.H;
    J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    int n = nthreads;
    if (n <= 0) n = 1;
    if (n > B * H) n = B * H;
    if (n <= 1) {
        worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n);
        for (int i = 0; i < n; ++i) pthread_create(&th[i], NULL, worker, &J);
        for (int i = 0; i < n; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * One recurrent step for N independent states ("Decoding Hybrid Linear
 * Attention Architectures", section 6: a constant-cost update of the
 * fixed-size state per decoded token).  S [N,H,dv,dk] is updated in place;
 * q,k [N,H,dk]; v,o [N,H,dv]; g [N,H] or [N,H,dk]; beta [N,H].
 * It is the forward above with T = 1 and S_T aliasing S0.
 */
int oracle_gdr_step(const void *q, const void *k, const void *v, int in_dtype,
                    const float *g, int gate_kind, const float *beta, double *S,
                    double *o, int N, int H, int dk, int dv, int nthreads) {
    if (!S) return -1;
    return oracle_gdr_fwd(q, k, v, in_dtype, g, gate_kind, beta, S, o, S, N, 1,
                          H, dk, dv, nthreads);
}

/*
 * Gated linear attention (additive write, no erase):
 *
 *     S_t = S_{t-1} Diag(alpha_t) + v_t k_t^T,    o_t = S_t q_t
 *
 * Source: "Decoding Hybrid Linear Attention Architectures", section 3 item 4
 * (GLA family: channel-wise forgetting, the write reverts to accumulation);
 * "Linear Attention Variants", GLA section (the same recurrence in the
 * transposed convention).  The gate enters as g = log alpha, scalar per head
 * or per key channel as above; the output reads the state after the write.
 * A separate plain loop: it shares nothing with the delta-rule one.
 */
typedef struct {
    const void *q, *k, *v;
    int in_dtype;
    const float *g;
    int gate_kind;
    const double *S0;
    double *o;
    double *S_T;
    int B, T, H, dk, dv;
    int next;
    pthread_mutex_t lock;
} gla_job_t;

static void gla_head(gla_job_t *J, int b, int h) {
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *kk = (double *)malloc(sizeof(double) * dk);
    double *qq = (double *)malloc(sizeof(double) * dk);
    double *alpha = (double *)malloc(sizeof(double) * dk);
    const size_t sidx = ((size_t)b * H + h) * (size_t)dv * dk;
    if (J->S0)
        memcpy(S, J->S0 + sidx, sizeof(double) * (size_t)dv * dk);
    else
        memset(S, 0, sizeof(double) * (size_t)dv * dk);
    for (int t = 0; t < T; ++t) {
        const size_t tok = ((size_t)b * T + t) * H + h;
        for (int j = 0; j < dk; ++j) {
            kk[j] = load_elem(J->k, tok * dk + j, J->in_dtype);
            qq[j] = load_elem(J->q, tok * dk + j, J->in_dtype);
            alpha[j] = exp((double)(J->gate_kind == OR_GATE_PER_CHANNEL ? J->g[tok * dk + j]
                                                                        : J->g[tok]));
        }
        /* decay the key axis, then add the outer product v_t k_t^T */
        for (int i = 0; i < dv; ++i) {
            const double vi = load_elem(J->v, tok * dv + i, J->in_dtype);
            for (int j = 0; j < dk; ++j)
                S[(size_t)i * dk + j] = S[(size_t)i * dk + j] * alpha[j] + vi * kk[j];
        }
        /* read-out after the write */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qq[j];
            J->o[tok * dv + i] = acc;
        }
    }
    if (J->S_T) memcpy(J->S_T + sidx, S, sizeof(double) * (size_t)dv * dk);
    free(S);
    free(kk);
    free(qq);
    free(alpha);
}

static void *gla_worker(void *arg) {
    gla_job_t *J = (gla_job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int w = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (w >= J->B * J->H) break;
        gla_head(J, w / J->H, w % J->H);
    }
    return NULL;
}

int oracle_gla_fwd(const void *q, const void *k, const void *v, int in_dtype, const float *g,
                   int gate_kind, const double *S0, double *o, double *S_T, int B, int T, int H,
                   int dk, int dv, int nthreads) {
    if (!q || !k || !v || !g || !o || B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (in_dtype != OR_F32 && in_dtype != OR_BF16) return -1;
    if (gate_kind != OR_GATE_SCALAR && gate_kind != OR_GATE_PER_CHANNEL) return -1;
    gla_job_t J;
    J.q = q; J.k = k; J.v = v; J.in_dtype = in_dtype; J.g = g; J.gate_kind = gate_kind;
    J.S0 = S0; J.o = o; J.S_T = S_T;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    int nt = nthreads > 0 ? nthreads : 1;
    if (nt > B * H) nt = B * H > 0 ? B * H : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nt);
    for (int i = 0; i < nt; ++i) pthread_create(&th[i], NULL, gla_worker, &J);
    for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * Backward of the gated delta-rule recurrence (reverse mode over tokens),
 * for training: given dL/do_t and dL/dS_T, the gradients of q, k, v,
 * g = log alpha, beta and S0.  "Decoding Hybrid Linear Attention
 * Architectures", section 5 (backpropagation through the same recurrence,
 * with recomputation); here the plainest form: the forward is run once,
 * keeping every state, then the steps are undone in reverse.
 *
 * One step, as in oracle_gdr_fwd:
 *     S' = S_{t-1} Diag(alpha)          p = S' k        u = beta (v - p)
 *     S_t = S' + u k^T                  o = S_t q
 * With G = dL/dS_t (dS_T at t = T, plus each later step's contribution):
 *     G   += do q^T,          dq = S_t^T do
 *     du   = G k,             dk = G^T u (+ S'^T dp below)
 *     dbeta = du . (v - p),   dv = beta du,   dp = -beta du
 *     dS'  = G + dp k^T,      dk += S'^T dp
 *     dg_j = sum_i S'[i][j] dS'[i][j]   (summed over j for a scalar gate)
 *     dS_{t-1} = dS' Diag(alpha)
 * dS0 = G after the first step.  Inputs as oracle_gdr_fwd; dout [B,T,H,dv]
 * and dS_T [B,H,dv,dk] (NULL: zero) in double; outputs in double, same
 * layouts as the inputs (dg [B,T,H] or [B,T,H,dk]).
 */
typedef struct {
    const void *q, *k, *v;
    int in_dtype;
    const float *g;
    int gate_kind;
    const float *beta;
    const double *S0, *dout, *dST;
    double *dq, *dk, *dv, *dg, *dbeta, *dS0;
    int B, T, H, dk_, dv_;
    int next;
    pthread_mutex_t lock;
} bwd_job_t;

static void bwd_head(bwd_job_t *J, int b, int h) {
    const int T = J->T, H = J->H, dk = J->dk_, dv = J->dv_;
    const size_t SS = (size_t)dv * dk;
    /* all states S_0 .. S_T, and the decayed S'_t of every step */
    double *St = (double *)malloc(sizeof(double) * SS * (size_t)(T + 1));
    double *Sp = (double *)malloc(sizeof(double) * SS * (size_t)(T > 0 ? T : 1));
    double *G = (double *)malloc(sizeof(double) * SS);
    double *dSp = (double *)malloc(sizeof(double) * SS);
    double *kk = (double *)malloc(sizeof(double) * dk);
    double *qq = (double *)malloc(sizeof(double) * dk);
    double *al = (double *)malloc(sizeof(double) * dk);
    double *vv = (double *)malloc(sizeof(double) * dv);
    double *pp = (double *)malloc(sizeof(double) * dv);
    double *uu = (double *)malloc(sizeof(double) * dv);
    double *du = (double *)malloc(sizeof(double) * dv);
    double *dp = (double *)malloc(sizeof(double) * dv);
    const size_t sidx = ((size_t)b * H + h) * SS;
    if (J->S0)
        memcpy(St, J->S0 + sidx, sizeof(double) * SS);
    else
        memset(St, 0, sizeof(double) * SS);

#define LOAD_TOKEN(t)                                                          \
    const size_t tok = ((size_t)b * T + (t)) * H + h;                          \
    for (int j = 0; j < dk; ++j) {                                             \
        kk[j] = load_elem(J->k, tok * dk + j, J->in_dtype);                    \
        qq[j] = load_elem(J->q, tok * dk + j, J->in_dtype);                    \
        al[j] = exp((double)(J->gate_kind == OR_GATE_PER_CHANNEL               \
                                 ? J->g[tok * dk + j] : J->g[tok]));           \
    }                                                                          \
    for (int i = 0; i < dv; ++i) vv[i] = load_elem(J->v, tok * dv + i, J->in_dtype); \
    const double be = (double)J->beta[tok];

    /* forward, keeping the states */
    for (int t = 0; t < T; ++t) {
        LOAD_TOKEN(t)
        const double *Sprev = St + SS * (size_t)t;
        double *S1 = Sp + SS * (size_t)t, *S2 = St + SS * (size_t)(t + 1);
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) {
                S1[(size_t)i * dk + j] = Sprev[(size_t)i * dk + j] * al[j];
                acc += S1[(size_t)i * dk + j] * kk[j];
            }
            const double u = be * (vv[i] - acc);
            for (int j = 0; j < dk; ++j) S2[(size_t)i * dk + j] = S1[(size_t)i * dk + j] + u * kk[j];
        }
        (void)qq;
        (void)tok;
    }

    /* reverse */
    if (J->dST)
        memcpy(G, J->dST + sidx, sizeof(double) * SS);
    else
        memset(G, 0, sizeof(double) * SS);
    for (int t = T - 1; t >= 0; --t) {
        LOAD_TOKEN(t)
        const double *S1 = Sp + SS * (size_t)t, *S2 = St + SS * (size_t)(t + 1);
        const double *dO = J->dout + tok * dv;
        /* o = S_t q */
        for (int j = 0; j < dk; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dv; ++i) acc += S2[(size_t)i * dk + j] * dO[i];
            J->dq[tok * dk + j] = acc;
        }
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) G[(size_t)i * dk + j] += dO[i] * qq[j];
        /* p and u of this step, recomputed from S' */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S1[(size_t)i * dk + j] * kk[j];
            pp[i] = acc;
            uu[i] = be * (vv[i] - acc);
        }
        /* S_t = S' + u k^T */
        double dbeta = 0.0;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += G[(size_t)i * dk + j] * kk[j];
            du[i] = acc;
            dbeta += acc * (vv[i] - pp[i]);
            J->dv[tok * dv + i] = be * acc;
            dp[i] = -be * acc;
        }
        J->dbeta[tok] = dbeta;
        for (int j = 0; j < dk; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dv; ++i)
                acc += G[(size_t)i * dk + j] * uu[i] + S1[(size_t)i * dk + j] * dp[i];
            J->dk[tok * dk + j] = acc;
        }
        /* dS' = G + dp k^T; dg; dS_{t-1} = dS' Diag(alpha) */
        double dgs = 0.0;
        for (int j = 0; j < dk; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dv; ++i) {
                const double d = G[(size_t)i * dk + j] + dp[i] * kk[j];
                dSp[(size_t)i * dk + j] = d;
                acc += S1[(size_t)i * dk + j] * d;
            }
            if (J->gate_kind == OR_GATE_PER_CHANNEL)
                J->dg[tok * dk + j] = acc;
            else
                dgs += acc;
        }
        if (J->gate_kind != OR_GATE_PER_CHANNEL) J->dg[tok] = dgs;
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) G[(size_t)i * dk + j] = dSp[(size_t)i * dk + j] * al[j];
    }
#undef LOAD_TOKEN
    if (J->dS0) memcpy(J->dS0 + sidx, G, sizeof(double) * SS);
    free(St); free(Sp); free(G); free(dSp); free(kk); free(qq); free(al);
    free(vv); free(pp); free(uu); free(du); free(dp);
}

static void *bwd_worker(void *arg) {
    bwd_job_t *J = (bwd_job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int w = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (w >= J->B * J->H) break;
        bwd_head(J, w / J->H, w % J->H);
    }
    return NULL;
}

int oracle_gdr_bwd(const void *q, const void *k, const void *v, int in_dtype,
                   const float *g, int gate_kind, const float *beta, const double *S0,
                   const double *dout, const double *dST, double *dq, double *dk,
                   double *dv, double *dg, double *dbeta, double *dS0, int B, int T,
                   int H, int dk_, int dv_, int nthreads) {
    if (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta)
        return -1;
    if (B < 0 || T < 0 || H < 0 || dk_ <= 0 || dv_ <= 0) return -1;
    if (in_dtype != OR_F32 && in_dtype != OR_BF16) return -1;
    if (gate_kind != OR_GATE_SCALAR && gate_kind != OR_GATE_PER_CHANNEL) return -1;
    bwd_job_t J;
    J.q = q; J.k = k; J.v = v; J.in_dtype = in_dtype;
    J.g = g; J.gate_kind = gate_kind; J.beta = beta;
    J.S0 = S0; J.dout = dout; J.dST = dST;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dg = dg; J.dbeta = dbeta; J.dS0 = dS0;
    J.B = B; J.T = T; J.H = H; J.dk_ = dk_; J.dv_ = dv_;
    J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    int n = nthreads;
    if (n <= 0) n = 1;
    if (n > B * H) n = B * H;
    if (n <= 1) {
        bwd_worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n);
        for (int i = 0; i < n; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
        for (int i = 0; i < n; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * Diagonal-plus-low-rank transition (DPLR), the generalised sibling of the
 * delta rule: "Decoding Hybrid Linear Attention Architectures", section 3
 * item 5:
 *
 *     S_t = S_{t-1} (Diag(alpha_t) + a_t b_t^T) + v_t k_t^T,    o_t = S_t q_t
 *
 * (the transition acts on the key axis; the write accumulates).  With
 * a = -beta (alpha . k), b = k and v scaled by beta it is the gated delta
 * rule with a per-channel gate.  q, k, a, b [B,T,H,dk]; v, o [B,T,H,dv];
 * g = log alpha [B,T,H] or [B,T,H,dk]; S0, S_T [B,H,dv,dk].  Per row i of S:
 *     x_i = S_i . a;   S_i <- S_i Diag(alpha) + x_i b^T + v_i k^T;   o_i = S_i . q
 */
typedef struct {
    const void *q, *k, *v, *a, *b;
    int in_dtype;
    const float *g;
    int gate_kind;
    const double *S0;
    double *o, *S_T;
    int B, T, H, dk, dv;
    int next;
    pthread_mutex_t lock;
} dplr_job_t;

static void dplr_head(dplr_job_t *J, int b_, int h) {
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *kk = (double *)malloc(sizeof(double) * dk);
    double *qq = (double *)malloc(sizeof(double) * dk);
    double *aa = (double *)malloc(sizeof(double) * dk);
    double *bb = (double *)malloc(sizeof(double) * dk);
    double *al = (double *)malloc(sizeof(double) * dk);
    const size_t sidx = ((size_t)b_ * H + h) * (size_t)dv * dk;
    if (J->S0)
        memcpy(S, J->S0 + sidx, sizeof(double) * (size_t)dv * dk);
    else
        memset(S, 0, sizeof(double) * (size_t)dv * dk);
    for (int t = 0; t < T; ++t) {
        const size_t tok = ((size_t)b_ * T + t) * H + h;
        for (int j = 0; j < dk; ++j) {
            kk[j] = load_elem(J->k, tok * dk + j, J->in_dtype);
            qq[j] = load_elem(J->q, tok * dk + j, J->in_dtype);
            aa[j] = load_elem(J->a, tok * dk + j, J->in_dtype);
            bb[j] = load_elem(J->b, tok * dk + j, J->in_dtype);
            al[j] = exp((double)(J->gate_kind == OR_GATE_PER_CHANNEL ? J->g[tok * dk + j]
                                                                      : J->g[tok]));
        }
        for (int i = 0; i < dv; ++i) {
            double *Si = S + (size_t)i * dk;
            double x = 0.0; /* S_{t-1} a, before the row changes */
            for (int j = 0; j < dk; ++j) x += Si[j] * aa[j];
            const double vi = load_elem(J->v, tok * dv + i, J->in_dtype);
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) {
                Si[j] = Si[j] * al[j] + x * bb[j] + vi * kk[j];
                acc += Si[j] * qq[j];
            }
            J->o[tok * dv + i] = acc;
        }
    }
    if (J->S_T) memcpy(J->S_T + sidx, S, sizeof(double) * (size_t)dv * dk);
    free(S); free(kk); free(qq); free(aa); free(bb); free(al);
}

static void *dplr_worker(void *arg) {
    dplr_job_t *J = (dplr_job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int w = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (w >= J->B * J->H) break;
        dplr_head(J, w / J->H, w % J->H);
    }
    return NULL;
}

int oracle_dplr_fwd(const void *q, const void *k, const void *v, const void *a, const void *b,
                    int in_dtype, const float *g, int gate_kind, const double *S0, double *o,
                    double *S_T, int B, int T, int H, int dk, int dv, int nthreads) {
    if (!q || !k || !v || !a || !b || !g || !o) return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (in_dtype != OR_F32 && in_dtype != OR_BF16) return -1;
    if (gate_kind != OR_GATE_SCALAR && gate_kind != OR_GATE_PER_CHANNEL) return -1;
    dplr_job_t J;
    J.q = q; J.k = k; J.v = v; J.a = a; J.b = b; J.in_dtype = in_dtype;
    J.g = g; J.gate_kind = gate_kind; J.S0 = S0; J.o = o; J.S_T = S_T;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    int n = nthreads;
    if (n <= 0) n = 1;
    if (n > B * H) n = B * H;
    if (n <= 1) {
        dplr_worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n);
        for (int i = 0; i < n; ++i) pthread_create(&th[i], NULL, dplr_worker, &J);
        for (int i = 0; i < n; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return 0;
}
