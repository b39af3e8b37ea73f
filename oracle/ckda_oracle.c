/*
 * ckda_oracle.c -- plain fp64 CPU oracle for the Complex KDA (CKDA) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * What it computes (one head of one sequence, token by token, in double
 * precision, the signed gate applied directly -- no sign folding, no chunks):
 *
 *   alpha_t = sign_t * exp(g_t)                 per key channel, |alpha| <= 1
 *   S_t     = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t     = S_t^T q_t                          (the updated state)
 *
 * Sources:
 *  - "openeurollm/complex-kda-1.3B-100B" model card, introduction: CKDA is KDA
 *    with a per-channel decay alpha in [-1, 1]; |alpha| is carried in log space
 *    (the input g = log|alpha|), the +-1 part separately (the input sign).
 *  - "Complex KDA: Understanding and Enhancing the Expressivity of Kimi Delta
 *    Attention", section 2 (Related work, "Linear RNNs"): the delta-rule
 *    transition I - beta k k^T, KDA's channel-wise gate, the transition acting
 *    on the columns of the state; section 3 ("CKDA"): KDA with the gate range
 *    [-1, 1] and beta in [0, 2].
 *  - The state has key channels as rows (dk x dv) and the output reads the
 *    state after the update; the pages' equation for this is lost in the
 *    extracted text, this is the plain reading of the recurrence as stated.
 *
 * Backward: reverse-mode differentiation of the same token recurrence,
 * written out by hand (derivation in the comments of step_bwd), with states
 * checkpointed every CKDA_ORACLE_CKPT tokens and recomputed per segment.
 * It returns the exact gradient with respect to g = log|alpha| for the g it
 * is given; the sign is piecewise constant and gets no gradient.  (The pages
 * defer their "backward convention" to an appendix that is not in the text.)
 *
 * Pins (tests, not here): orthogonality / Frobenius-norm preservation at
 * |alpha| = 1, beta = 2, unit k; the 2-D rotation by pi + 2 phi; spectral norm
 * <= 1; dense brute-force products; scalar closed forms; finite differences.
 *
 * Layouts (all row-major, contiguous):
 *   tokens of all sequences packed along one axis, offsets cu_seqlens[n_seq+1]
 *   q, k, g : [T_total, H, dk]   v, o, dO : [T_total, H, dv]
 *   sign    : [T_total, H, dk] int8 (+1 / -1)   beta : [T_total, H]
 *   S0, ST, dST, dS0 : [n_seq, H, dk, dv]
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define CKDA_ORACLE_CKPT 64

/* ------------------------------------------------------------------ */
/* one token, forward                                                  */
/* ------------------------------------------------------------------ */

/* S (dk x dv) is advanced in place by one token.  If X is non-null it
 * receives Diag(alpha) S_{t-1}.  o (dv) receives S_t^T q if non-null. */
static void step_fwd(int dk, int dv, double *S, const double *q,
                     const double *k, const double *v, const double *g,
                     const int8_t *sg, double beta, double *o, double *kx)
{
    /* X = Diag(alpha) S_{t-1}, alpha_i = sign_i * exp(g_i) */
    for (int i = 0; i < dk; ++i) {
        double a = (double)sg[i] * exp(g[i]);
        for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
    }
    /* kx = X^T k */
    for (int j = 0; j < dv; ++j) kx[j] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) kx[j] += k[i] * S[i * dv + j];
    /* S_t = X - beta k (k^T X) + beta k v^T */
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[i * dv + j] += beta * k[i] * (v[j] - kx[j]);
    /* o_t = S_t^T q */
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
    }
}

/* ------------------------------------------------------------------ */
/* one token, backward                                                 */
/* ------------------------------------------------------------------ */

/* Inputs: Sprev = S_{t-1}, Snew = S_t, G = dL/dS_t accumulated from later
 * tokens (overwritten with dL/dS_{t-1}).  Writes dq, dk, dv, dg, *dbeta.
 *
 * Derivation (X = Diag(alpha) Sprev, r = v - X^T k, S_t = X + beta k r^T):
 *   o_t = S_t^T q         =>  G += q dO^T,  dq = S_t dO
 *   Gk = G^T k
 *   dv    = beta Gk
 *   dbeta = Gk . r
 *   dk    = beta (G r - X Gk)
 *   dX    = G - beta k Gk^T
 *   dg_i  = sum_j dX_ij X_ij          (d alpha_i / d g_i = alpha_i)
 *   dS_{t-1} = Diag(alpha) dX
 */
static void step_bwd(int dk, int dv, const double *Sprev, const double *Snew,
                     double *G, const double *q, const double *k,
                     const double *v, const double *g, const int8_t *sg,
                     double beta, const double *dO, double *dq, double *dk_,
                     double *dv_, double *dg, double *dbeta, double *X,
                     double *r, double *Gk)
{
    /* output term */
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) G[i * dv + j] += q[i] * dO[j];
    for (int i = 0; i < dk; ++i) {
        double s = 0.0;
        for (int j = 0; j < dv; ++j) s += Snew[i * dv + j] * dO[j];
        dq[i] = s;
    }
    /* recompute X and r */
    for (int i = 0; i < dk; ++i) {
        double a = (double)sg[i] * exp(g[i]);
        for (int j = 0; j < dv; ++j) X[i * dv + j] = a * Sprev[i * dv + j];
    }
    for (int j = 0; j < dv; ++j) {
        double s = 0.0;
        for (int i = 0; i < dk; ++i) s += k[i] * X[i * dv + j];
        r[j] = v[j] - s;
    }
    for (int j = 0; j < dv; ++j) {
        double s = 0.0;
        for (int i = 0; i < dk; ++i) s += G[i * dv + j] * k[i];
        Gk[j] = s;
    }
    double db = 0.0;
    for (int j = 0; j < dv; ++j) {
        dv_[j] = beta * Gk[j];
        db += Gk[j] * r[j];
    }
    *dbeta = db;
    for (int i = 0; i < dk; ++i) {
        double gr = 0.0, xg = 0.0;
        for (int j = 0; j < dv; ++j) {
            gr += G[i * dv + j] * r[j];
            xg += X[i * dv + j] * Gk[j];
        }
        dk_[i] = beta * (gr - xg);
    }
    /* dX = G - beta k Gk^T ; dg ; G <- Diag(alpha) dX */
    for (int i = 0; i < dk; ++i) {
        double a = (double)sg[i] * exp(g[i]);
        double s = 0.0;
        for (int j = 0; j < dv; ++j) {
            double dx = G[i * dv + j] - beta * k[i] * Gk[j];
            s += dx * X[i * dv + j];
            G[i * dv + j] = a * dx;
        }
        dg[i] = s;
    }
}

/* ------------------------------------------------------------------ */
/* job pool over independent (sequence, head) pairs                     */
/* ------------------------------------------------------------------ */

typedef struct {
    int kind; /* 0 fwd, 1 bwd, 2 decode */
    int n_seq, H, dk, dv, chunk;
    const int64_t *cu;
    const double *q, *k, *v, *g, *beta, *S0, *dO, *dST;
    const int8_t *sign;
    double *o, *ST, *chunk_states, *state;
    double *dq, *dk_, *dv_, *dg, *dbeta, *dS0;
    const int64_t *chunk_off; /* per sequence, first global chunk index */
    int64_t next;
    int64_t njobs;
    int failed;
    pthread_mutex_t mu;
} pool_t;

static int64_t take_job(pool_t *p)
{
    pthread_mutex_lock(&p->mu);
    int64_t j = p->next < p->njobs ? p->next++ : -1;
    pthread_mutex_unlock(&p->mu);
    return j;
}

static void run_fwd(pool_t *p, int64_t job)
{
    const int H = p->H, dk = p->dk, dv = p->dv;
    const int n = (int)(job / H), h = (int)(job % H);
    const int64_t t0 = p->cu[n], t1 = p->cu[n + 1];
    double *S = (double *)malloc(sizeof(double) * dk * dv);
    double *kx = (double *)malloc(sizeof(double) * dv);
    if (!S || !kx) { p->failed = 1; free(S); free(kx); return; }
    if (p->S0)
        memcpy(S, p->S0 + ((int64_t)n * H + h) * dk * dv, sizeof(double) * dk * dv);
    else
        memset(S, 0, sizeof(double) * dk * dv);
    for (int64_t t = t0; t < t1; ++t) {
        if (p->chunk_states && (t - t0) % p->chunk == 0) {
            int64_t c = p->chunk_off[n] + (t - t0) / p->chunk;
            memcpy(p->chunk_states + (c * H + h) * dk * dv, S,
                   sizeof(double) * dk * dv);
        }
        const int64_t th = t * H + h;
        step_fwd(dk, dv, S, p->q + th * dk, p->k + th * dk, p->v + th * dv,
                 p->g + th * dk, p->sign + th * dk, p->beta[th],
                 p->o ? p->o + th * dv : NULL, kx);
    }
    if (p->ST)
        memcpy(p->ST + ((int64_t)n * H + h) * dk * dv, S, sizeof(double) * dk * dv);
    free(S);
    free(kx);
}

static void run_bwd(pool_t *p, int64_t job)
{
    const int H = p->H, dk = p->dk, dv = p->dv;
    const int n = (int)(job / H), h = (int)(job % H);
    const int64_t t0 = p->cu[n], t1 = p->cu[n + 1], len = t1 - t0;
    const int64_t sz = (int64_t)dk * dv;
    const int64_t nseg = (len + CKDA_ORACLE_CKPT - 1) / CKDA_ORACLE_CKPT;
    /* ckpt[s] = state before token s*CKPT of this sequence; seg[i] = state
     * after token i of the current segment. */
    double *ckpt = (double *)malloc(sizeof(double) * sz * (nseg + 1));
    double *seg = (double *)malloc(sizeof(double) * sz * (CKDA_ORACLE_CKPT + 1));
    double *G = (double *)malloc(sizeof(double) * sz);
    double *X = (double *)malloc(sizeof(double) * sz);
    double *kx = (double *)malloc(sizeof(double) * dv);
    double *r = (double *)malloc(sizeof(double) * dv);
    double *Gk = (double *)malloc(sizeof(double) * dv);
    if (!ckpt || !seg || !G || !X || !kx || !r || !Gk) {
        p->failed = 1;
        goto done;
    }
    /* forward pass, keeping one state per segment */
    double *S = seg; /* scratch */
    if (p->S0)
        memcpy(S, p->S0 + ((int64_t)n * H + h) * sz, sizeof(double) * sz);
    else
        memset(S, 0, sizeof(double) * sz);
    for (int64_t t = t0; t < t1; ++t) {
        if ((t - t0) % CKDA_ORACLE_CKPT == 0)
            memcpy(ckpt + ((t - t0) / CKDA_ORACLE_CKPT) * sz, S, sizeof(double) * sz);
        const int64_t th = t * H + h;
        step_fwd(dk, dv, S, p->q + th * dk, p->k + th * dk, p->v + th * dv,
                 p->g + th * dk, p->sign + th * dk, p->beta[th], NULL, kx);
    }
    /* seed with dL/dS_T */
    if (p->dST)
        memcpy(G, p->dST + ((int64_t)n * H + h) * sz, sizeof(double) * sz);
    else
        memset(G, 0, sizeof(double) * sz);
    /* reverse over segments */
    for (int64_t s = nseg - 1; s >= 0; --s) {
        const int64_t a = t0 + s * CKDA_ORACLE_CKPT;
        const int64_t b = (a + CKDA_ORACLE_CKPT < t1) ? a + CKDA_ORACLE_CKPT : t1;
        memcpy(seg, ckpt + s * sz, sizeof(double) * sz);
        for (int64_t t = a; t < b; ++t) {
            double *Snext = seg + (t - a + 1) * sz;
            memcpy(Snext, seg + (t - a) * sz, sizeof(double) * sz);
            const int64_t th = t * H + h;
            step_fwd(dk, dv, Snext, p->q + th * dk, p->k + th * dk,
                     p->v + th * dv, p->g + th * dk, p->sign + th * dk,
                     p->beta[th], NULL, kx);
        }
        for (int64_t t = b - 1; t >= a; --t) {
            const int64_t th = t * H + h;
            step_bwd(dk, dv, seg + (t - a) * sz, seg + (t - a + 1) * sz, G,
                     p->q + th * dk, p->k + th * dk, p->v + th * dv,
                     p->g + th * dk, p->sign + th * dk, p->beta[th],
                     p->dO + th * dv, p->dq + th * dk, p->dk_ + th * dk,
                     p->dv_ + th * dv, p->dg + th * dk, p->dbeta + th, X, r, Gk);
        }
    }
    if (p->dS0)
        memcpy(p->dS0 + ((int64_t)n * H + h) * sz, G, sizeof(double) * sz);
done:
    free(ckpt); free(seg); free(G); free(X); free(kx); free(r); free(Gk);
}

static void run_decode(pool_t *p, int64_t job)
{
    const int dk = p->dk, dv = p->dv;
    double kx[1024];
    if (dv > 1024) { p->failed = 1; return; }
    step_fwd(dk, dv, p->state + job * dk * dv, p->q + job * dk, p->k + job * dk,
             p->v + job * dv, p->g + job * dk, p->sign + job * dk, p->beta[job],
             p->o + job * dv, kx);
}

static void *worker(void *arg)
{
    pool_t *p = (pool_t *)arg;
    for (;;) {
        int64_t j = take_job(p);
        if (j < 0) break;
        if (p->kind == 0) run_fwd(p, j);
        else if (p->kind == 1) run_bwd(p, j);
        else run_decode(p, j);
    }
    return NULL;
}

static int run_pool(pool_t *p, int nthreads)
{
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    if ((int64_t)nthreads > p->njobs) nthreads = (int)(p->njobs > 0 ? p->njobs : 1);
    pthread_mutex_init(&p->mu, NULL);
    pthread_t th[512];
    int started = 0;
    for (int i = 1; i < nthreads; ++i)
        if (pthread_create(&th[started], NULL, worker, p) == 0) ++started;
    worker(p);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&p->mu);
    return p->failed ? -1 : 0;
}

/* number of worker threads a call with nthreads <= 0 uses */
int ckda_oracle_default_threads(void)
{
    return (int)sysconf(_SC_NPROCESSORS_ONLN);
}

/* Forward over n_seq packed sequences.  chunk_states (nullable) receives
 * the state before token j*chunk of each sequence, at global chunk index
 * (sum over earlier sequences of ceil(len/chunk)) + j, layout [., H, dk, dv]. */
int ckda_oracle_fwd(int n_seq, const int64_t *cu_seqlens, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *g, const int8_t *sign, const double *beta,
                    const double *S0, double *o, double *ST, int chunk,
                    double *chunk_states, int nthreads)
{
    if (n_seq < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    int64_t *off = NULL;
    if (chunk_states) {
        if (chunk <= 0) return -1;
        off = (int64_t *)malloc(sizeof(int64_t) * (n_seq + 1));
        if (!off) return -1;
        off[0] = 0;
        for (int i = 0; i < n_seq; ++i) {
            int64_t len = cu_seqlens[i + 1] - cu_seqlens[i];
            off[i + 1] = off[i] + (len + chunk - 1) / chunk;
        }
    }
    pool_t p;
    memset(&p, 0, sizeof(p));
    p.kind = 0; p.n_seq = n_seq; p.H = H; p.dk = dk; p.dv = dv; p.chunk = chunk;
    p.cu = cu_seqlens; p.q = q; p.k = k; p.v = v; p.g = g; p.sign = sign;
    p.beta = beta; p.S0 = S0; p.o = o; p.ST = ST; p.chunk_states = chunk_states;
    p.chunk_off = off; p.njobs = (int64_t)n_seq * H;
    int rc = run_pool(&p, nthreads);
    free(off);
    return rc;
}

int ckda_oracle_bwd(int n_seq, const int64_t *cu_seqlens, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *g, const int8_t *sign, const double *beta,
                    const double *S0, const double *dO, const double *dST,
                    double *dq, double *dk_, double *dv_, double *dg,
                    double *dbeta, double *dS0, int nthreads)
{
    if (n_seq < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    pool_t p;
    memset(&p, 0, sizeof(p));
    p.kind = 1; p.n_seq = n_seq; p.H = H; p.dk = dk; p.dv = dv;
    p.cu = cu_seqlens; p.q = q; p.k = k; p.v = v; p.g = g; p.sign = sign;
    p.beta = beta; p.S0 = S0; p.dO = dO; p.dST = dST;
    p.dq = dq; p.dk_ = dk_; p.dv_ = dv_; p.dg = dg; p.dbeta = dbeta; p.dS0 = dS0;
    p.njobs = (int64_t)n_seq * H;
    return run_pool(&p, nthreads);
}

/* One recurrent step for N*H independent states, in place.
 * q, k, g, sign : [N, H, dk]; v, o : [N, H, dv]; beta : [N, H];
 * state : [N, H, dk, dv]. */
int ckda_oracle_decode(int N, int H, int dk, int dv, const double *q,
                       const double *k, const double *v, const double *g,
                       const int8_t *sign, const double *beta, double *state,
                       double *o, int nthreads)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    pool_t p;
    memset(&p, 0, sizeof(p));
    p.kind = 2; p.H = H; p.dk = dk; p.dv = dv;
    p.q = q; p.k = k; p.v = v; p.g = g; p.sign = sign; p.beta = beta;
    p.state = state; p.o = o;
    p.njobs = (int64_t)N * H;
    return run_pool(&p, nthreads);
}
