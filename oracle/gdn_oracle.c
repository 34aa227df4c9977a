/*
 * gdn_oracle.c -- the ORACLE for the gated delta rule: a plain, slow, float64,
 * token-by-token CPU recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  It exists to check the CUDA path, never to stand in
 * for it.  Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load it.  It shares no code, header, table or helper with the CUDA
 * library; nothing here is blocked, chunked, fused or reordered.
 *
 * What it computes (per batch item b and head h, independently):
 *
 *   S_t = S_{t-1} ( alpha_t ( I - beta_t k_t k_t^T ) ) + beta_t v_t k_t^T      (1)
 *   o_t = S_t q_t                                                             (2)
 *
 * (1) is the gated delta rule as stated in "Gated Delta Networks: Improving
 * Mamba2 with Delta Rule" (atlas.scime.ai summary, section "Approach") and again,
 * in damaged LaTeX where "k_t^{o}p" stands for k_t^T, in "Gated DeltaNet:
 * Harmonizing Gating and the Delta Rule for Superior Linear RNNs" (wispaper.ai
 * blog, section "Methodology: The Gated Delta Rule").  The orientation of the
 * state follows from the write term beta v k^T: S has Dv rows and Dk columns.
 *
 * (2) is not written on the pages; the reading adopted is the usual linear
 * attention read-out with the state AFTER the token's own update.
 *
 * Input conventions (readings where the pages are silent): the gate is passed
 * as log(alpha) (<= 0) and alpha = exp(log alpha) is taken here; beta is passed
 * as is.  All arithmetic is double precision.
 *
 * Row i of the product S_{t-1} (alpha (I - beta k k^T)) is written out as
 *   alpha * S[i][j] - alpha * beta * (sum_m S[i][m] k[m]) * k[j]
 * which is the same matrix product with the sum over m collected once per row.
 *
 * Layouts (all row-major, C order):
 *   forward:  q,k [B,T,H,Dk]   v [B,T,H,Dv]   log_alpha,beta [B,T,H]
 *             S0,S_T [B,H,Dv,Dk]   o [B,T,H,Dv]
 *   decode:   q,k [steps,B,H,Dk]  v [steps,B,H,Dv]  log_alpha,beta [steps,B,H]
 *             S [B,H,Dv,Dk] (updated in place)   o [steps,B,H,Dv]
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

/* One token of (1) and (2) on one head: S (Dv x Dk) is updated in place and
 * o (Dv) receives S_t q_t. */
static void gdn_token(double *S, const double *q, const double *k,
                      const double *v, double log_alpha, double beta,
                      double *o, long Dk, long Dv)
{
    const double alpha = exp(log_alpha);
    for (long i = 0; i < Dv; ++i) {
        double *row = S + i * Dk;
        double sk = 0.0; /* (S_{t-1} k_t)_i */
        for (long m = 0; m < Dk; ++m)
            sk += row[m] * k[m];
        for (long j = 0; j < Dk; ++j)
            row[j] = alpha * row[j] - alpha * beta * sk * k[j] + beta * v[i] * k[j];
        double oi = 0.0; /* (S_t q_t)_i */
        for (long j = 0; j < Dk; ++j)
            oi += row[j] * q[j];
        o[i] = oi;
    }
}

/* Where token t of unit u lives: element offset = base + t * stride. */
typedef struct {
    const double *q, *k, *v, *la, *beta;
    double *o, *S;
    long T, Dk, Dv;
    long tstride_qk, tstride_v, tstride_g; /* element stride between tokens */
    const int *units;
    int n_units;
    int n_threads;
    int thread_id;
    int mode; /* 0 forward, 1 decode */
    long B, H;
} job_t;

static void run_unit(const job_t *j, long u)
{
    const long b = u / j->H, h = u % j->H;
    long qk0, v0, g0;
    if (j->mode == 0) { /* [B,T,H,*] */
        qk0 = (b * j->T * j->H + h) * j->Dk;
        v0 = (b * j->T * j->H + h) * j->Dv;
        g0 = b * j->T * j->H + h;
    } else { /* [steps,B,H,*] */
        qk0 = (b * j->H + h) * j->Dk;
        v0 = (b * j->H + h) * j->Dv;
        g0 = b * j->H + h;
    }
    double *S = j->S + u * j->Dv * j->Dk;
    for (long t = 0; t < j->T; ++t) {
        gdn_token(S, j->q + qk0 + t * j->tstride_qk, j->k + qk0 + t * j->tstride_qk,
                  j->v + v0 + t * j->tstride_v, j->la[g0 + t * j->tstride_g],
                  j->beta[g0 + t * j->tstride_g], j->o + v0 + t * j->tstride_v,
                  j->Dk, j->Dv);
    }
}

static void *worker(void *arg)
{
    const job_t *j = (const job_t *)arg;
    const long n = j->units ? j->n_units : j->B * j->H;
    for (long i = j->thread_id; i < n; i += j->n_threads)
        run_unit(j, j->units ? (long)j->units[i] : i);
    return NULL;
}

static int run_job(job_t *proto, int nthreads)
{
    const long n = proto->units ? proto->n_units : proto->B * proto->H;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > n)
        nthreads = (int)(n > 0 ? n : 1);
    job_t *jobs = (job_t *)malloc(sizeof(job_t) * (size_t)nthreads);
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!jobs || !tid) {
        free(jobs);
        free(tid);
        return -2;
    }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = *proto;
        jobs[i].n_threads = nthreads;
        jobs[i].thread_id = i;
    }
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&tid[i], NULL, worker, &jobs[i]) != 0)
            break;
        started = i;
    }
    /* thread 0 runs on the caller; if a pthread failed to start, the caller
     * picks up its share afterwards */
    worker(&jobs[0]);
    for (int i = 1; i <= started; ++i)
        pthread_join(tid[i], NULL);
    for (int i = started + 1; i < nthreads; ++i)
        worker(&jobs[i]);
    free(jobs);
    free(tid);
    return 0;
}

static int check_units(const int *units, int n_units, long n_all)
{
    if (!units)
        return 0;
    if (n_units < 0)
        return -1;
    for (int i = 0; i < n_units; ++i)
        if (units[i] < 0 || units[i] >= n_all)
            return -1;
    return 0;
}

/*
 * Full-sequence recurrence.  S_T receives the final state of every processed
 * unit (it is also the working state); S0 may be NULL for a zero initial state.
 * units/n_units: NULL runs every (b,h) unit (u = b*H + h); otherwise only the
 * listed units are computed and only their slices of o and S_T are written.
 * Returns 0, or -1 on a bad argument, -2 on allocation failure.
 */
int gdn_oracle_forward(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta,
                       const double *S0, double *o, double *S_T,
                       long B, long T, long H, long Dk, long Dv,
                       const int *units, int n_units, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !o || !S_T)
        return -1;
    if (B <= 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0)
        return -1;
    if (check_units(units, n_units, B * H))
        return -1;
    const long n = units ? n_units : B * H;
    for (long i = 0; i < n; ++i) {
        const long u = units ? units[i] : i;
        double *dst = S_T + u * Dv * Dk;
        if (S0)
            memcpy(dst, S0 + u * Dv * Dk, sizeof(double) * (size_t)(Dv * Dk));
        else
            memset(dst, 0, sizeof(double) * (size_t)(Dv * Dk));
    }
    job_t j;
    memset(&j, 0, sizeof(j));
    j.q = q; j.k = k; j.v = v; j.la = log_alpha; j.beta = beta;
    j.o = o; j.S = S_T;
    j.T = T; j.Dk = Dk; j.Dv = Dv; j.B = B; j.H = H;
    j.tstride_qk = H * Dk; j.tstride_v = H * Dv; j.tstride_g = H;
    j.units = units; j.n_units = n_units; j.mode = 0;
    return run_job(&j, nthreads);
}

/*
 * `steps` successive single-token updates of the state S (in place), one token
 * per (b,h) per step -- the recurrent (decoding) form of the same rule.
 */
int gdn_oracle_decode(const double *q, const double *k, const double *v,
                      const double *log_alpha, const double *beta,
                      double *S, double *o,
                      long steps, long B, long H, long Dk, long Dv,
                      const int *units, int n_units, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !o || !S)
        return -1;
    if (B <= 0 || steps < 0 || H <= 0 || Dk <= 0 || Dv <= 0)
        return -1;
    if (check_units(units, n_units, B * H))
        return -1;
    job_t j;
    memset(&j, 0, sizeof(j));
    j.q = q; j.k = k; j.v = v; j.la = log_alpha; j.beta = beta;
    j.o = o; j.S = S;
    j.T = steps; j.Dk = Dk; j.Dv = Dv; j.B = B; j.H = H;
    j.tstride_qk = B * H * Dk; j.tstride_v = B * H * Dv; j.tstride_g = B * H;
    j.units = units; j.n_units = n_units; j.mode = 1;
    return run_job(&j, nthreads);
}

/*
 * Backward: the exact reverse-mode derivative of (1) and (2) for a scalar loss
 * L with given dL/do_t (d_o) and dL/dS_T (dS_T, NULL for zero).  The pages name
 * the parallel (chunkwise) training algorithm but print no backward; the plain
 * reading is the gradient of the forward above, taken token by token in reverse.
 * With G the gradient of S_t (all later uses), A_t = alpha (I - beta k k^T):
 *
 *   G      += do_t q_t^T                          (from o_t = S_t q_t)
 *   dq_t    = S_t^T do_t
 *   dv_t    = beta G k
 *   dbeta_t = (v - alpha S_{t-1} k) . (G k)
 *   dalpha  = <G, S_{t-1}> - beta (S_{t-1} k) . (G k),  dlog_alpha_t = alpha dalpha
 *   dk_t    = beta G^T v - alpha beta (G^T S_{t-1} k + S_{t-1}^T G k)
 *   G      <- G A_t = alpha (G - beta (G k) k^T)  (the gradient of S_{t-1})
 *
 * and dS0 is G after token 0.  S_{t-1} is needed in reverse order: the states at
 * every CKPT-th token are kept from a forward sweep and each block of tokens is
 * swept forward again from its checkpoint before it is walked backwards.
 */
#define CKPT 64

typedef struct {
    const double *q, *k, *v, *la, *beta, *S0, *d_o, *dS_T;
    double *dq, *dk, *dv, *dla, *dbeta, *dS0;
    long B, T, H, Dk, Dv;
    const int *units;
    int n_units, n_threads, thread_id;
    int status;
} bjob_t;

static void bwd_unit(bjob_t *j, long u)
{
    const long b = u / j->H, h = u % j->H, T = j->T, H = j->H, Dk = j->Dk, Dv = j->Dv;
    const long SZ = Dv * Dk;
    const long nblk = (T + CKPT - 1) / CKPT;
    /* ck[c]: state before token c*CKPT; st[i]: state after token blk*CKPT+i-1 */
    double *ck = (double *)malloc(sizeof(double) * (size_t)((nblk > 0 ? nblk : 1) * SZ));
    double *st = (double *)malloc(sizeof(double) * (size_t)((CKPT + 1) * SZ));
    double *G = (double *)malloc(sizeof(double) * (size_t)SZ);
    double *o_scratch = (double *)malloc(sizeof(double) * (size_t)Dv);
    double *sk = (double *)malloc(sizeof(double) * (size_t)Dv);
    double *Gk = (double *)malloc(sizeof(double) * (size_t)Dv);
    if (!ck || !st || !G || !o_scratch || !sk || !Gk) {
        j->status = -2;
        free(ck); free(st); free(G); free(o_scratch); free(sk); free(Gk);
        return;
    }
#define QK(t) (((b * T + (t)) * H + h) * Dk)
#define VV(t) (((b * T + (t)) * H + h) * Dv)
#define GG(t) ((b * T + (t)) * H + h)
    /* forward sweep keeping the checkpoints */
    double *S = st;
    if (j->S0)
        memcpy(S, j->S0 + u * SZ, sizeof(double) * (size_t)SZ);
    else
        memset(S, 0, sizeof(double) * (size_t)SZ);
    for (long t = 0; t < T; ++t) {
        if (t % CKPT == 0)
            memcpy(ck + (t / CKPT) * SZ, S, sizeof(double) * (size_t)SZ);
        gdn_token(S, j->q + QK(t), j->k + QK(t), j->v + VV(t), j->la[GG(t)], j->beta[GG(t)],
                  o_scratch, Dk, Dv);
    }
    if (j->dS_T)
        memcpy(G, j->dS_T + u * SZ, sizeof(double) * (size_t)SZ);
    else
        memset(G, 0, sizeof(double) * (size_t)SZ);
    for (long blk = nblk - 1; blk >= 0; --blk) {
        const long t0 = blk * CKPT, t1 = (t0 + CKPT < T) ? t0 + CKPT : T;
        memcpy(st, ck + blk * SZ, sizeof(double) * (size_t)SZ);
        for (long t = t0; t < t1; ++t) {
            double *nxt = st + (t - t0 + 1) * SZ;
            memcpy(nxt, st + (t - t0) * SZ, sizeof(double) * (size_t)SZ);
            gdn_token(nxt, j->q + QK(t), j->k + QK(t), j->v + VV(t), j->la[GG(t)],
                      j->beta[GG(t)], o_scratch, Dk, Dv);
        }
        for (long t = t1 - 1; t >= t0; --t) {
            const double *Sp = st + (t - t0) * SZ;     /* S_{t-1} */
            const double *Sc = st + (t - t0 + 1) * SZ; /* S_t */
            const double *q = j->q + QK(t), *k = j->k + QK(t), *v = j->v + VV(t);
            const double *dout = j->d_o + VV(t);
            const double alpha = exp(j->la[GG(t)]), beta = j->beta[GG(t)];
            double *dq = j->dq + QK(t), *dk = j->dk + QK(t), *dv = j->dv + VV(t);
            for (long i = 0; i < Dv; ++i)
                for (long m = 0; m < Dk; ++m)
                    G[i * Dk + m] += dout[i] * q[m];
            for (long m = 0; m < Dk; ++m) {
                double a = 0.0;
                for (long i = 0; i < Dv; ++i)
                    a += Sc[i * Dk + m] * dout[i];
                dq[m] = a;
            }
            double dbeta = 0.0, dalpha = 0.0;
            for (long i = 0; i < Dv; ++i) {
                double a = 0.0, c = 0.0;
                for (long m = 0; m < Dk; ++m) {
                    a += Sp[i * Dk + m] * k[m];
                    c += G[i * Dk + m] * k[m];
                    dalpha += G[i * Dk + m] * Sp[i * Dk + m];
                }
                sk[i] = a;
                Gk[i] = c;
                dv[i] = beta * c;
                dbeta += (v[i] - alpha * a) * c;
                dalpha -= beta * a * c;
            }
            for (long m = 0; m < Dk; ++m) {
                double gv = 0.0, gs = 0.0, sg = 0.0;
                for (long i = 0; i < Dv; ++i) {
                    gv += G[i * Dk + m] * v[i];
                    gs += G[i * Dk + m] * sk[i];
                    sg += Sp[i * Dk + m] * Gk[i];
                }
                dk[m] = beta * gv - alpha * beta * (gs + sg);
            }
            j->dbeta[GG(t)] = dbeta;
            j->dla[GG(t)] = alpha * dalpha;
            for (long i = 0; i < Dv; ++i)
                for (long m = 0; m < Dk; ++m)
                    G[i * Dk + m] = alpha * (G[i * Dk + m] - beta * Gk[i] * k[m]);
        }
    }
    memcpy(j->dS0 + u * SZ, G, sizeof(double) * (size_t)SZ);
#undef QK
#undef VV
#undef GG
    free(ck); free(st); free(G); free(o_scratch); free(sk); free(Gk);
}

static void *bwd_worker(void *arg)
{
    bjob_t *j = (bjob_t *)arg;
    const long n = j->units ? j->n_units : j->B * j->H;
    for (long i = j->thread_id; i < n; i += j->n_threads)
        bwd_unit(j, j->units ? (long)j->units[i] : i);
    return NULL;
}

/*
 * Gradients of every input for the units listed (all when units is NULL):
 * dq, dk [B,T,H,Dk], dv [B,T,H,Dv], dlog_alpha, dbeta [B,T,H], dS0 [B,H,Dv,Dk].
 * S0 and dS_T may be NULL (zero).  Only the listed units' slices are written.
 * Returns 0, -1 on a bad argument, -2 on allocation failure.
 */
int gdn_oracle_backward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta, const double *S0,
                        const double *d_o, const double *dS_T,
                        double *dq, double *dk, double *dv, double *dlog_alpha,
                        double *dbeta, double *dS0,
                        long B, long T, long H, long Dk, long Dv,
                        const int *units, int n_units, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !d_o || !dq || !dk || !dv || !dlog_alpha ||
        !dbeta || !dS0)
        return -1;
    if (B <= 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0)
        return -1;
    if (check_units(units, n_units, B * H))
        return -1;
    const long n = units ? n_units : B * H;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > n)
        nthreads = (int)(n > 0 ? n : 1);
    bjob_t *jobs = (bjob_t *)malloc(sizeof(bjob_t) * (size_t)nthreads);
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!jobs || !tid) {
        free(jobs);
        free(tid);
        return -2;
    }
    for (int i = 0; i < nthreads; ++i) {
        bjob_t *j = &jobs[i];
        memset(j, 0, sizeof(*j));
        j->q = q; j->k = k; j->v = v; j->la = log_alpha; j->beta = beta; j->S0 = S0;
        j->d_o = d_o; j->dS_T = dS_T;
        j->dq = dq; j->dk = dk; j->dv = dv; j->dla = dlog_alpha; j->dbeta = dbeta; j->dS0 = dS0;
        j->B = B; j->T = T; j->H = H; j->Dk = Dk; j->Dv = Dv;
        j->units = units; j->n_units = n_units; j->n_threads = nthreads; j->thread_id = i;
    }
    int started = 0;
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&tid[i], NULL, bwd_worker, &jobs[i]) != 0)
            break;
        started = i;
    }
    bwd_worker(&jobs[0]);
    for (int i = 1; i <= started; ++i)
        pthread_join(tid[i], NULL);
    for (int i = started + 1; i < nthreads; ++i)
        bwd_worker(&jobs[i]);
    int status = 0;
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status)
            status = jobs[i].status;
    free(jobs);
    free(tid);
    return status;
}

/*
 * Channel-wise gates (Gated DeltaNet-2, "Gated DeltaNet-2: Decoupling Erase and
 * Write in Linear Attention", abstract): a decay per key channel alpha_t in
 * (0,1]^Dk (given as log alpha, as above), a channel-wise erase gate b_t
 * (Dk, on the key side) and a channel-wise write gate w_t (Dv, on the value
 * side).  The pages give the roles and the reductions but not the formula; the
 * reading taken keeps one rank-one edit per token:
 *
 *   S_t = S_{t-1} Diag(alpha_t) ( I - (b_t o k_t) k_t^T ) + (w_t o v_t) k_t^T   (3)
 *   o_t = S_t q_t
 *
 * which is the rule (1) when alpha_t, b_t and w_t are all the scalar alpha_t,
 * beta_t, beta_t ("reducing to KDA when both gates collapse to the same scalar
 * and to Gated DeltaNet when the decay also collapses").  Row i of (3):
 *   d_j = alpha_j S[i][j];  e = sum_j d_j b_j k_j;
 *   S[i][j] = d_j - e k_j + w_i v_i k_j
 */
static void gdn2_token(double *S, const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *b, const double *w,
                       double *o, long Dk, long Dv)
{
    for (long i = 0; i < Dv; ++i) {
        double *row = S + i * Dk;
        double e = 0.0;
        for (long j = 0; j < Dk; ++j) {
            row[j] = exp(log_alpha[j]) * row[j];
            e += row[j] * b[j] * k[j];
        }
        for (long j = 0; j < Dk; ++j)
            row[j] = row[j] - e * k[j] + w[i] * v[i] * k[j];
        double oi = 0.0;
        for (long j = 0; j < Dk; ++j)
            oi += q[j] * row[j];
        o[i] = oi;
    }
}

typedef struct {
    const double *q, *k, *v, *la, *b, *w;
    double *o, *S;
    long B, T, H, Dk, Dv;
    const int *units;
    int n_units, n_threads, thread_id;
} cwjob_t;

static void *cw_worker(void *arg)
{
    const cwjob_t *j = (const cwjob_t *)arg;
    const long n = j->units ? j->n_units : j->B * j->H;
    for (long ii = j->thread_id; ii < n; ii += j->n_threads) {
        const long u = j->units ? (long)j->units[ii] : ii;
        const long b = u / j->H, h = u % j->H;
        double *S = j->S + u * j->Dv * j->Dk;
        for (long t = 0; t < j->T; ++t) {
            const long row = (b * j->T + t) * j->H + h; /* token row of [B,T,H,*] */
            gdn2_token(S, j->q + row * j->Dk, j->k + row * j->Dk, j->v + row * j->Dv,
                       j->la + row * j->Dk, j->b + row * j->Dk, j->w + row * j->Dv,
                       j->o + row * j->Dv, j->Dk, j->Dv);
        }
    }
    return NULL;
}

/*
 * Whole-sequence recurrence (3): q,k,log_alpha,b [B,T,H,Dk]; v,w [B,T,H,Dv];
 * S0 [B,H,Dv,Dk] or NULL; o [B,T,H,Dv]; S_T [B,H,Dv,Dk].  units as for
 * gdn_oracle_forward.  Returns 0, -1 on a bad argument, -2 on allocation failure.
 */
int gdn_oracle_forward_cw(const double *q, const double *k, const double *v,
                          const double *log_alpha, const double *b, const double *w,
                          const double *S0, double *o, double *S_T,
                          long B, long T, long H, long Dk, long Dv,
                          const int *units, int n_units, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !b || !w || !o || !S_T)
        return -1;
    if (B <= 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0)
        return -1;
    if (check_units(units, n_units, B * H))
        return -1;
    const long n = units ? n_units : B * H;
    for (long i = 0; i < n; ++i) {
        const long u = units ? units[i] : i;
        double *dst = S_T + u * Dv * Dk;
        if (S0)
            memcpy(dst, S0 + u * Dv * Dk, sizeof(double) * (size_t)(Dv * Dk));
        else
            memset(dst, 0, sizeof(double) * (size_t)(Dv * Dk));
    }
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > n)
        nthreads = (int)(n > 0 ? n : 1);
    cwjob_t *jobs = (cwjob_t *)malloc(sizeof(cwjob_t) * (size_t)nthreads);
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!jobs || !tid) {
        free(jobs);
        free(tid);
        return -2;
    }
    for (int i = 0; i < nthreads; ++i) {
        cwjob_t *j = &jobs[i];
        memset(j, 0, sizeof(*j));
        j->q = q; j->k = k; j->v = v; j->la = log_alpha; j->b = b; j->w = w;
        j->o = o; j->S = S_T;
        j->B = B; j->T = T; j->H = H; j->Dk = Dk; j->Dv = Dv;
        j->units = units; j->n_units = n_units; j->n_threads = nthreads; j->thread_id = i;
    }
    int started = 0;
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&tid[i], NULL, cw_worker, &jobs[i]) != 0)
            break;
        started = i;
    }
    cw_worker(&jobs[0]);
    for (int i = 1; i <= started; ++i)
        pthread_join(tid[i], NULL);
    for (int i = started + 1; i < nthreads; ++i)
        cw_worker(&jobs[i]);
    free(jobs);
    free(tid);
    return 0;
}
