/*
 * gdn_oracle.c -- FP64 sequential reference for the gated delta-net scan.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness oracle that the
 * tests, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py`
 * compare the CUDA library against.  It is not part of the product path, it
 * shares no code, header, table or helper with the CUDA library, and nothing
 * in the library links or calls it.
 *
 * What it computes (one (b,h) sequence at a time, all arithmetic in double):
 *
 *   causal  (mode 0):  S_t = a_t (I - e_t k_t k_t^T) S_{t-1} + w_t k_t v_t^T
 *                      o_t = S_t^T q_t                          t = 1..T
 *   reverse (mode 1):  R_t = a_t (I - e_t k_t k_t^T) R_{t+1} + w_t k_t v_t^T
 *                      o_t = R_{t+1}^T q_t   (read BEFORE token t is written)
 *   bidir   (mode 2):  o_t = causal o_t + reverse o_t
 *
 * The product operator uses e_t = w_t = beta_t (one coefficient for the erase
 * and for the write).  The separate erase coefficient e_t and write
 * coefficient w_t exist only so that the tests can switch the delta-rule
 * erase off while keeping the write, which is the "drop the delta-rule
 * update" special case that reduces the operator to gated linear attention.
 *
 * Sources (web pages; the pages give the operator in words, the formula is
 * the one the project fixes for the gated delta rule):
 *  - issue "[Research] Explore linear attention for the streaming video
 *    models", section "We already ship a hybrid linear-attention model":
 *    gated delta-net linear attention with a matrix-valued recurrent state
 *    per head; the causal, forward-only variant is the streaming form.
 *  - same issue, section "Suggested phases" (Phase 1): the streaming state
 *    lifecycle, i.e. the state is carried from one call to the next
 *    (state in / state out below).
 *  - "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
 *    Generation" (AI summary), section "Methodology in Plain English": a
 *    forward and a backward recurrent state cover disjoint regions of the
 *    clip and their readouts are added, so no token is counted twice.  Read
 *    plainly, the backward readout at token t uses the reverse state that
 *    holds tokens t+1..T only (mode 1 above).
 *  - "SANA-Video 2.0" review, section "Future work": dropping the delta-rule
 *    update turns the operator into plain gated linear attention (e_t = 0).
 *
 * Layout: q,k [B,T,H,dk], v,o [B,T,H,dv], alpha/erase/write [B,T,H],
 * states [B,H,dk,dv] with the key dimension as the row index; all double,
 * contiguous, row-major.  Work is split over (b,h) pairs with pthreads.
 */
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, H, dk, dv, mode;
    const double *q, *k, *v, *alpha, *erase, *write;
    const double *s_fwd0, *s_bwd0; /* initial states or NULL (= zero) */
    double *o, *s_fwd_out, *s_bwd_out;
    int next_task;                 /* next (b,h) index to take */
    pthread_mutex_t lock;
} job_t;

/* o[t] (+)= S^T q[t] for one token: S is dk x dv, q has dk entries. */
static void readout(const double *S, const double *q, int dk, int dv,
                    double *o, int accumulate)
{
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * q[i];
        o[j] = accumulate ? o[j] + acc : acc;
    }
}

/* S <- a (I - e k k^T) S + w k v^T, written as
 *   p = S^T k ;  S <- a (S - e k p^T) + w k v^T                            */
static void transition(double *S, double *p, const double *k, const double *v,
                       double a, double e, double w, int dk, int dv)
{
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * k[i];
        p[j] = acc;
    }
    for (int i = 0; i < dk; ++i) {
        double *row = S + (size_t)i * dv;
        const double ki = k[i];
        for (int j = 0; j < dv; ++j)
            row[j] = a * (row[j] - e * ki * p[j]) + w * ki * v[j];
    }
}

static void run_one(job_t *J, int bh, double *S, double *p)
{
    const int b = bh / J->H, h = bh % J->H;
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    const size_t sdim = (size_t)dk * dv;

    /* causal pass (modes 0 and 2) */
    if (J->mode == 0 || J->mode == 2) {
        if (J->s_fwd0) memcpy(S, J->s_fwd0 + (size_t)bh * sdim, sdim * sizeof(double));
        else memset(S, 0, sdim * sizeof(double));
        for (int t = 0; t < T; ++t) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            transition(S, p, J->k + tok * dk, J->v + tok * dv, J->alpha[tok],
                       J->erase[tok], J->write[tok], dk, dv);
            readout(S, J->q + tok * dk, dk, dv, J->o + tok * dv, 0);
        }
        if (J->s_fwd_out) memcpy(J->s_fwd_out + (size_t)bh * sdim, S, sdim * sizeof(double));
    }
    /* reverse pass with the strict readout (modes 1 and 2) */
    if (J->mode == 1 || J->mode == 2) {
        const int acc = (J->mode == 2);
        if (J->s_bwd0) memcpy(S, J->s_bwd0 + (size_t)bh * sdim, sdim * sizeof(double));
        else memset(S, 0, sdim * sizeof(double));
        for (int t = T - 1; t >= 0; --t) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            readout(S, J->q + tok * dk, dk, dv, J->o + tok * dv, acc);
            transition(S, p, J->k + tok * dk, J->v + tok * dv, J->alpha[tok],
                       J->erase[tok], J->write[tok], dk, dv);
        }
        if (J->s_bwd_out) memcpy(J->s_bwd_out + (size_t)bh * sdim, S, sdim * sizeof(double));
    }
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dk * J->dv);
    double *p = (double *)malloc(sizeof(double) * (size_t)J->dv);
    if (S && p) {
        for (;;) {
            pthread_mutex_lock(&J->lock);
            const int bh = J->next_task++;
            pthread_mutex_unlock(&J->lock);
            if (bh >= J->B * J->H) break;
            run_one(J, bh, S, p);
        }
    }
    free(S);
    free(p);
    return NULL;
}

/*
 * gdn_oracle_scan: run the recurrence for every (b,h) sequence.
 *   mode      0 causal, 1 reverse with strict readout, 2 bidirectional sum
 *   erase     per-token erase coefficient e_t; write: write coefficient w_t
 *             (the product operator passes beta for both)
 *   s_fwd0    initial causal state (NULL = zero);  s_fwd_out: final causal
 *             state after token T (NULL = not written)
 *   s_bwd0    initial reverse state R_{T+1} (NULL = zero); s_bwd_out: R_1
 *   threads   number of worker threads (<= 0: one)
 * Returns 0, or -1 on a bad argument or an allocation failure.
 */
int gdn_oracle_scan(int B, int T, int H, int dk, int dv, int mode,
                    const double *q, const double *k, const double *v,
                    const double *alpha, const double *erase, const double *write,
                    const double *s_fwd0, const double *s_bwd0,
                    double *o, double *s_fwd_out, double *s_bwd_out, int threads)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0 || mode < 0 || mode > 2) return -1;
    if (T > 0 && (!q || !k || !v || !alpha || !erase || !write || !o)) return -1;
    job_t J;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.mode = mode;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.erase = erase; J.write = write;
    J.s_fwd0 = s_fwd0; J.s_bwd0 = s_bwd0;
    J.o = o; J.s_fwd_out = s_fwd_out; J.s_bwd_out = s_bwd_out;
    J.next_task = 0;
    pthread_mutex_init(&J.lock, NULL);
    int n = threads <= 0 ? 1 : threads;
    if (n > B * H) n = B * H > 0 ? B * H : 1;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n);
    if (!tid) { pthread_mutex_destroy(&J.lock); return -1; }
    int started = 0;
    for (int i = 1; i < n; ++i)
        if (pthread_create(&tid[started], NULL, worker, &J) == 0) ++started;
    worker(&J); /* the calling thread works too */
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
