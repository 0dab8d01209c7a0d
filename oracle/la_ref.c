/*
 * la_ref.c - the oracle: a plain, slow, float64 CPU implementation of causal
 * linear attention with an optional decay and normaliser.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load or call this code.  It shares no code
 * with the CUDA library and is not a fallback for it.
 *
 * It follows the recurrent definition token by token, with no chunking and no
 * reordering:
 *
 *   S_t = g_t S_{t-1} + k_t v_t^T          (tensortonic "CS336 L04 linear
 *                                           attention duality": S_t = S_{t-1} +
 *                                           k_t v_t^T with a zero start, here
 *                                           with the decay factor of
 *                                           Jamie-Stirling/RetNet issue 21,
 *                                           cumulative_ema: state * factor + value)
 *   z_t = g_t z_{t-1} + k_t                (flash-linear-attention issue 268:
 *                                           the key sum Sigma k_j carried as the
 *                                           "Z-state"; decayed like S, a reading)
 *   y_t = q_t^T S_t                        (tensortonic page: the output includes
 *                                           the current token)
 *   y_t = q_t^T S_t / q_t^T z_t            (flash-linear-attention issue 268,
 *                                           opening comment: QKV / QK1)
 *
 * g_t = exp(l_t) where l_t is the natural log of the decay, given per head
 * (retention's gamma) or per step (the general EMA of RetNet issue 21).
 * Inputs are float64 arrays; callers up-cast bf16/fp32 inputs exactly.
 *
 * Threads run over independent (b, h) sequences only; each sequence is one
 * sequential loop over t.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *log_g;
    int decay_kind;           /* 0 none, 1 per head [H], 2 per step [B,H,T] */
    int normalize;
    const double *init_state, *init_z;
    double *out, *final_state, *final_z;
    int B, H, T, Dk, Dv;
    int first_bh, last_bh;    /* this worker's [first, last) range of b*H+h */
} fwd_job;

/* Decay factor g_t of token t of sequence bh = b*H + h. */
static double decay_at(int decay_kind, const double* log_g, int H, int T, int bh, int t)
{
    if (decay_kind == 0) return 1.0;
    if (decay_kind == 1) return exp(log_g[bh % H]);
    return exp(log_g[(size_t)bh * T + t]);
}

static double decay_factor(const fwd_job* j, int bh, int t)
{
    return decay_at(j->decay_kind, j->log_g, j->H, j->T, bh, t);
}

static void forward_one(const fwd_job* j, int bh, double* S, double* z)
{
    const int T = j->T, Dk = j->Dk, Dv = j->Dv;
    const size_t sq = (size_t)bh * T * Dk, sv = (size_t)bh * T * Dv;
    const size_t ss = (size_t)bh * Dk * Dv, sz = (size_t)bh * Dk;

    for (int a = 0; a < Dk * Dv; ++a) S[a] = j->init_state ? j->init_state[ss + a] : 0.0;
    for (int a = 0; a < Dk; ++a) z[a] = (j->normalize && j->init_z) ? j->init_z[sz + a] : 0.0;

    for (int t = 0; t < T; ++t) {
        const double* qt = j->q + sq + (size_t)t * Dk;
        const double* kt = j->k + sq + (size_t)t * Dk;
        const double* vt = j->v + sv + (size_t)t * Dv;
        const double g = decay_factor(j, bh, t);

        /* state update: decay, then add the outer product k_t v_t^T */
        for (int i = 0; i < Dk; ++i)
            for (int c = 0; c < Dv; ++c)
                S[i * Dv + c] = g * S[i * Dv + c] + kt[i] * vt[c];
        if (j->normalize)
            for (int i = 0; i < Dk; ++i) z[i] = g * z[i] + kt[i];

        /* read-out with the updated state */
        double den = 0.0;
        if (j->normalize)
            for (int i = 0; i < Dk; ++i) den += qt[i] * z[i];
        for (int c = 0; c < Dv; ++c) {
            double num = 0.0;
            for (int i = 0; i < Dk; ++i) num += qt[i] * S[i * Dv + c];
            j->out[sv + (size_t)t * Dv + c] = j->normalize ? num / den : num;
        }
    }
    if (j->final_state)
        for (int a = 0; a < Dk * Dv; ++a) j->final_state[ss + a] = S[a];
    if (j->final_z && j->normalize)
        for (int a = 0; a < Dk; ++a) j->final_z[sz + a] = z[a];
}

static void* forward_worker(void* arg)
{
    const fwd_job* j = (const fwd_job*)arg;
    double* S = (double*)malloc(sizeof(double) * (size_t)j->Dk * j->Dv);
    double* z = (double*)malloc(sizeof(double) * (size_t)j->Dk);
    if (S && z)
        for (int bh = j->first_bh; bh < j->last_bh; ++bh) forward_one(j, bh, S, z);
    free(S);
    free(z);
    return NULL;
}

/*
 * Whole-sequence forward.  Returns 0 on success, -1 on a bad argument or an
 * allocation failure.  init_state / init_z / final_state / final_z may be
 * NULL.  nthreads <= 0 means one thread.
 */
int la_ref_forward(const double* q, const double* k, const double* v,
                   int decay_kind, const double* log_g, int normalize,
                   const double* init_state, const double* init_z,
                   double* out, double* final_state, double* final_z,
                   int B, int H, int T, int Dk, int Dv, int nthreads)
{
    if (B < 0 || H < 0 || T < 0 || Dk < 1 || Dv < 1) return -1;
    if (decay_kind < 0 || decay_kind > 2) return -1;
    if (decay_kind != 0 && !log_g) return -1;
    const int nbh = B * H;
    if (nbh == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nbh) nthreads = nbh;

    fwd_job* jobs = (fwd_job*)calloc((size_t)nthreads, sizeof(fwd_job));
    pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return -1; }
    int rc = 0;
    for (int w = 0; w < nthreads; ++w) {
        fwd_job* j = &jobs[w];
        j->q = q; j->k = k; j->v = v; j->log_g = log_g;
        j->decay_kind = decay_kind; j->normalize = normalize;
        j->init_state = init_state; j->init_z = init_z;
        j->out = out; j->final_state = final_state; j->final_z = final_z;
        j->B = B; j->H = H; j->T = T; j->Dk = Dk; j->Dv = Dv;
        j->first_bh = (int)((long long)nbh * w / nthreads);
        j->last_bh = (int)((long long)nbh * (w + 1) / nthreads);
    }
    int started = 0;
    for (int w = 1; w < nthreads; ++w) {
        if (pthread_create(&tid[w], NULL, forward_worker, &jobs[w]) != 0) { rc = -1; break; }
        started = w;
    }
    if (rc == 0) forward_worker(&jobs[0]);
    for (int w = 1; w <= started; ++w) pthread_join(tid[w], NULL);
    free(jobs);
    free(tid);
    return rc;
}

/*
 * One decode step for every (b, h), in place on state [B,H,Dk,Dv] and z
 * [B,H,Dk]: the same loop body as one iteration of la_ref_forward's t loop.
 * decay_kind 2 reads log_g as [B,H] (this token's decay).
 */
int la_ref_decode_step(const double* q, const double* k, const double* v,
                       int decay_kind, const double* log_g, int normalize,
                       double* state, double* z, double* out,
                       int B, int H, int Dk, int Dv)
{
    if (B < 0 || H < 0 || Dk < 1 || Dv < 1) return -1;
    if (decay_kind < 0 || decay_kind > 2) return -1;
    if (decay_kind != 0 && !log_g) return -1;
    if (normalize && !z) return -1;
    for (int bh = 0; bh < B * H; ++bh) {
        const double* qt = q + (size_t)bh * Dk;
        const double* kt = k + (size_t)bh * Dk;
        const double* vt = v + (size_t)bh * Dv;
        double* S = state + (size_t)bh * Dk * Dv;
        double* zz = normalize ? z + (size_t)bh * Dk : NULL;
        double g = 1.0;
        if (decay_kind == 1) g = exp(log_g[bh % H]);
        if (decay_kind == 2) g = exp(log_g[bh]);

        for (int i = 0; i < Dk; ++i)
            for (int c = 0; c < Dv; ++c)
                S[i * Dv + c] = g * S[i * Dv + c] + kt[i] * vt[c];
        if (normalize)
            for (int i = 0; i < Dk; ++i) zz[i] = g * zz[i] + kt[i];

        double den = 0.0;
        if (normalize)
            for (int i = 0; i < Dk; ++i) den += qt[i] * zz[i];
        for (int c = 0; c < Dv; ++c) {
            double num = 0.0;
            for (int i = 0; i < Dk; ++i) num += qt[i] * S[i * Dv + c];
            out[(size_t)bh * Dv + c] = normalize ? num / den : num;
        }
    }
    return 0;
}

/*
 * ------------------------------------------------------------------ backward
 *
 * Gradients of a scalar loss through the same recurrence, by the chain rule
 * applied step by step from the last token back to the first (reverse-mode
 * differentiation of the loop above; RWKV-LM discussion 189, opening
 * summary, notes that these gradients are themselves cumulative sums, which
 * the GPU path uses; this oracle uses only the chain rule).  Given
 * dy = dL/dy_t and optionally dL/dS_T, dL/dz_T, with the state gradient
 * G = dL/dS_t and the key-sum gradient w = dL/dz_t carried backwards:
 *
 *   unnormalised:  G += q_t dy_t^T;  dq_t = S_t dy_t
 *   normalised:    n_t = S_t^T q_t, d_t = q_t . z_t, e = dy_t / d_t,
 *                  f = -(dy_t . n_t) / d_t^2;
 *                  G += q_t e^T;  w += f q_t;  dq_t = S_t e + f z_t
 *   then           dk_t = G v_t (+ w);   dv_t = G^T k_t;
 *                  dL/dlog g_t = g_t (<G, S_{t-1}> + <w, z_{t-1}>);
 *                  G <- g_t G;  w <- g_t w
 *
 * and dL/dS_0 = G, dL/dz_0 = w at the end.  S_{t-1} comes from a forward
 * sweep: states are kept every K = ceil(sqrt(T)) tokens and each block of K
 * is recomputed from its checkpoint before it is walked backwards.
 */
typedef struct {
    const double *q, *k, *v, *log_g, *dy;
    int decay_kind, normalize;
    const double *init_state, *init_z, *d_final_state, *d_final_z;
    double *dq, *dk, *dv, *dlog, *d_init_state, *d_init_z;
    int B, H, T, Dk, Dv;
    int first_bh, last_bh;
    int ok;
} bwd_job;

static double bwd_decay(const bwd_job* j, int bh, int t)
{
    return decay_at(j->decay_kind, j->log_g, j->H, j->T, bh, t);
}

/* One step of the forward recurrence on (S, z) for token t. */
static void bwd_step_forward(const bwd_job* j, int bh, int t, double* S, double* z)
{
    const int Dk = j->Dk, Dv = j->Dv;
    const double* kt = j->k + ((size_t)bh * j->T + t) * Dk;
    const double* vt = j->v + ((size_t)bh * j->T + t) * Dv;
    const double g = bwd_decay(j, bh, t);
    for (int i = 0; i < Dk; ++i)
        for (int c = 0; c < Dv; ++c) S[i * Dv + c] = g * S[i * Dv + c] + kt[i] * vt[c];
    if (j->normalize)
        for (int i = 0; i < Dk; ++i) z[i] = g * z[i] + kt[i];
}

static int backward_one(const bwd_job* j, int bh)
{
    const int T = j->T, Dk = j->Dk, Dv = j->Dv, DD = Dk * Dv;
    const size_t ss = (size_t)bh * DD, sz = (size_t)bh * Dk;
    int K = 1;
    while ((long long)K * K < T) ++K;
    const int nblk = T > 0 ? (T + K - 1) / K : 0;
    /* ck[b]: state before block b's first token; blk[i]: state before token b*K+i */
    double* ckS = (double*)malloc(sizeof(double) * (size_t)(nblk + 1) * DD);
    double* ckz = (double*)malloc(sizeof(double) * (size_t)(nblk + 1) * Dk);
    double* blkS = (double*)malloc(sizeof(double) * (size_t)(K + 1) * DD);
    double* blkz = (double*)malloc(sizeof(double) * (size_t)(K + 1) * Dk);
    double* G = (double*)malloc(sizeof(double) * DD);
    double* w = (double*)malloc(sizeof(double) * Dk);
    double* e = (double*)malloc(sizeof(double) * Dv);
    if (!ckS || !ckz || !blkS || !blkz || !G || !w || !e) {
        free(ckS); free(ckz); free(blkS); free(blkz); free(G); free(w); free(e);
        return -1;
    }
    /* forward sweep: checkpoints */
    for (int a = 0; a < DD; ++a) blkS[a] = (j->init_state != NULL) ? j->init_state[ss + a] : 0.0;
    for (int a = 0; a < Dk; ++a) blkz[a] = (j->normalize && j->init_z != NULL) ? j->init_z[sz + a] : 0.0;
    for (int t = 0; t < T; ++t) {
        if (t % K == 0) {
            memcpy(ckS + (size_t)(t / K) * DD, blkS, sizeof(double) * DD);
            memcpy(ckz + (size_t)(t / K) * Dk, blkz, sizeof(double) * Dk);
        }
        bwd_step_forward(j, bh, t, blkS, blkz);
    }
    /* backward sweep */
    for (int a = 0; a < DD; ++a) G[a] = j->d_final_state ? j->d_final_state[ss + a] : 0.0;
    for (int a = 0; a < Dk; ++a) w[a] = (j->normalize && j->d_final_z) ? j->d_final_z[sz + a] : 0.0;
    for (int b = nblk - 1; b >= 0; --b) {
        const int t0 = b * K, t1 = (t0 + K < T) ? t0 + K : T;
        memcpy(blkS, ckS + (size_t)b * DD, sizeof(double) * DD);
        memcpy(blkz, ckz + (size_t)b * Dk, sizeof(double) * Dk);
        for (int t = t0; t < t1; ++t) {
            memcpy(blkS + (size_t)(t - t0 + 1) * DD, blkS + (size_t)(t - t0) * DD, sizeof(double) * DD);
            memcpy(blkz + (size_t)(t - t0 + 1) * Dk, blkz + (size_t)(t - t0) * Dk, sizeof(double) * Dk);
            bwd_step_forward(j, bh, t, blkS + (size_t)(t - t0 + 1) * DD, blkz + (size_t)(t - t0 + 1) * Dk);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            const double* St = blkS + (size_t)(t - t0 + 1) * DD;   /* S_t */
            const double* Sp = blkS + (size_t)(t - t0) * DD;       /* S_{t-1} */
            const double* zt = blkz + (size_t)(t - t0 + 1) * Dk;
            const double* zp = blkz + (size_t)(t - t0) * Dk;
            const size_t rq = ((size_t)bh * T + t) * Dk, rv = ((size_t)bh * T + t) * Dv;
            const double* qt = j->q + rq;
            const double* kt = j->k + rq;
            const double* vt = j->v + rv;
            const double* dyt = j->dy + rv;
            const double g = bwd_decay(j, bh, t);
            double f = 0.0;
            if (j->normalize) {
                double den = 0.0, dn = 0.0;
                for (int i = 0; i < Dk; ++i) den += qt[i] * zt[i];
                for (int c = 0; c < Dv; ++c) {
                    double num = 0.0;
                    for (int i = 0; i < Dk; ++i) num += qt[i] * St[i * Dv + c];
                    dn += dyt[c] * num;
                    e[c] = dyt[c] / den;
                }
                f = -dn / (den * den);
            } else {
                for (int c = 0; c < Dv; ++c) e[c] = dyt[c];
            }
            /* dq_t = S_t e (+ f z_t) */
            for (int i = 0; i < Dk; ++i) {
                double s = 0.0;
                for (int c = 0; c < Dv; ++c) s += St[i * Dv + c] * e[c];
                j->dq[rq + i] = s + (j->normalize ? f * zt[i] : 0.0);
            }
            /* G += q_t e^T, w += f q_t */
            for (int i = 0; i < Dk; ++i)
                for (int c = 0; c < Dv; ++c) G[i * Dv + c] += qt[i] * e[c];
            if (j->normalize)
                for (int i = 0; i < Dk; ++i) w[i] += f * qt[i];
            /* dk_t = G v_t (+ w), dv_t = G^T k_t */
            for (int i = 0; i < Dk; ++i) {
                double s = 0.0;
                for (int c = 0; c < Dv; ++c) s += G[i * Dv + c] * vt[c];
                j->dk[rq + i] = s + (j->normalize ? w[i] : 0.0);
            }
            for (int c = 0; c < Dv; ++c) {
                double s = 0.0;
                for (int i = 0; i < Dk; ++i) s += G[i * Dv + c] * kt[i];
                j->dv[rv + c] = s;
            }
            /* dL/dlog g_t = g_t (<G, S_{t-1}> + <w, z_{t-1}>) */
            double dg = 0.0;
            for (int a = 0; a < DD; ++a) dg += G[a] * Sp[a];
            if (j->normalize)
                for (int i = 0; i < Dk; ++i) dg += w[i] * zp[i];
            if (j->dlog) j->dlog[(size_t)bh * T + t] = g * dg;
            /* carry to S_{t-1}: S_t = g_t S_{t-1} + ... */
            for (int a = 0; a < DD; ++a) G[a] *= g;
            if (j->normalize)
                for (int i = 0; i < Dk; ++i) w[i] *= g;
        }
    }
    if (j->d_init_state)
        for (int a = 0; a < DD; ++a) j->d_init_state[ss + a] = G[a];
    if (j->d_init_z && j->normalize)
        for (int a = 0; a < Dk; ++a) j->d_init_z[sz + a] = w[a];
    free(ckS); free(ckz); free(blkS); free(blkz); free(G); free(w); free(e);
    return 0;
}

static void* backward_worker(void* arg)
{
    bwd_job* j = (bwd_job*)arg;
    j->ok = 1;
    for (int bh = j->first_bh; bh < j->last_bh; ++bh)
        if (backward_one(j, bh) != 0) { j->ok = 0; break; }
    return NULL;
}

/*
 * Whole-sequence backward.  dlog receives dL/dlog g_t per token [B,H,T]
 * (for a per-head decay the caller sums it over b and t).  Optional (NULL):
 * init_state, init_z, d_final_state, d_final_z, dlog, d_init_state, d_init_z.
 * Returns 0, or -1 on a bad argument or an allocation failure.
 */
int la_ref_backward(const double* q, const double* k, const double* v,
                    int decay_kind, const double* log_g, int normalize,
                    const double* init_state, const double* init_z,
                    const double* dy, const double* d_final_state, const double* d_final_z,
                    double* dq, double* dk, double* dv, double* dlog,
                    double* d_init_state, double* d_init_z,
                    int B, int H, int T, int Dk, int Dv, int nthreads)
{
    if (B < 0 || H < 0 || T < 0 || Dk < 1 || Dv < 1) return -1;
    if (decay_kind < 0 || decay_kind > 2) return -1;
    if (decay_kind != 0 && !log_g) return -1;
    const int nbh = B * H;
    if (nbh == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nbh) nthreads = nbh;
    bwd_job* jobs = (bwd_job*)calloc((size_t)nthreads, sizeof(bwd_job));
    pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return -1; }
    for (int w = 0; w < nthreads; ++w) {
        bwd_job* j = &jobs[w];
        j->q = q; j->k = k; j->v = v; j->log_g = log_g; j->dy = dy;
        j->decay_kind = decay_kind; j->normalize = normalize;
        j->init_state = init_state; j->init_z = init_z;
        j->d_final_state = d_final_state; j->d_final_z = d_final_z;
        j->dq = dq; j->dk = dk; j->dv = dv; j->dlog = dlog;
        j->d_init_state = d_init_state; j->d_init_z = d_init_z;
        j->B = B; j->H = H; j->T = T; j->Dk = Dk; j->Dv = Dv;
        j->first_bh = (int)((long long)nbh * w / nthreads);
        j->last_bh = (int)((long long)nbh * (w + 1) / nthreads);
    }
    int rc = 0, started = 0;
    for (int w = 1; w < nthreads; ++w) {
        if (pthread_create(&tid[w], NULL, backward_worker, &jobs[w]) != 0) { rc = -1; break; }
        started = w;
    }
    if (rc == 0) backward_worker(&jobs[0]);
    for (int w = 1; w <= started; ++w) pthread_join(tid[w], NULL);
    for (int w = 0; w <= started && rc == 0; ++w)
        if (!jobs[w].ok) rc = -1;
    free(jobs);
    free(tid);
    return rc;
}
