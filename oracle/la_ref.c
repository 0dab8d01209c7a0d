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

/* Decay factor of token t of sequence (b, h). */
static double decay_factor(const fwd_job* j, int bh, int t)
{
    if (j->decay_kind == 0) return 1.0;
    if (j->decay_kind == 1) return exp(j->log_g[bh % j->H]);
    return exp(j->log_g[(size_t)bh * j->T + t]);
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
