/*
 * wkv4_ref.c - the oracle of the RWKV-4 WKV recurrence: a plain, slow,
 * float64 CPU implementation.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load or call this code.  It shares no code
 * with the CUDA library and is not a fallback for it.
 *
 * Source: BlinkDL/RWKV-LM issue 167, "Questions about formula 14 and code
 * implementation in the paper" (opening comment: formula 14 and the
 * recurrent form of the WKV operator).  Per batch b and channel c, with a
 * time decay w (natural log of the per-step factor, <= 0) and a bonus u for
 * the current token, both per channel, the output at token t is the weighted
 * average of the values seen so far,
 *
 *   wkv_t = ( sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u + k_t}     ).
 *
 * This file evaluates that definition directly as an online weighted mean:
 * before token t it keeps the mean R = N / D of the earlier values under
 * their weights (N and D the two sums over i < t) and the log of the total
 * weight, L = log D.  Adding a value x with log weight a to a mean (R, L)
 * moves the mean towards x by the new value's share of the total weight,
 * sigma(a - L) = e^a / (e^L + e^a), and the log weight becomes
 * logaddexp(L, a).  So, per token:
 *   out_t = R + sigma(u + k_t - L) (v_t - R)           (bonus weight, not kept)
 *   R    <- R + sigma(k_t - (w + L)) (v_t - R)         (earlier weights decayed by e^w)
 *   L    <- logaddexp(w + L, k_t)
 * No exponential of a key is formed, only of differences of log weights;
 * an empty state (no weight yet) is L = -infinity.
 *
 * State interface: [B, 3, C] with the planes (aa, bb, pp), read as the sums
 * N = e^pp aa and D = e^pp bb (the representation the library's kernel uses;
 * it is not unique: (aa e^s, bb e^s, pp - s) is the same state).  On input
 * R = aa / bb and L = pp + log bb (bb = 0: the empty state); on output
 * (aa, bb, pp) = (R, 1, L), or (0, 0, -1e38) for a state that is still empty.
 * Layouts: k, v, out [B, T, C]; w, u [C].  Every (b, c) is an independent
 * sequential loop over t.
 */
#include <math.h>
#include <stddef.h>

#define WKV4_EMPTY_SCALE (-1e38)

/* The logistic function 1 / (1 + e^-x), without overflow for large |x|. */
static double sigmoid(double x)
{
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    const double e = exp(x);
    return e / (1.0 + e);
}

/* log(e^a + e^b), exact for a or b = -infinity. */
static double logaddexp(double a, double b)
{
    if (a == -INFINITY) return b;
    if (b == -INFINITY) return a;
    const double hi = a > b ? a : b, lo = a > b ? b : a;
    return hi + log1p(exp(lo - hi));
}

/*
 * Returns 0, or -1 on a bad argument.  init_state / final_state may be NULL
 * (an empty state / not written).
 */
int la_ref_wkv4(const double* k, const double* v, const double* w, const double* u,
                const double* init_state, double* out, double* final_state, int B, int T, int C)
{
    if (B < 0 || T < 0 || C < 1 || !w || !u) return -1;
    if (B > 0 && T > 0 && (!k || !v || !out)) return -1;
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < C; ++c) {
            const size_t s = (size_t)b * 3 * C + c;
            double mean = 0.0, logw = -INFINITY;  /* R and L: no weight yet */
            if (init_state && init_state[s + C] > 0.0) {
                mean = init_state[s] / init_state[s + C];
                logw = init_state[s + 2 * C] + log(init_state[s + C]);
            }
            for (int t = 0; t < T; ++t) {
                const size_t i = ((size_t)b * T + t) * C + c;
                const double kt = k[i], vt = v[i];
                /* the current token joins the earlier ones with the bonus weight */
                out[i] = mean + sigmoid(u[c] + kt - logw) * (vt - mean);
                /* then, without the bonus, into the decayed state */
                const double decayed = logw + w[c];
                mean += sigmoid(kt - decayed) * (vt - mean);
                logw = logaddexp(decayed, kt);
            }
            if (final_state) {
                const int empty = logw == -INFINITY;
                final_state[s] = empty ? 0.0 : mean;
                final_state[s + C] = empty ? 0.0 : 1.0;
                final_state[s + 2 * C] = empty ? WKV4_EMPTY_SCALE : logw;
            }
        }
    }
    return 0;
}
