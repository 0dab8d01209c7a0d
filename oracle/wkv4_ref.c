/*
 * wkv4_ref.c - the oracle of the RWKV-4 WKV recurrence: a plain, slow,
 * float64 CPU implementation.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load or call this code.  It shares no code
 * with the CUDA library and is not a fallback for it.
 *
 * Source: BlinkDL/RWKV-LM issue 167, "Questions about formula 14 and code
 * implementation in the paper" (the att_seq time loop quoted in the opening
 * comment).  Per batch b and channel c, with a time decay w (natural log of
 * the per-step factor, <= 0) and a bonus u for the current token, both per
 * channel, the output at token t is the weighted average
 *
 *   wkv_t = ( sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u + k_t}     )
 *
 * and the loop carries the two sums as (aa, bb) measured against a running
 * log scale pp (the true sums are e^pp aa and e^pp bb), so that no exponential
 * of a large key is ever formed: each step takes the larger of the two log
 * weights it combines as the new scale and exponentiates only differences
 * that are <= 0.  Per token, in the page's order:
 *   1. read-out: combine the state (log weight pp) with the current token
 *      (log weight u + k_t) and divide;
 *   2. update: decay the state (log weight w + pp) and add the current token
 *      (log weight k_t); the larger log weight becomes the new pp.
 * An empty state is aa = bb = 0 with pp = -1e38 (a finite stand-in for
 * minus infinity, so that pp - p stays a number).
 *
 * Layouts: k, v, out [B, T, C]; w, u [C]; state [B, 3, C] holding the planes
 * aa, bb, pp.  Every (b, c) is an independent sequential loop over t.
 */
#include <math.h>
#include <stddef.h>

#define WKV4_EMPTY_SCALE (-1e38)

/* Weights of two terms with log weights la and lb against their larger log
 * weight: *fa = e^(la - m), *fb = e^(lb - m); returns m. */
static double shifted_pair(double la, double lb, double* fa, double* fb)
{
    const double m = la > lb ? la : lb;
    *fa = exp(la - m);
    *fb = exp(lb - m);
    return m;
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
            double aa = init_state ? init_state[s] : 0.0;
            double bb = init_state ? init_state[s + C] : 0.0;
            double pp = init_state ? init_state[s + 2 * C] : WKV4_EMPTY_SCALE;
            for (int t = 0; t < T; ++t) {
                const size_t i = ((size_t)b * T + t) * C + c;
                const double kt = k[i], vt = v[i];
                double fs, fx;
                /* 1. read-out: state at log weight pp, this token at u + k_t */
                shifted_pair(pp, u[c] + kt, &fs, &fx);
                out[i] = (fs * aa + fx * vt) / (fs * bb + fx);
                /* 2. update: state decayed to w + pp, this token added at k_t */
                const double m = shifted_pair(w[c] + pp, kt, &fs, &fx);
                aa = fs * aa + fx * vt;
                bb = fs * bb + fx;
                pp = m;
            }
            if (final_state) {
                final_state[s] = aa;
                final_state[s + C] = bb;
                final_state[s + 2 * C] = pp;
            }
        }
    }
    return 0;
}
