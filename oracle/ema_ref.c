/*
 * ema_ref.c - the oracle of the cumulative exponential moving average: a
 * plain, slow, float64 CPU implementation.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load or call this code.  It shares no code
 * with the CUDA library and is not a fallback for it.
 *
 * Source: Jamie-Stirling/RetNet issue 21, "Proposed improvement/
 * collaboration: removing the O(T^2) training cost", the cumulative_ema
 * function: element-wise values and factors of the same shape, scanned
 * along one axis so that each output is the previous output times this
 * step's factor plus this step's value.  (The function's docstring, as
 * extracted, adds the next output instead of the next value; the pairing
 * operator that the function applies adds the value, and that reading is
 * the one taken.)  The first output is the first value.  The reverse
 * flag gives the non-reversed scan of the time-reversed arguments, reversed
 * back, i.e. the same recurrence run from the last step to the first.  A
 * carried state s (0 when absent) enters before the first step of the scan:
 * out_first = f_first * s + x_first.
 *
 * Layouts: x, f, out [B, T, C] (the scanned axis T, channels fastest);
 * init_state, final_state [B, C].  Every (b, c) is an independent loop.
 */
#include <stddef.h>

int la_ref_ema(const double* x, const double* f, const double* init_state, double* out, double* final_state,
               int B, int T, int C, int reverse)
{
    if (B < 0 || T < 0 || C < 1) return -1;
    if (B > 0 && T > 0 && (!x || !f || !out)) return -1;
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < C; ++c) {
            double s = init_state ? init_state[(size_t)b * C + c] : 0.0;
            for (int step = 0; step < T; ++step) {
                const int t = reverse ? T - 1 - step : step;
                const size_t i = ((size_t)b * T + t) * C + c;
                s = f[i] * s + x[i];
                out[i] = s;
            }
            if (final_state) final_state[(size_t)b * C + c] = s;
        }
    }
    return 0;
}
