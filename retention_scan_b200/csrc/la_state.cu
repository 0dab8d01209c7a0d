// la_state.cu - states of consecutive spans of a sequence, and their fold.
//
// A span that starts from the zero state leaves (S_j, z_j) and multiplies
// whatever state enters it by its total decay G_j = exp(L_j), L_j the sum of
// its log decays.  Consecutive spans combine with the associative operator of
// RetNet issue 21 ("Proposed improvement/collaboration: removing the O(T^2)
// training cost", the paragraph on the associative EMA operator):
//     (S_a, G_a) o (S_b, G_b) = (G_b S_a + S_b, G_a G_b),
// so the state after spans 0..n-1 entered with S_init is the left fold
//     S <- S_init;  for j = 0..n-1:  S <- exp(L_j) S + S_j       (z likewise)
// and the fold's total log decay is sum_j L_j.  One thread per output element
// folds its n inputs in span order; the fold is tiny next to the scans that
// produce the spans.
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) fold_kernel(const CombineArgs a) {
    const long long DkDv = static_cast<long long>(a.Dk) * a.Dv;
    const long long nS = a.BH * DkDv;
    const long long nz = a.out_z ? static_cast<long long>(a.BH) * a.Dk : 0;
    const long long nL = a.out_L ? a.BH : 0;
    const long long total = nS + nz + nL;
    for (long long i = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * kThreads) {
        if (i < nS + nz) {
            const bool is_S = i < nS;
            const long long r = is_S ? i : i - nS;
            const long long width = is_S ? DkDv : a.Dk;
            const int bh = static_cast<int>(r / width);
            const long long e = r % width;
            const float* init = is_S ? a.init_S : a.init_z;
            float acc = init ? init[static_cast<long long>(bh) * width + e] : 0.f;
            for (int j = 0; j < a.n; ++j) {
                const float L = a.L[j * a.L_span + bh * a.L_bh];
                const float g = a.log2_units ? exp2f(L) : expf(L);
                const float x = is_S ? a.S[j * a.S_span + bh * a.S_bh + e] : a.z[j * a.z_span + bh * a.z_bh + e];
                acc = fmaf(g, acc, x);
            }
            (is_S ? a.out_S : a.out_z)[static_cast<long long>(bh) * width + e] = acc;
        } else {
            const int bh = static_cast<int>(i - nS - nz);
            float L = 0.f;
            for (int j = 0; j < a.n; ++j) L += a.L[j * a.L_span + bh * a.L_bh];
            a.out_L[bh] = a.log2_units ? L * 0.6931471805599453f : L;
        }
    }
}

// Natural-log total of a sequence's decay per (b, h), summed in double.
__global__ void __launch_bounds__(kThreads) log_total_kernel(const float* log_g, int kind, int H, int T, float* out) {
    const int bh = blockIdx.x;
    double s = 0.0;
    if (kind == LA_DECAY_PER_STEP) {
        const float* l = log_g + static_cast<size_t>(bh) * T;
        for (int t = threadIdx.x; t < T; t += kThreads) s += l[t];
    } else if (kind == LA_DECAY_PER_HEAD && threadIdx.x == 0) {
        s = static_cast<double>(log_g[bh % H]) * T;
    }
    __shared__ double part[kThreads / 32];
    for (int o = 16; o > 0; o /= 2) s += __shfl_down_sync(0xffffffffu, s, o);
    if (threadIdx.x % 32 == 0) part[threadIdx.x / 32] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < kThreads / 32; ++w) t += part[w];
        out[bh] = static_cast<float>(t);
    }
}

}  // namespace

cudaError_t launch_fold(const CombineArgs& a) {
    const long long total = static_cast<long long>(a.BH) * a.Dk * a.Dv + (a.out_z ? 1LL * a.BH * a.Dk : 0) +
                            (a.out_L ? a.BH : 0);
    if (total == 0) return cudaSuccess;
    const long long blocks = (total + kThreads - 1) / kThreads;
    fold_kernel<<<static_cast<int>(blocks < 148 * 16 ? blocks : 148 * 16), kThreads, 0, a.stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_log_total(const float* log_g, int kind, int BH, int H, int T, float* out, cudaStream_t stream) {
    if (BH == 0) return cudaSuccess;
    log_total_kernel<<<BH, kThreads, 0, stream>>>(log_g, kind, H, T, out);
    return cudaGetLastError();
}

}  // namespace la
