// la_fwd_f32.cu - whole-sequence forward for fp32 inputs, on fp32 FMA units.
//
// One CTA per (b, h) runs the recurrence token by token (the tensortonic
// "CS336 L04 linear attention duality" recurrent form, with the per-step
// decay of RetNet issue 21 and the key-sum normaliser of
// flash-linear-attention issue 268).  The fp32 state S [Dk, Dv] lives in
// shared memory; thread c owns value column c, so the update of column c
// and its read-out q_t^T S_t[:, c] need no synchronisation.  No TF32: every
// product is an fp32 FMA.
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kThreads = 128;

__global__ void __launch_bounds__(kThreads) fwd_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    int decay_kind, const float* __restrict__ log_g, int normalize,
    const float* __restrict__ init_state, const float* __restrict__ init_z,
    float* __restrict__ out, float* __restrict__ final_state, float* __restrict__ final_z,
    int H, int T, int Dk, int Dv) {
    extern __shared__ float smem[];
    float* S = smem;                    // [Dk][Dv]
    float* qs = S + Dk * Dv;            // [Dk]
    float* ks = qs + Dk;                // [Dk]
    float* vs = ks + Dk;                // [Dv]
    float* zs = vs + Dv;                // [Dk]

    const int bh = blockIdx.x;
    const int h = bh % H;
    const int tid = threadIdx.x;
    const size_t sq = static_cast<size_t>(bh) * T * Dk;
    const size_t sv = static_cast<size_t>(bh) * T * Dv;

    for (int e = tid; e < Dk * Dv; e += kThreads)
        S[e] = init_state ? init_state[static_cast<size_t>(bh) * Dk * Dv + e] : 0.f;
    for (int i = tid; i < Dk; i += kThreads)
        zs[i] = (normalize && init_z) ? init_z[static_cast<size_t>(bh) * Dk + i] : 0.f;
    const float g_head = decay_kind == LA_DECAY_PER_HEAD ? expf(log_g[h]) : 1.f;

    for (int t = 0; t < T; ++t) {
        __syncthreads();  // previous token's readers are done with qs/ks/vs
        for (int i = tid; i < Dk; i += kThreads) {
            qs[i] = q[sq + static_cast<size_t>(t) * Dk + i];
            ks[i] = k[sq + static_cast<size_t>(t) * Dk + i];
        }
        for (int c = tid; c < Dv; c += kThreads) vs[c] = v[sv + static_cast<size_t>(t) * Dv + c];
        const float g = decay_kind == LA_DECAY_PER_STEP ? expf(log_g[static_cast<size_t>(bh) * T + t])
                                                         : g_head;
        __syncthreads();

        if (normalize)
            for (int i = tid; i < Dk; i += kThreads) zs[i] = fmaf(g, zs[i], ks[i]);
        // thread c owns value column c (Dv <= kThreads)
        float num = 0.f;
        if (tid < Dv) {
            const float vc = vs[tid];
            for (int i = 0; i < Dk; ++i) {
                const float s = fmaf(ks[i], vc, g * S[i * Dv + tid]);
                S[i * Dv + tid] = s;
                num = fmaf(qs[i], s, num);
            }
            if (!normalize) out[sv + static_cast<size_t>(t) * Dv + tid] = num;
        }
        if (normalize) {
            __syncthreads();  // z_t complete
            float den = 0.f;
            for (int i = 0; i < Dk; ++i) den = fmaf(qs[i], zs[i], den);
            if (tid < Dv) out[sv + static_cast<size_t>(t) * Dv + tid] = num / den;
        }
    }
    __syncthreads();
    if (final_state)
        for (int e = tid; e < Dk * Dv; e += kThreads)
            final_state[static_cast<size_t>(bh) * Dk * Dv + e] = S[e];
    if (final_z && normalize)
        for (int i = tid; i < Dk; i += kThreads) final_z[static_cast<size_t>(bh) * Dk + i] = zs[i];
}

}  // namespace

cudaError_t launch_fwd_f32(const FwdArgs& a) {
    const size_t smem = sizeof(float) * (static_cast<size_t>(a.Dk) * a.Dv + 3 * a.Dk + a.Dv);
    cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    fwd_f32_kernel<<<a.B * a.H, kThreads, smem, a.stream>>>(
        static_cast<const float*>(a.q), static_cast<const float*>(a.k), static_cast<const float*>(a.v),
        a.decay_kind, a.log_g, a.normalize, a.init_state, a.init_z, static_cast<float*>(a.out),
        a.final_state, a.final_z, a.H, a.T, a.Dk, a.Dv);
    return cudaGetLastError();
}

}  // namespace la
