// la_fwd_f32.cu - whole-sequence forward (or reverse) scan for fp32 inputs,
// on fp32 FMA units.
//
// One CTA per (b, h) runs the recurrence token by token (the tensortonic
// "CS336 L04 linear attention duality" recurrent form, with the per-step
// decay of RetNet issue 21 and the key-sum normaliser of
// flash-linear-attention issue 268; the reverse scan is the same recurrence
// from the last token back to the first).  Thread c owns value column c of
// the fp32 state S [Dk, Dv] and holds it in registers (the key width padded
// to a compile-time bound), so the update of column c and its read-out
// q_t^T S_t[:, c] touch no shared memory and need no synchronisation; the
// read-out's sum runs as four interleaved chains.  Tokens are staged kTile
// at a time: one coalesced load of the tile's q, k, v and decays, then the
// tile's steps run without a barrier (with the normaliser, the threads that
// own z write q_t,i z_t,i for the whole tile first and one barrier later
// every thread sums its token's row).  No TF32: every product is an fp32
// FMA.
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kThreads = 128;
constexpr int kTile = 32;

// The prologue's feature map: elu(x) + 1 = (x > 0 ? x + 1 : e^x).
__device__ __forceinline__ float feature(float x, int fmap) {
    return fmap == LA_FEATURE_ELU1 ? (x > 0.f ? x + 1.f : expf(x)) : x;
}

template <int DKP>
__global__ void __launch_bounds__(kThreads) fwd_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    int decay_kind, const float* __restrict__ log_g, int normalize,
    const float* __restrict__ init_state, const float* __restrict__ init_z,
    float* __restrict__ out, float* __restrict__ final_state, float* __restrict__ final_z,
    int H, int T, int Dk, int Dv, int reverse, int accumulate, int fmap, float qscale) {
    extern __shared__ float smem[];
    float* qs = smem;                   // [kTile][Dk]
    float* ks = qs + kTile * Dk;        // [kTile][Dk]
    float* vs = ks + kTile * Dk;        // [kTile][Dv]
    float* gs = vs + kTile * Dv;        // [kTile]
    float* qz = gs + kTile;             // [kTile][Dk]: q_t,i z_t,i (normaliser only)

    const int bh = blockIdx.x;
    const int h = bh % H;
    const int tid = threadIdx.x;
    const bool own = tid < Dv;  // thread c owns value column c
    const size_t sq = static_cast<size_t>(bh) * T * Dk;
    const size_t sv = static_cast<size_t>(bh) * T * Dv;
    const size_t s0 = static_cast<size_t>(bh) * Dk * Dv;

    float S[DKP];  // S[i][tid], i < Dk
#pragma unroll
    for (int i = 0; i < DKP; ++i) S[i] = (own && i < Dk && init_state) ? init_state[s0 + static_cast<size_t>(i) * Dv + tid] : 0.f;
    float zi = 0.f;  // z_i, owned by thread i < Dk
    if (normalize && init_z && tid < Dk) zi = init_z[static_cast<size_t>(bh) * Dk + tid];
    const float g_head = decay_kind == LA_DECAY_PER_HEAD ? expf(log_g[h]) : 1.f;

    const int ntiles = (T + kTile - 1) / kTile;
    for (int it = 0; it < ntiles; ++it) {
        const int tile = reverse ? ntiles - 1 - it : it;
        const int t0 = tile * kTile, nt = min(kTile, T - t0);
        __syncthreads();  // the previous tile's readers are done
        for (int e = tid; e < nt * Dk; e += kThreads) {
            qs[e] = qscale * feature(q[sq + static_cast<size_t>(t0) * Dk + e], fmap);
            ks[e] = feature(k[sq + static_cast<size_t>(t0) * Dk + e], fmap);
        }
        for (int e = tid; e < nt * Dv; e += kThreads) vs[e] = v[sv + static_cast<size_t>(t0) * Dv + e];
        for (int j = tid; j < nt; j += kThreads)
            gs[j] = decay_kind == LA_DECAY_PER_STEP ? expf(log_g[static_cast<size_t>(bh) * T + t0 + j]) : g_head;
        __syncthreads();

        if (normalize) {
            if (tid < Dk)
                for (int jj = 0; jj < nt; ++jj) {
                    const int j = reverse ? nt - 1 - jj : jj;
                    zi = fmaf(gs[j], zi, ks[j * Dk + tid]);
                    qz[j * Dk + tid] = qs[j * Dk + tid] * zi;
                }
            __syncthreads();
        }
        if (own) {
            for (int jj = 0; jj < nt; ++jj) {
                const int j = reverse ? nt - 1 - jj : jj;
                const float vc = vs[j * Dv + tid], g = gs[j];
                const float* qj = qs + j * Dk;
                const float* kj = ks + j * Dk;
                float num[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < DKP; ++i) {
                    if (i < Dk) {
                        S[i] = fmaf(kj[i], vc, g * S[i]);
                        num[i & 3] = fmaf(qj[i], S[i], num[i & 3]);
                    }
                }
                float y = (num[0] + num[1]) + (num[2] + num[3]);
                if (normalize) {
                    float den = 0.f;
                    for (int i = 0; i < Dk; ++i) den += qz[j * Dk + i];
                    y = y / den;
                }
                if (out) {  // (null: the state alone, la_chunk_state_ws)
                    float* o = out + sv + static_cast<size_t>(t0 + j) * Dv + tid;
                    *o = accumulate ? *o + y : y;
                }
            }
        }
    }
    if (final_state && own)
#pragma unroll
        for (int i = 0; i < DKP; ++i)
            if (i < Dk) final_state[s0 + static_cast<size_t>(i) * Dv + tid] = S[i];
    if (final_z && normalize && tid < Dk) final_z[static_cast<size_t>(bh) * Dk + tid] = zi;
}

template <int DKP>
cudaError_t launch_f32(const FwdArgs& a) {
    const size_t smem = sizeof(float) * (3 * kTile * static_cast<size_t>(a.Dk) + kTile * a.Dv + kTile);
    cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<DKP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    fwd_f32_kernel<DKP><<<a.B * a.H, kThreads, smem, a.stream>>>(
        static_cast<const float*>(a.q), static_cast<const float*>(a.k), static_cast<const float*>(a.v),
        a.decay_kind, a.log_g, a.normalize, a.init_state, a.init_z, static_cast<float*>(a.out),
        a.final_state, a.final_z, a.H, a.T, a.Dk, a.Dv, a.reverse, a.accumulate, a.feature_map, a.q_scale);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_f32(const FwdArgs& a) {
    // the state column's registers: the key width padded to 16, 32, 64 or 128
    if (a.Dk <= 16) return launch_f32<16>(a);
    if (a.Dk <= 32) return launch_f32<32>(a);
    if (a.Dk <= 64) return launch_f32<64>(a);
    return launch_f32<128>(a);
}

}  // namespace la
