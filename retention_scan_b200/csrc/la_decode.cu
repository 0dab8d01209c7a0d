// la_decode.cu - one token of the recurrence, state updated in place.
//
//   S <- g S + k v^T,  z <- g z + k,  y = q^T S (/ q^T z)
//
// This is the generation-time path of flash-linear-attention issue 268 (only
// the newest token is passed, the KV state and the key sum are carried), with
// the decay of RetNet issue 21.  It is bound by HBM: every call reads and
// writes the whole fp32 state once (8 Dk Dv bytes per (b, h)) and does 4 Dk Dv
// flops on it.
//
// Layout of the work: one CTA of 256 threads per (b, h).  Thread i owns the
// float4 column block c4 = i % (Dv/4) and the rows r = i / (Dv/4) + n R,
// R = 256 / (Dv/4).  Each warp therefore streams whole 16-byte-aligned row
// segments (coalesced), with eight independent 16-byte loads in flight per
// thread before any store.  State traffic uses streaming (evict-first) cache
// hints because a state is touched once per call.  Column partial sums of
// q^T S' are reduced through shared memory; q^T z' by warp shuffles.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;  // rows loaded before they are updated

__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(p);
    const float2 a = __bfloat1622float2(h[0]);
    const float2 b = __bfloat1622float2(h[1]);
    return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(float* p, float4 x) { *reinterpret_cast<float4*>(p) = x; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 x) {
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(p);
    h[0] = __floats2bfloat162_rn(x.x, x.y);
    h[1] = __floats2bfloat162_rn(x.z, x.w);
}
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// The prologue's feature map: elu(x) + 1 = (x > 0 ? x + 1 : e^x).
__device__ __forceinline__ float feature(float x, int fmap) {
    return fmap == LA_FEATURE_ELU1 ? (x > 0.f ? x + 1.f : expf(x)) : x;
}

__device__ __forceinline__ float decay_of(int kind, const float* log_g, int bh, int h) {
    if (kind == LA_DECAY_PER_HEAD) return expf(log_g[h]);
    if (kind == LA_DECAY_PER_STEP) return expf(log_g[bh]);
    return 1.f;
}

// Sum of x over the CTA; every thread gets the result.  `red` holds one float
// per warp.
__device__ __forceinline__ float block_sum(float x, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    if (l == 0) red[w] = x;
    __syncthreads();
    float s = 0.f;
    for (int i = 0; i < static_cast<int>(blockDim.x) / 32; ++i) s += red[i];
    return s;
}

template <typename TIn, int C4>
__global__ void __launch_bounds__(kThreads) decode_vec_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v, int decay_kind,
    const float* __restrict__ log_g, int normalize, float* __restrict__ state, float* __restrict__ z,
    TIn* __restrict__ out, int H, int Dk, int fmap, float qscale) {
    constexpr int Dv = 4 * C4;
    constexpr int R = kThreads / C4;
    __shared__ float qs[128], ks[128];
    __shared__ float4 part[kThreads];
    __shared__ float red[kThreads / 32];

    const int bh = blockIdx.x, tid = threadIdx.x;
    const float g = decay_of(decay_kind, log_g, bh, bh % H);
    if (tid < Dk) {
        qs[tid] = qscale * feature(to_f(q[static_cast<size_t>(bh) * Dk + tid]), fmap);
        ks[tid] = feature(to_f(k[static_cast<size_t>(bh) * Dk + tid]), fmap);
    }
    const int c4 = tid % C4, r0 = tid / C4;
    const float4 vv = load4(v + static_cast<size_t>(bh) * Dv + 4 * c4);
    __syncthreads();

    float4* S4 = reinterpret_cast<float4*>(state + static_cast<size_t>(bh) * Dk * Dv);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = r0; i0 < Dk; i0 += kBatch * R) {
        float4 s[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * R;
            if (i < Dk) s[u] = __ldcs(S4 + i * C4 + c4);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * R;
            if (i < Dk) {
                const float ki = ks[i], qi = qs[i];
                float4 x = s[u];
                x.x = fmaf(ki, vv.x, g * x.x);
                x.y = fmaf(ki, vv.y, g * x.y);
                x.z = fmaf(ki, vv.z, g * x.z);
                x.w = fmaf(ki, vv.w, g * x.w);
                __stcs(S4 + i * C4 + c4, x);
                acc.x = fmaf(qi, x.x, acc.x);
                acc.y = fmaf(qi, x.y, acc.y);
                acc.z = fmaf(qi, x.z, acc.z);
                acc.w = fmaf(qi, x.w, acc.w);
            }
        }
    }
    part[tid] = acc;

    float den = 1.f;
    if (normalize) {
        float p = 0.f;
        for (int i = tid; i < Dk; i += kThreads) {
            float* zp = z + static_cast<size_t>(bh) * Dk + i;
            const float zi = fmaf(g, *zp, ks[i]);
            *zp = zi;
            p = fmaf(qs[i], zi, p);
        }
        den = block_sum(p, red);  // contains a __syncthreads
    } else {
        __syncthreads();
    }
    if (tid < C4) {
        float4 y = part[tid];
        for (int r = 1; r < R; ++r) {
            const float4 o = part[r * C4 + tid];
            y.x += o.x; y.y += o.y; y.z += o.z; y.w += o.w;
        }
        if (normalize) { y.x /= den; y.y /= den; y.z /= den; y.w /= den; }
        store4(out + static_cast<size_t>(bh) * Dv + 4 * tid, y);
    }
}

// Any Dk, Dv <= 128: thread c owns value column c and walks the rows.
template <typename TIn>
__global__ void __launch_bounds__(128) decode_generic_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v, int decay_kind,
    const float* __restrict__ log_g, int normalize, float* __restrict__ state, float* __restrict__ z,
    TIn* __restrict__ out, int H, int Dk, int Dv, int fmap, float qscale) {
    __shared__ float qs[128], ks[128];
    __shared__ float red[4];
    const int bh = blockIdx.x, tid = threadIdx.x;
    const float g = decay_of(decay_kind, log_g, bh, bh % H);
    if (tid < Dk) {
        qs[tid] = qscale * feature(to_f(q[static_cast<size_t>(bh) * Dk + tid]), fmap);
        ks[tid] = feature(to_f(k[static_cast<size_t>(bh) * Dk + tid]), fmap);
    }
    __syncthreads();
    float num = 0.f;
    if (tid < Dv) {
        const float vc = to_f(v[static_cast<size_t>(bh) * Dv + tid]);
        float* S = state + static_cast<size_t>(bh) * Dk * Dv;
        for (int i = 0; i < Dk; ++i) {
            const float s = fmaf(ks[i], vc, g * S[i * Dv + tid]);
            S[i * Dv + tid] = s;
            num = fmaf(qs[i], s, num);
        }
    }
    float den = 1.f;
    if (normalize) {
        float p = 0.f;
        if (tid < Dk) {
            float* zp = z + static_cast<size_t>(bh) * Dk + tid;
            const float zi = fmaf(g, *zp, ks[tid]);
            *zp = zi;
            p = qs[tid] * zi;
        }
        den = block_sum(p, red);
    }
    if (tid < Dv) from_f(out + static_cast<size_t>(bh) * Dv + tid, normalize ? num / den : num);
}

template <typename TIn>
cudaError_t launch_typed(const DecodeArgs& a) {
    const TIn* q = static_cast<const TIn*>(a.q);
    const TIn* k = static_cast<const TIn*>(a.k);
    const TIn* v = static_cast<const TIn*>(a.v);
    TIn* out = static_cast<TIn*>(a.out);
    const int grid = a.B * a.H;
#define LA_DECODE_VEC(C4)                                                                            \
    decode_vec_kernel<TIn, C4><<<grid, kThreads, 0, a.stream>>>(q, k, v, a.decay_kind, a.log_g,     \
                                                                 a.normalize, a.state, a.z, out, a.H, \
                                                                 a.Dk, a.feature_map, a.q_scale)
    switch (a.Dv) {
        case 4: LA_DECODE_VEC(1); break;
        case 8: LA_DECODE_VEC(2); break;
        case 16: LA_DECODE_VEC(4); break;
        case 32: LA_DECODE_VEC(8); break;
        case 64: LA_DECODE_VEC(16); break;
        case 128: LA_DECODE_VEC(32); break;
        default:
            decode_generic_kernel<TIn><<<grid, 128, 0, a.stream>>>(q, k, v, a.decay_kind, a.log_g,
                                                                   a.normalize, a.state, a.z, out, a.H,
                                                                   a.Dk, a.Dv, a.feature_map, a.q_scale);
    }
#undef LA_DECODE_VEC
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, la_dtype dtype) {
    return dtype == LA_BF16 ? launch_typed<__nv_bfloat16>(a) : launch_typed<float>(a);
}

}  // namespace la
