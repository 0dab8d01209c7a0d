// la_bwd.cu - the small kernels of the backward pass: transposed carried
// states, the decay shifted by one token for the reverse scans, the gradient
// of the initial state, and the gradient of the log decay as a suffix sum.
// The three scans that give dq, dk and dv run on the forward and reverse scan
// kernels (la_api.cu orchestrates them).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kDlogTokens = 256;  // tokens per block of the decay-gradient scan

int grid_for(long long n, int threads) {
    const long long b = (n + threads - 1) / threads;
    return static_cast<int>(std::min<long long>(std::max<long long>(b, 1), 148LL * 16));
}

// One 32 x 32 tile per block (32 x 8 threads); the tile passes through
// shared memory so that both the read and the write are coalesced.
__global__ void transpose_kernel(const float* __restrict__ in, float* __restrict__ out, int BH, int R, int C) {
    __shared__ float tile[32][33];
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    for (int bh = blockIdx.z; bh < BH; bh += gridDim.z) {
        const float* src = in + static_cast<size_t>(bh) * R * C;
        float* dst = out + static_cast<size_t>(bh) * R * C;
        for (int i = threadIdx.y; i < 32; i += 8) {
            const int r = r0 + i, c = c0 + threadIdx.x;
            if (r < R && c < C) tile[i][threadIdx.x] = src[static_cast<size_t>(r) * C + c];
        }
        __syncthreads();
        for (int i = threadIdx.y; i < 32; i += 8) {
            const int c = c0 + i, r = r0 + threadIdx.x;
            if (r < R && c < C) dst[static_cast<size_t>(c) * R + r] = tile[threadIdx.x][i];
        }
        __syncthreads();
    }
}

__global__ void shift_decay_kernel(const float* __restrict__ lg, int kind, float* __restrict__ out, int H, int T,
                                   long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long bh = i / T;
        const int t = static_cast<int>(i - bh * T);
        float x = 0.f;
        if (t + 1 < T) x = kind == LA_DECAY_PER_STEP ? lg[i + 1] : lg[bh % H];
        out[i] = x;
    }
}

__global__ void scale_first_kernel(float* __restrict__ s, const float* __restrict__ lg, int kind, int H, int T,
                                   int n, long long total) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long bh = i / n;
        const float l = kind == LA_DECAY_PER_STEP ? lg[bh * T] : lg[bh % H];
        s[i] *= expf(l);
    }
}

template <typename E>
__device__ __forceinline__ float to_f(E x) {
    return static_cast<float>(x);
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

// <dSf, S_T> per (b, h), with S_T given transposed; one block per (b, h).
__global__ void terminal_kernel(const float* __restrict__ dsf, const float* __restrict__ st_t, double* __restrict__ out,
                                int Dk, int Dv) {
    const int bh = blockIdx.x;
    const size_t base = static_cast<size_t>(bh) * Dk * Dv;
    double acc = 0.0;
    for (int e = threadIdx.x; e < Dk * Dv; e += blockDim.x) {
        const int i = e / Dv, j = e % Dv;
        acc += static_cast<double>(dsf[base + e]) * st_t[base + static_cast<size_t>(j) * Dk + i];
    }
    __shared__ double red[256];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int o = blockDim.x / 2; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[bh] = red[0];
}

// Block (blk, bh): a_t = q_t . dq_t - k_t . dk_t for its kDlogTokens tokens
// (one warp per token at a time, fp32), the suffix sums of a inside the
// block, written to x (per step) or summed (per head); the block's total of
// a and of its local suffix sums go to the scratch for the second pass.
template <typename E>
__global__ void __launch_bounds__(256) dlog_block_kernel(const E* __restrict__ q, const E* __restrict__ k,
                                                         const E* __restrict__ dq, const E* __restrict__ dk,
                                                         float* __restrict__ x, int per_step, int T, int Dk,
                                                         int nblk, double* __restrict__ blk_a,
                                                         double* __restrict__ blk_x) {
    __shared__ float a[kDlogTokens];
    __shared__ float wsum[8];
    const int blk = blockIdx.x, bh = blockIdx.y;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int t0 = blk * kDlogTokens;
    const int n = min(kDlogTokens, T - t0);
    for (int i = warp; i < kDlogTokens; i += 8) {
        float s = 0.f;
        if (i < n) {
            const size_t row = (static_cast<size_t>(bh) * T + t0 + i) * Dk;
            for (int e = lane; e < Dk; e += 32)
                s += to_f(q[row + e]) * to_f(dq[row + e]) - to_f(k[row + e]) * to_f(dk[row + e]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        }
        if (lane == 0) a[i] = s;
    }
    __syncthreads();
    // suffix sums: thread i holds token i; warp-level inclusive suffix scan,
    // then the totals of the later warps
    const int i = threadIdx.x;
    float v = a[i];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, v, o);
        if (lane + o < 32) v += y;
    }
    if (lane == 0) wsum[warp] = v;  // lane 0 holds its warp's total
    __syncthreads();
    for (int w = warp + 1; w < 8; ++w) v += wsum[w];
    if (per_step && i < n) x[static_cast<size_t>(bh) * T + t0 + i] = v;
    // block totals (double): a over the block, and the local suffix sums
    __shared__ double red[256];
    red[i] = i < n ? static_cast<double>(v) : 0.0;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (i < o) red[i] += red[i + o];
        __syncthreads();
    }
    if (i == 0) {
        blk_x[static_cast<size_t>(bh) * nblk + blk] = red[0];
        double ta = 0.0;
        for (int w = 0; w < 8; ++w) ta += wsum[w];
        blk_a[static_cast<size_t>(bh) * nblk + blk] = ta;
    }
}

// Block (blk, bh): the offset of block blk is the terminal term plus the
// totals of a over every later block; per step it is added to the block's
// tokens, per head the block's contribution (its local sums plus n times the
// offset) goes to blk_x for the final reduction.
__global__ void dlog_offset_kernel(float* __restrict__ x, int per_step, int T, int nblk,
                                   const double* __restrict__ blk_a, double* __restrict__ blk_x,
                                   const double* __restrict__ terminal) {
    const int blk = blockIdx.x, bh = blockIdx.y;
    __shared__ double off;
    if (threadIdx.x == 0) {
        double o = terminal ? terminal[bh] : 0.0;
        for (int j = nblk - 1; j > blk; --j) o += blk_a[static_cast<size_t>(bh) * nblk + j];
        off = o;
    }
    __syncthreads();
    const int t0 = blk * kDlogTokens, n = min(kDlogTokens, T - t0);
    if (per_step) {
        if (threadIdx.x < n) {
            float* p = x + static_cast<size_t>(bh) * T + t0 + threadIdx.x;
            *p = static_cast<float>(static_cast<double>(*p) + off);
        }
    } else if (threadIdx.x == 0) {
        blk_x[static_cast<size_t>(bh) * nblk + blk] += n * off;
    }
}

// Per head: the sum over b and blocks, in a fixed order (deterministic).
__global__ void dlog_head_kernel(float* __restrict__ out, int B, int H, int nblk, const double* __restrict__ blk_x) {
    const int h = blockIdx.x;
    __shared__ double red[256];
    double acc = 0.0;
    for (int e = threadIdx.x; e < B * nblk; e += blockDim.x) {
        const int b = e / nblk, j = e % nblk;
        acc += blk_x[static_cast<size_t>(b * H + h) * nblk + j];
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[h] = static_cast<float>(red[0]);
}

}  // namespace

cudaError_t launch_transpose(const float* in, float* out, int BH, int R, int C, cudaStream_t stream) {
    const dim3 grid((C + 31) / 32, (R + 31) / 32, std::min(BH, 65535));
    transpose_kernel<<<grid, dim3(32, 8), 0, stream>>>(in, out, BH, R, C);
    return cudaGetLastError();
}

cudaError_t launch_shift_decay(const float* log_g, int kind, float* out, int B, int H, int T, cudaStream_t stream) {
    const long long n = static_cast<long long>(B) * H * T;
    shift_decay_kernel<<<grid_for(n, 256), 256, 0, stream>>>(log_g, kind, out, H, T, n);
    return cudaGetLastError();
}

cudaError_t launch_scale_by_first_decay(float* s, const float* log_g, int kind, int B, int H, int T, int n,
                                        cudaStream_t stream) {
    const long long total = static_cast<long long>(B) * H * n;
    scale_first_kernel<<<grid_for(total, 256), 256, 0, stream>>>(s, log_g, kind, H, T, n, total);
    return cudaGetLastError();
}

size_t dlog_scratch_doubles(int B, int H, int T) {
    const size_t BH = static_cast<size_t>(B) * H;
    const size_t nblk = (static_cast<size_t>(T) + kDlogTokens - 1) / kDlogTokens;
    return BH + 2 * BH * nblk;  // terminal terms, block totals of a, block sums of x
}

cudaError_t launch_dlog(const DlogArgs& a) {
    const int BH = a.B * a.H;
    const int nblk = (a.T + kDlogTokens - 1) / kDlogTokens;
    if (nblk > 65535 || BH > 65535) return cudaErrorInvalidValue;
    double* terminal = a.d_final_state ? a.scratch : nullptr;
    double* blk_a = a.scratch + BH;
    double* blk_x = blk_a + static_cast<size_t>(BH) * nblk;
    if (terminal) {
        terminal_kernel<<<BH, 256, 0, a.stream>>>(a.d_final_state, a.final_state_t, terminal, a.Dk, a.Dv);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int per_step = a.kind == LA_DECAY_PER_STEP;
    const dim3 grid(nblk, BH);
    if (a.dtype == LA_BF16)
        dlog_block_kernel<__nv_bfloat16><<<grid, 256, 0, a.stream>>>(
            static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
            static_cast<const __nv_bfloat16*>(a.dq), static_cast<const __nv_bfloat16*>(a.dk), a.d_log_g, per_step,
            a.T, a.Dk, nblk, blk_a, blk_x);
    else
        dlog_block_kernel<float><<<grid, 256, 0, a.stream>>>(
            static_cast<const float*>(a.q), static_cast<const float*>(a.k), static_cast<const float*>(a.dq),
            static_cast<const float*>(a.dk), a.d_log_g, per_step, a.T, a.Dk, nblk, blk_a, blk_x);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dlog_offset_kernel<<<grid, kDlogTokens, 0, a.stream>>>(a.d_log_g, per_step, a.T, nblk, blk_a, blk_x, terminal);
    e = cudaGetLastError();
    if (e != cudaSuccess || per_step) return e;
    dlog_head_kernel<<<a.H, 256, 0, a.stream>>>(a.d_log_g, a.B, a.H, nblk, blk_x);
    return cudaGetLastError();
}

}  // namespace la
