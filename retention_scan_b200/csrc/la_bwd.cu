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

// <dSf, S_T> (+ <dzf, z_T>) per (b, h); S_T[i][j] at st[bh * st_bh + i * st_i
// + j * st_j], z_T[i] at zt[bh * zt_bh + i * zt_i]; one block per (b, h).
__global__ void terminal_kernel(const float* __restrict__ dsf, const float* __restrict__ st, long long st_bh,
                                int st_i, int st_j, const float* __restrict__ dzf, const float* __restrict__ zt,
                                long long zt_bh, int zt_i, double* __restrict__ out, int Dk, int Dv) {
    const int bh = blockIdx.x;
    const size_t base = static_cast<size_t>(bh) * Dk * Dv;
    double acc = 0.0;
    if (dsf)
        for (int e = threadIdx.x; e < Dk * Dv; e += blockDim.x) {
            const int i = e / Dv, j = e % Dv;
            acc += static_cast<double>(dsf[base + e]) *
                   st[bh * st_bh + static_cast<long long>(i) * st_i + static_cast<long long>(j) * st_j];
        }
    if (dzf)
        for (int i = threadIdx.x; i < Dk; i += blockDim.x)
            acc += static_cast<double>(dzf[static_cast<size_t>(bh) * Dk + i]) *
                   zt[bh * zt_bh + static_cast<long long>(i) * zt_i];
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
    constexpr int VEC = 16 / sizeof(E);  // elements per 16-byte load
    const int lpt = Dk / VEC;            // lanes per token with 16-byte loads
    if (Dk % VEC == 0 && lpt <= 32 && (lpt & (lpt - 1)) == 0) {
        // groups of lpt lanes each take one token (a row of 16-byte loads),
        // 32 / lpt tokens per warp at a time
        const int tpw = 32 / lpt, sub = lane / lpt, l = lane % lpt;
        for (int i0 = warp * tpw; i0 < kDlogTokens; i0 += 8 * tpw) {
            const int i = i0 + sub;
            float s = 0.f;
            if (i < n) {
                const size_t row = (static_cast<size_t>(bh) * T + t0 + i) * Dk + static_cast<size_t>(l) * VEC;
                const uint4 vq = *reinterpret_cast<const uint4*>(q + row);
                const uint4 vdq = *reinterpret_cast<const uint4*>(dq + row);
                const uint4 vk = *reinterpret_cast<const uint4*>(k + row);
                const uint4 vdk = *reinterpret_cast<const uint4*>(dk + row);
                const E* eq = reinterpret_cast<const E*>(&vq);
                const E* edq = reinterpret_cast<const E*>(&vdq);
                const E* ek = reinterpret_cast<const E*>(&vk);
                const E* edk = reinterpret_cast<const E*>(&vdk);
#pragma unroll
                for (int e = 0; e < VEC; ++e) s += to_f(eq[e]) * to_f(edq[e]) - to_f(ek[e]) * to_f(edk[e]);
            }
            for (int o = lpt / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (l == 0 && i < kDlogTokens) a[i] = s;
        }
    } else {
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

// Per (b, h): blk_off[j] = the totals of a over the blocks after j, in
// chunks of 256 blocks from the end (a fixed summation order).
__global__ void dlog_suffix_kernel(const double* __restrict__ blk_a, double* __restrict__ blk_off, int nblk) {
    const int bh = blockIdx.x;
    __shared__ double sh[256];
    double carry = 0.0;  // totals of the blocks after the current chunk
    for (int c1 = nblk; c1 > 0; c1 -= 256) {
        const int c0 = c1 > 256 ? c1 - 256 : 0, m = c1 - c0;
        const int j = c0 + threadIdx.x;
        sh[threadIdx.x] = threadIdx.x < m ? blk_a[static_cast<size_t>(bh) * nblk + j] : 0.0;
        __syncthreads();
        double acc = carry;
        for (int jj = threadIdx.x + 1; jj < m; ++jj) acc += sh[jj];
        if (threadIdx.x < m) blk_off[static_cast<size_t>(bh) * nblk + j] = acc;
        double tot = 0.0;
        for (int jj = 0; jj < m; ++jj) tot += sh[jj];
        carry += tot;
        __syncthreads();
    }
}

// Block (blk, bh): the offset of block blk is the terminal term plus the
// totals of a over every later block; per step it is added to the block's
// tokens, per head the block's contribution (its local sums plus n times the
// offset) goes to blk_x for the final reduction.
__global__ void dlog_offset_kernel(float* __restrict__ x, int per_step, int T, int nblk,
                                   const double* __restrict__ blk_off, double* __restrict__ blk_x,
                                   const double* __restrict__ terminal) {
    const int blk = blockIdx.x, bh = blockIdx.y;
    const double off = (terminal ? terminal[bh] : 0.0) + blk_off[static_cast<size_t>(bh) * nblk + blk];
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

// [n][16] panel with column 0 = 1 and the rest 0 (the value panel whose scan
// gives the key sum: S = sum k 1^T, so q^T S = q . z in column 0).
template <typename E>
__global__ void ones_panel_kernel(E* __restrict__ out, long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n * 16;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        out[i] = static_cast<E>((i & 15) == 0 ? 1.f : 0.f);
}

// Per (b, h): the Dk vector x into column 0 of a [Dk][16] panel (rows) or
// row 0 of a [16][Dk] panel (cols), zeros elsewhere, fp32.
__global__ void vec_panel_kernel(const float* __restrict__ x, float* __restrict__ out, int Dk, int rows,
                                 long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long bh = i / (16LL * Dk);
        const int e = static_cast<int>(i - bh * 16LL * Dk);
        float val = 0.f;
        if (x) {
            if (rows && (e & 15) == 0) val = x[bh * Dk + e / 16];
            if (!rows && e < Dk) val = x[bh * Dk + e];
        }
        out[i] = val;
    }
}

// Normalised output y = n / den: per token, dn = dy / den and
// dden = -(dy . y) / den = -(dy . n) / den^2 (the latter as column 0 of a
// 16-wide panel); from y, whose rounding is one of the ratio, a rounding of
// den scales dn and dden alike.  One warp per token.
template <typename E>
__global__ void norm_grad_kernel(const E* __restrict__ dy, const E* __restrict__ y,
                                 const E* __restrict__ den_panel, E* __restrict__ dn, E* __restrict__ dden_panel,
                                 int Dv, long long ntok) {
    const int lane = threadIdx.x % 32;
    const long long w0 = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) / 32;
    const long long nw = static_cast<long long>(gridDim.x) * blockDim.x / 32;
    for (long long t = w0; t < ntok; t += nw) {
        const float den = to_f(den_panel[t * 16]);
        const float inv = 1.f / den;
        const size_t row = static_cast<size_t>(t) * Dv;
        float dot = 0.f;
        for (int c = lane; c < Dv; c += 32) {
            const float g = to_f(dy[row + c]);
            dot = fmaf(g, to_f(y[row + c]), dot);
            dn[row + c] = static_cast<E>(g * inv);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (lane < 16) dden_panel[t * 16 + lane] = static_cast<E>(lane == 0 ? -dot * inv : 0.f);
    }
}

// PK[t] = [v_t | 1 | 0 ...], W wide (W > Dv).
template <typename E>
__global__ void pack_value_panel_kernel(const E* __restrict__ v, E* __restrict__ pk, int Dv, int W, long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n * W;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long t = i / W;
        const int c = static_cast<int>(i - t * W);
        pk[i] = c < Dv ? v[t * Dv + c] : static_cast<E>(c == Dv ? 1.f : 0.f);
    }
}

// [S | z | 0] as [Dk][W] fp32 per (b, h) (S [Dk][Dv], z [Dk]; null: zeros).
__global__ void pack_state_panel_kernel(const float* __restrict__ S, const float* __restrict__ z,
                                        float* __restrict__ out, int Dk, int Dv, int W, long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long bhi = i / W;  // bh * Dk + row
        const int c = static_cast<int>(i - bhi * W);
        float x = 0.f;
        if (c < Dv && S) x = S[bhi * Dv + c];
        if (c == Dv && z) x = z[bhi];
        out[i] = x;
    }
}

// From [n | den | ..] (W wide): PQ[t] = [dn_t | dden_t | 0 ...] (W wide) and
// dn [t] (Dv wide); dn = dy / den, dden = -(dy . n) / den^2.  One warp per token.
template <typename E>
__global__ void norm_grad_panel_kernel(const E* __restrict__ dy, const E* __restrict__ nd, E* __restrict__ pq,
                                       E* __restrict__ dn, int Dv, int W, long long ntok) {
    const int lane = threadIdx.x % 32;
    const long long w0 = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) / 32;
    const long long nw = static_cast<long long>(gridDim.x) * blockDim.x / 32;
    for (long long t = w0; t < ntok; t += nw) {
        const size_t rw = static_cast<size_t>(t) * W, rv = static_cast<size_t>(t) * Dv;
        const float inv = 1.f / to_f(nd[rw + Dv]);
        float dot = 0.f;
        for (int c = lane; c < Dv; c += 32) {
            const float g = to_f(dy[rv + c]);
            dot = fmaf(g, to_f(nd[rw + c]), dot);
            const E x = static_cast<E>(g * inv);
            dn[rv + c] = x;
            pq[rw + c] = x;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        for (int c = Dv + lane; c < W; c += 32) pq[rw + c] = static_cast<E>(c == Dv ? -dot * inv * inv : 0.f);
    }
}

// out[bh][i] = g_1 * panel[bh * rows * Dk + row * Dk + i] (one row of a
// [rows][Dk] state panel), g_1 the decay of the sequence's first token (1
// without a decay).
__global__ void panel_row_scaled_kernel(const float* __restrict__ panel, float* __restrict__ out,
                                        const float* __restrict__ lg, int kind, int H, int T, int Dk, int rows,
                                        int row, long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long bh = i / Dk;
        const int e = static_cast<int>(i - bh * Dk);
        float g = 1.f;
        if (kind == LA_DECAY_PER_STEP) g = expf(lg[bh * T]);
        if (kind == LA_DECAY_PER_HEAD) g = expf(lg[bh % H]);
        out[i] = g * panel[(bh * rows + row) * static_cast<long long>(Dk) + e];
    }
}

}  // namespace

cudaError_t launch_ones_panel(void* out, long long n, la_dtype dtype, cudaStream_t stream) {
    if (dtype == LA_BF16)
        ones_panel_kernel<__nv_bfloat16><<<grid_for(n * 16, 256), 256, 0, stream>>>(static_cast<__nv_bfloat16*>(out), n);
    else
        ones_panel_kernel<float><<<grid_for(n * 16, 256), 256, 0, stream>>>(static_cast<float*>(out), n);
    return cudaGetLastError();
}

cudaError_t launch_vec_panel(const float* x, float* out, int BH, int Dk, bool rows, cudaStream_t stream) {
    const long long n = 16LL * BH * Dk;
    vec_panel_kernel<<<grid_for(n, 256), 256, 0, stream>>>(x, out, Dk, rows ? 1 : 0, n);
    return cudaGetLastError();
}

cudaError_t launch_norm_grad(const void* dy, const void* y, const void* den_panel, void* dn, void* dden_panel,
                             int Dv, long long ntok, la_dtype dtype, cudaStream_t stream) {
    const int grid = grid_for(ntok * 32, 256);
    if (dtype == LA_BF16)
        norm_grad_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(dy), static_cast<const __nv_bfloat16*>(y),
            static_cast<const __nv_bfloat16*>(den_panel), static_cast<__nv_bfloat16*>(dn),
            static_cast<__nv_bfloat16*>(dden_panel), Dv, ntok);
    else
        norm_grad_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(dy), static_cast<const float*>(y),
                                                         static_cast<const float*>(den_panel), static_cast<float*>(dn),
                                                         static_cast<float*>(dden_panel), Dv, ntok);
    return cudaGetLastError();
}

cudaError_t launch_pack_value_panel(const void* v, void* pk, int Dv, int W, long long ntok, la_dtype dtype,
                                   cudaStream_t stream) {
    const int grid = grid_for(ntok * W, 256);
    if (dtype == LA_BF16)
        pack_value_panel_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(v),
                                                                         static_cast<__nv_bfloat16*>(pk), Dv, W, ntok);
    else
        pack_value_panel_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(v), static_cast<float*>(pk),
                                                                 Dv, W, ntok);
    return cudaGetLastError();
}

cudaError_t launch_pack_state_panel(const float* S, const float* z, float* out, int BH, int Dk, int Dv, int W,
                                    cudaStream_t stream) {
    const long long n = static_cast<long long>(BH) * Dk * W;
    pack_state_panel_kernel<<<grid_for(n, 256), 256, 0, stream>>>(S, z, out, Dk, Dv, W, n);
    return cudaGetLastError();
}

cudaError_t launch_norm_grad_panel(const void* dy, const void* nd, void* pq, void* dn, int Dv, int W, long long ntok,
                                   la_dtype dtype, cudaStream_t stream) {
    const int grid = grid_for(ntok * 32, 256);
    if (dtype == LA_BF16)
        norm_grad_panel_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(dy), static_cast<const __nv_bfloat16*>(nd),
            static_cast<__nv_bfloat16*>(pq), static_cast<__nv_bfloat16*>(dn), Dv, W, ntok);
    else
        norm_grad_panel_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(dy),
                                                               static_cast<const float*>(nd), static_cast<float*>(pq),
                                                               static_cast<float*>(dn), Dv, W, ntok);
    return cudaGetLastError();
}

cudaError_t launch_panel_row_scaled(const float* panel, float* out, const float* log_g, int kind, int B, int H,
                                    int T, int Dk, int rows, int row, cudaStream_t stream) {
    const long long n = static_cast<long long>(B) * H * Dk;
    panel_row_scaled_kernel<<<grid_for(n, 256), 256, 0, stream>>>(panel, out, log_g, kind, H, T, Dk, rows, row, n);
    return cudaGetLastError();
}

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
    return BH + 3 * BH * nblk;  // terminal terms, block totals of a, block sums of x, block offsets
}

cudaError_t launch_dlog(const DlogArgs& a) {
    const int BH = a.B * a.H;
    const int nblk = (a.T + kDlogTokens - 1) / kDlogTokens;
    if (nblk > 65535 || BH > 65535) return cudaErrorInvalidValue;
    double* terminal = (a.d_final_state || a.d_final_z) ? a.scratch : nullptr;
    double* blk_a = a.scratch + BH;
    double* blk_x = blk_a + static_cast<size_t>(BH) * nblk;
    double* blk_off = blk_x + static_cast<size_t>(BH) * nblk;
    if (terminal) {
        terminal_kernel<<<BH, 256, 0, a.stream>>>(a.d_final_state, a.st, a.st_bh, a.st_i, a.st_j, a.d_final_z, a.zt,
                                                  a.zt_bh, a.zt_i, terminal, a.Dk, a.Dv);
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
    dlog_suffix_kernel<<<BH, 256, 0, a.stream>>>(blk_a, blk_off, nblk);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dlog_offset_kernel<<<grid, kDlogTokens, 0, a.stream>>>(a.d_log_g, per_step, a.T, nblk, blk_off, blk_x, terminal);
    e = cudaGetLastError();
    if (e != cudaSuccess || per_step) return e;
    dlog_head_kernel<<<a.H, 256, 0, a.stream>>>(a.d_log_g, a.B, a.H, nblk, blk_x);
    return cudaGetLastError();
}

}  // namespace la
