// la_wkv4.cu - the RWKV-4 WKV recurrence (BlinkDL/RWKV-LM issue 167, the
// att_seq time loop), one thread per channel.
//
// Per batch b and channel c, with time decay w (log of the per-step factor)
// and bonus u, the output is the decayed average
//     wkv_t = (sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u + k_t} v_t)
//           / (sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u + k_t})
// carried as (aa, bb) against a running log scale pp, exactly as the page's
// loop does: a read-out that takes max(pp, u + k_t) as its scale, then an
// update that takes max(w + pp, k_t); only differences <= 0 are
// exponentiated, so no key can overflow.  The kernel runs the loop in fp32
// in log2 units (every log value times log2 e, exponentials by ex2).
//
// Data movement: a CTA owns one batch row and kCW consecutive channels.  One
// producer thread streams [kTT tokens x kCW channels] tiles of k and v into
// a ring of kStages shared-memory stages with TMA (about 96 KB in flight per
// CTA, two CTAs per SM), so the HBM latency is hidden behind the sequential
// per-token work; each consumer thread reads its channel's column of the
// tile and writes its output directly (a warp writes 32 consecutive values).
// Every barrier wait gives up after kWaitLimitNs, sets the device error word
// and unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

constexpr int kCW = 64;                 // channels per CTA (one per consumer thread)
constexpr int kStages = 6;
constexpr int kConsumerWarps = kCW / 32;
constexpr int kThreads = 32 * (kConsumerWarps + 1);  // + one producer warp
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kEmptyScale = -1e38f;   // pp of an empty state (aa = bb = 0)

template <typename E>
struct Tile {
    static constexpr int TT = sizeof(E) == 2 ? 64 : 32;           // tokens per stage
    static constexpr int BYTES = TT * kCW * static_cast<int>(sizeof(E));  // one array's tile
    static constexpr int STAGE = 2 * BYTES;                        // k tile, then v tile
    static constexpr int SMEM = kStages * STAGE + 256;             // + barriers
};

// Weights of two terms with log2 weights a and b against the larger one:
// one of them is 1, the other 2^-|a - b| (one exponential per pair).
__device__ __forceinline__ void shifted_pair(float a, float b, float& fa, float& fb) {
    const float d = a - b;
    const float t = ex2_approx(-fabsf(d));
    fa = d >= 0.f ? 1.f : t;
    fb = d >= 0.f ? t : 1.f;
}

__device__ __forceinline__ float load_f(const float* p) { return *p; }
__device__ __forceinline__ float load_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void store_e(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_e(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename E>
__global__ void __launch_bounds__(kThreads) wkv4_kernel(const __grid_constant__ CUtensorMap tmk,
                                                        const __grid_constant__ CUtensorMap tmv,
                                                        const float* __restrict__ w, const float* __restrict__ u,
                                                        const float* init_state, E* __restrict__ out,
                                                        float* final_state, int T, int C, int* err) {
    using G = Tile<E>;
    // used as declared (not realigned through an integer), so that the
    // compiler keeps the shared address space and reads tiles with LDS;
    // TMA without swizzle needs 16-byte alignment only
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kStages * G::STAGE);
    uint64_t* empty = full + kStages;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + kStages);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int b = blockIdx.y, c0 = blockIdx.x * kCW;
    const int ntiles = (T + G::TT - 1) / G::TT;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // producer: one thread issues the tile loads in order
        if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < ntiles; ++j) {
                const int s = j % kStages;
                if (j >= kStages && !mbar_wait_bounded(&empty[s], ((j / kStages) - 1) & 1, kWaitLimitNs)) {
                    *abort = 1;
                    if (err) atomicCAS(err, 0, kErrTmaWait);
                    break;
                }
                if (*abort) break;
                uint8_t* st = sm + s * G::STAGE;
                mbar_arrive_expect_tx(&full[s], G::STAGE);
                tma_load_3d(st, &tmk, &full[s], c0, j * G::TT, b);
                tma_load_3d(st + G::BYTES, &tmv, &full[s], c0, j * G::TT, b);
                ++issued;
            }
            // copies in flight land before the CTA's shared memory goes away
            for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
                mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, kWaitLimitNs);
        }
        return;
    }

    // consumer: thread = channel
    const int c = c0 + threadIdx.x;
    const bool live = c < C;
    const float W = live ? w[c] * kLog2e : 0.f;
    const float U = live ? u[c] * kLog2e : 0.f;
    float aa = 0.f, bb = 0.f, P = kEmptyScale * kLog2e;
    if (live && init_state) {
        const float* s0 = init_state + static_cast<size_t>(b) * 3 * C + c;
        aa = s0[0];
        bb = s0[C];
        P = s0[2 * C] * kLog2e;
    }
    E* o = out + static_cast<size_t>(b) * T * C + c;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j % kStages;
        // whole-warp bounded wait on the tile
        bool got = mbar_try_wait(&full[s], (j / kStages) & 1);
        if (!__all_sync(0xffffffffu, got)) {
            const uint64_t t0 = global_timer_ns();
            while (true) {
                if (!got) got = mbar_try_wait_sleep(&full[s], (j / kStages) & 1, 20000);
                if (__all_sync(0xffffffffu, got)) break;
                bool give_up = *abort != 0 || global_timer_ns() - t0 > kWaitLimitNs;
                if (__any_sync(0xffffffffu, give_up)) {
                    if (lane == 0) {
                        *abort = 1;
                        if (err) atomicCAS(err, 0, kErrTmaWait);
                    }
                    ok = false;
                    break;
                }
            }
            if (!ok) break;
        }
        const E* tk = reinterpret_cast<const E*>(sm + s * G::STAGE) + threadIdx.x;
        const E* tv = reinterpret_cast<const E*>(sm + s * G::STAGE + G::BYTES) + threadIdx.x;
        const int n = min(G::TT, T - j * G::TT);
        // one token: read-out (the state at log weight P, this token at
        // U + K), then update (the state decayed to W + P, this token at K)
        auto step = [&](float K, float v) -> float {
            float e1, e2;
            shifted_pair(P, U + K, e1, e2);
            const float y = __fdividef(fmaf(e1, aa, e2 * v), fmaf(e1, bb, e2));
            const float d = W + P;
            float f1, f2;
            shifted_pair(d, K, f1, f2);
            aa = fmaf(f1, aa, f2 * v);
            bb = fmaf(f1, bb, f2);
            P = fmaxf(d, K);
            return y;
        };
        if (live) {
            // batches of 8 tokens: the next batch's tile reads are issued
            // before this batch's dependent steps, the outputs stored after
            // them, so that memory latency stays off the recurrence's path
            const int nb = n / 8;
            float kk[8], vv[8];
            if (nb > 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kk[e] = load_f(tk + e * kCW);
                    vv[e] = load_f(tv + e * kCW);
                }
            }
            for (int bi = 0; bi < nb; ++bi) {
                float kn[8], vn[8], yy[8];
                const int nxt = bi + 1 < nb ? (bi + 1) * 8 : bi * 8;  // (a harmless re-read at the end)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kn[e] = load_f(tk + (nxt + e) * kCW);
                    vn[e] = load_f(tv + (nxt + e) * kCW);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) yy[e] = step(kk[e] * kLog2e, vv[e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) store_e(o + static_cast<size_t>(e) * C, yy[e]);
                o += static_cast<size_t>(8) * C;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kk[e] = kn[e];
                    vv[e] = vn[e];
                }
            }
            for (int i = nb * 8; i < n; ++i) {
                store_e(o, step(load_f(tk + i * kCW) * kLog2e, load_f(tv + i * kCW)));
                o += C;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ok && live && final_state) {
        float* s1 = final_state + static_cast<size_t>(b) * 3 * C + c;
        s1[0] = aa;
        s1[C] = bb;
        s1[2 * C] = P * (1.f / kLog2e);
    }
}

// [B, T, C] tensor, boxes of [1, TT tokens, kCW channels], no swizzle.
bool make_wkv_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int es, int B, int T, int C, int TT) {
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(C) * es, static_cast<cuuint64_t>(C) * es * T};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kCW), static_cast<cuuint32_t>(TT), 1};
    const cuuint32_t elem[3] = {1, 1, 1};
    return f(map, dt, 3, const_cast<void*>(base), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename E>
cudaError_t launch_typed(const Wkv4Args& a, CUtensorMapDataType dt) {
    using G = Tile<E>;
    CUtensorMap tmk, tmv;
    if (!make_wkv_map(&tmk, a.k, dt, sizeof(E), a.B, a.T, a.C, G::TT) ||
        !make_wkv_map(&tmv, a.v, dt, sizeof(E), a.B, a.T, a.C, G::TT))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(wkv4_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    const dim3 grid((a.C + kCW - 1) / kCW, a.B);
    wkv4_kernel<E><<<grid, kThreads, G::SMEM, a.stream>>>(tmk, tmv, a.w, a.u, a.init_state, static_cast<E*>(a.out),
                                                          a.final_state, a.T, a.C, a.err_word);
    return cudaGetLastError();
}

// No tokens: the final state is the initial one (or the empty state).
__global__ void wkv4_pass_state_kernel(const float* init_state, float* final_state, int C, long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int plane = static_cast<int>((i / C) % 3);
        final_state[i] = init_state ? init_state[i] : (plane == 2 ? kEmptyScale : 0.f);
    }
}

}  // namespace

cudaError_t launch_wkv4(const Wkv4Args& a) {
    if (a.T == 0) {
        if (!a.final_state || a.final_state == a.init_state) return cudaSuccess;
        const long long n = 3LL * a.B * a.C;
        const int grid = static_cast<int>(n / 256 + 1 < 148 * 8 ? n / 256 + 1 : 148 * 8);
        wkv4_pass_state_kernel<<<grid, 256, 0, a.stream>>>(a.init_state, a.final_state, a.C, n);
        return cudaGetLastError();
    }
    return a.dtype == LA_BF16 ? launch_typed<__nv_bfloat16>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)
                              : launch_typed<float>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

}  // namespace la
