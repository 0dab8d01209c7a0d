// la_ema.cu - the cumulative exponential moving average of RetNet issue 21
// ("Proposed improvement/collaboration: removing the O(T^2) training
// cost", the cumulative_ema function): element-wise values x and factors f
// of one shape, scanned along T per channel,
//     s <- f_t s + x_t,   out_t = s,
// or, with the reverse flag, the same recurrence from the last step back to
// the first.  A carried state enters before the first scanned step.
//
// One CTA per (batch row, 64 channels): a producer thread streams
// [TT tokens x 64 channels] tiles of x and f into a ring of shared-memory
// stages with TMA (in scan order: from the last tile for the reverse scan),
// and each consumer thread runs the recurrences of two adjacent channels in
// fp32 (one 4- or 8-byte shared-memory load per array and step, one packed
// store, two independent FMA chains), eight tokens ahead of the dependent
// steps.  The direction is a template argument.
// Every barrier wait gives up after kWaitLimitNs, sets the device error word
// and unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

constexpr int kCW = 64;
constexpr int kStages = 4;
constexpr int kConsumerWarps = kCW / 64;  // two channels per thread
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr uint64_t kWaitLimitNs = 1000000000ull;

template <typename E>
struct EmaTile {
    static constexpr int TT = sizeof(E) == 2 ? 64 : 32;
    static constexpr int BYTES = TT * kCW * static_cast<int>(sizeof(E));
    static constexpr int STAGE = 2 * BYTES;  // x tile, then f tile
    static constexpr int SMEM = kStages * STAGE + 256;
};

// two adjacent channels
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ void store2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void store2(__nv_bfloat16* p, float2 v) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}

template <typename E, bool REV>
__global__ void __launch_bounds__(kThreads) ema_kernel(const __grid_constant__ CUtensorMap tmx,
                                                       const __grid_constant__ CUtensorMap tmf,
                                                       const float* init_state, E* __restrict__ out,
                                                       float* final_state, int T, int C, int* err) {
    using G = EmaTile<E>;
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kStages * G::STAGE);
    uint64_t* empty = full + kStages;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + kStages);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int b = blockIdx.y, c0 = blockIdx.x * kCW;
    const int ntiles = (T + G::TT - 1) / G::TT;
    auto tile_of = [&](int j) { return REV ? ntiles - 1 - j : j; };  // memory tile of the j-th scanned tile

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmx);
        prefetch_tensormap(&tmf);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
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
                tma_load_3d(st, &tmx, &full[s], c0, tile_of(j) * G::TT, b);
                tma_load_3d(st + G::BYTES, &tmf, &full[s], c0, tile_of(j) * G::TT, b);
                ++issued;
            }
            for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
                mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, kWaitLimitNs);
        }
        return;
    }

    const int c = c0 + 2 * threadIdx.x;  // channels c, c + 1 (C is even)
    const bool live = c < C;
    float2 sv = make_float2(0.f, 0.f);
    if (live && init_state) sv = make_float2(init_state[static_cast<size_t>(b) * C + c],
                                             init_state[static_cast<size_t>(b) * C + c + 1]);
    E* ob = out + static_cast<size_t>(b) * T * C + c;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j % kStages;
        bool got = mbar_try_wait(&full[s], (j / kStages) & 1);
        if (!__all_sync(0xffffffffu, got)) {
            const uint64_t tw = global_timer_ns();
            while (true) {
                if (!got) got = mbar_try_wait_sleep(&full[s], (j / kStages) & 1, 20000);
                if (__all_sync(0xffffffffu, got)) break;
                const bool give_up = *abort != 0 || global_timer_ns() - tw > kWaitLimitNs;
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
        const E* tx = reinterpret_cast<const E*>(sm + s * G::STAGE) + 2 * threadIdx.x;
        const E* tf = reinterpret_cast<const E*>(sm + s * G::STAGE + G::BYTES) + 2 * threadIdx.x;
        const int t0 = tile_of(j) * G::TT;
        const int n = min(G::TT, T - t0);
        if (live) {
            // rows in scan order: forward from row 0, reverse from row n - 1
            const E* px = tx + (REV ? (n - 1) * kCW : 0);
            const E* pf = tf + (REV ? (n - 1) * kCW : 0);
            E* po = ob + static_cast<size_t>(t0 + (REV ? n - 1 : 0)) * C;
            constexpr int dr = REV ? -kCW : kCW;
            const long long dout = REV ? -static_cast<long long>(C) : static_cast<long long>(C);
            const int nb = n / 8;
            float2 xx[8], ff[8];
            if (nb > 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    xx[e] = load2(px + e * dr);
                    ff[e] = load2(pf + e * dr);
                }
            }
            for (int bi = 0; bi < nb; ++bi) {
                float2 xn[8], fn[8], yy[8];
                const int nxt = bi + 1 < nb ? 8 : 0;  // (a harmless re-read at the end)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    xn[e] = load2(px + (nxt + e) * dr);
                    fn[e] = load2(pf + (nxt + e) * dr);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sv.x = fmaf(ff[e].x, sv.x, xx[e].x);
                    sv.y = fmaf(ff[e].y, sv.y, xx[e].y);
                    yy[e] = sv;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) store2(po + e * dout, yy[e]);
                po += 8 * dout;
                px += 8 * dr;
                pf += 8 * dr;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    xx[e] = xn[e];
                    ff[e] = fn[e];
                }
            }
            for (int i = nb * 8; i < n; ++i) {
                const float2 x2 = load2(px), f2 = load2(pf);
                sv.x = fmaf(f2.x, sv.x, x2.x);
                sv.y = fmaf(f2.y, sv.y, x2.y);
                store2(po, sv);
                po += dout;
                px += dr;
                pf += dr;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ok && live && final_state) {
        final_state[static_cast<size_t>(b) * C + c] = sv.x;
        final_state[static_cast<size_t>(b) * C + c + 1] = sv.y;
    }
}

template <typename E, bool REV>
cudaError_t launch_typed(const EmaArgs& a, CUtensorMapDataType dt) {
    using G = EmaTile<E>;
    CUtensorMap tmx, tmf;
    if (!make_btc_map(&tmx, a.x, dt, sizeof(E), a.B, a.T, a.C, kCW, G::TT) ||
        !make_btc_map(&tmf, a.f, dt, sizeof(E), a.B, a.T, a.C, kCW, G::TT))
        return cudaErrorInvalidValue;
    const cudaError_t e =
        cudaFuncSetAttribute(ema_kernel<E, REV>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    ema_kernel<E, REV><<<dim3((a.C + kCW - 1) / kCW, a.B), kThreads, G::SMEM, a.stream>>>(
        tmx, tmf, a.init_state, static_cast<E*>(a.out), a.final_state, a.T, a.C, a.err_word);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ema(const EmaArgs& a) {
    if (a.T == 0) {  // no steps: the state passes through
        if (!a.final_state || a.final_state == a.init_state) return cudaSuccess;
        const size_t bytes = sizeof(float) * static_cast<size_t>(a.B) * a.C;
        return a.init_state ? cudaMemcpyAsync(a.final_state, a.init_state, bytes, cudaMemcpyDeviceToDevice, a.stream)
                            : cudaMemsetAsync(a.final_state, 0, bytes, a.stream);
    }
    if (a.dtype == LA_BF16)
        return a.reverse ? launch_typed<__nv_bfloat16, true>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)
                         : launch_typed<__nv_bfloat16, false>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    return a.reverse ? launch_typed<float, true>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32)
                     : launch_typed<float, false>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

}  // namespace la
