// la_wkv4.cu - the RWKV-4 WKV recurrence (BlinkDL/RWKV-LM issue 167, the
// att_seq time loop), two channels per thread.
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
// Data movement: a CTA owns one batch row, kCW consecutive channels and one
// T-segment.  One producer thread streams [TT tokens x kCW channels] tiles
// of k and v into a ring of kStages shared-memory stages with TMA (four CTAs
// per SM, about 200 KB in flight per SM), so the HBM latency is hidden
// behind the sequential per-token work; each consumer thread reads its two
// channels' columns of the tile as one pair and writes its two outputs as
// one pair (a warp writes 64 consecutive values).  The two channels' chains
// are independent, and their adds, multiplies and fmas issue as packed
// fp32x2 instructions.
//
// Parallelism: a channel's recurrence is sequential in t, and B x C channels
// alone leave each scheduler about one warp.  With a workspace, each sequence
// is cut into T-segments: a state pass computes every earlier segment's own
// (aa, bb, pp) from an empty state, and the output pass starts segment s
// from the initial state combined with them in order (decay the running
// state over a segment's tokens, then add that segment's state with the same
// max-shifted weighting the loop uses), which multiplies the independent
// chains per SM.
// Every barrier wait gives up after kWaitLimitNs, sets the device error word
// and unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

constexpr int kConsumerWarps = 2;
constexpr int kCW = 64 * kConsumerWarps;  // channels per CTA: two per consumer thread
constexpr int kStages = 3;                // 3 x 16 KB: four CTAs per SM
constexpr int kThreads = 32 * (kConsumerWarps + 1);  // + one producer warp
constexpr int kCtasPerSm = 4;
constexpr int kMinSegTokens = 512;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kEmptyScale = -1e38f;   // pp of an empty state (aa = bb = 0)

template <typename E>
struct Tile {
    static constexpr int TT = sizeof(E) == 2 ? 32 : 16;           // tokens per stage
    static constexpr int BYTES = TT * kCW * static_cast<int>(sizeof(E));  // one array's tile
    static constexpr int STAGE = 2 * BYTES;                        // k tile, then v tile
    static constexpr int SMEM = kStages * STAGE + 256;             // + barriers
};

// T-segments: segment s covers tokens [s * seg_len, min(T, (s + 1) * seg_len)).
// The state pass (state_pass = 1, segments 0 .. nseg - 2) writes each
// segment's own state, from an empty one, to ws slot s + 1, and its segment-0
// CTAs copy the initial state to slot 0; the output pass starts segment s
// from slot 0 combined with slots 1 .. s.  ws is [B][nseg][3][C] fp32.
struct WkvParams {
    const float* w;
    const float* u;
    const float* init_state;
    void* out;
    float* final_state;
    float* ws;
    int T, C, seg_len, nseg, state_pass;
    int* err;
};

// Weights of two terms with log2 weights a and b against the larger one:
// one of them is 1, the other 2^-|a - b| (one exponential per pair).
__device__ __forceinline__ void shifted_pair(float a, float b, float& fa, float& fb) {
    const float d = a - b;
    const float t = ex2_approx(-fabsf(d));
    fa = d >= 0.f ? 1.f : t;
    fb = d >= 0.f ? t : 1.f;
}

// The same weights from the difference d = a - b.
__device__ __forceinline__ void shifted_diff(float d, float& fa, float& fb) {
    const float t = ex2_approx(-fabsf(d));
    fa = d >= 0.f ? 1.f : t;
    fb = d >= 0.f ? t : 1.f;
}

// Two adjacent channels' values as fp32 pairs.
__device__ __forceinline__ float2 load_f2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load_f2(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ void store_e2(float* p, float2 y) { *reinterpret_cast<float2*>(p) = y; }
__device__ __forceinline__ void store_e2(__nv_bfloat16* p, float2 y) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(y.x, y.y);
}


template <typename E>
__global__ void __launch_bounds__(kThreads) wkv4_kernel(const __grid_constant__ CUtensorMap tmk,
                                                        const __grid_constant__ CUtensorMap tmv,
                                                        const __grid_constant__ WkvParams p) {
    using G = Tile<E>;
    // used as declared (not realigned through an integer), so that the
    // compiler keeps the shared address space and reads tiles with LDS;
    // TMA without swizzle needs 16-byte alignment only
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kStages * G::STAGE);
    uint64_t* empty = full + kStages;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + kStages);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int b = blockIdx.y, c0 = blockIdx.x * kCW, seg = blockIdx.z;
    const int T = p.T, C = p.C;
    const int t0 = seg * p.seg_len, t1 = min(T, t0 + p.seg_len);
    const int j0 = t0 / G::TT, ntiles = (t1 - t0 + G::TT - 1) / G::TT;  // seg_len is a multiple of TT

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
                    if (p.err) atomicCAS(p.err, 0, kErrTmaWait);
                    break;
                }
                if (*abort) break;
                uint8_t* st = sm + s * G::STAGE;
                mbar_arrive_expect_tx(&full[s], G::STAGE);
                tma_load_3d(st, &tmk, &full[s], c0, (j0 + j) * G::TT, b);
                tma_load_3d(st + G::BYTES, &tmv, &full[s], c0, (j0 + j) * G::TT, b);
                ++issued;
            }
            // copies in flight land before the CTA's shared memory goes away
            for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
                mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, kWaitLimitNs);
        }
        return;
    }

    // consumer: thread = two adjacent channels (C is even, so a pair never
    // straddles the end)
    const int c = c0 + 2 * threadIdx.x;
    const bool live = c < C;
    const size_t plane = static_cast<size_t>(C);
    float W[2], U[2], aa[2], bb[2], P[2];
    float* slot0 = p.ws ? p.ws + static_cast<size_t>(b) * p.nseg * 3 * plane + c : nullptr;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        W[e] = live ? p.w[c + e] * kLog2e : 0.f;
        U[e] = live ? p.u[c + e] * kLog2e : 0.f;
        aa[e] = 0.f;
        bb[e] = 0.f;
        P[e] = kEmptyScale * kLog2e;
        if (!live) continue;
        if (p.state_pass) {
            if (seg == 0) {  // keep the initial state for the output pass
                const float* s0 = p.init_state ? p.init_state + static_cast<size_t>(b) * 3 * plane + c + e : nullptr;
                slot0[e] = s0 ? s0[0] : 0.f;
                slot0[e + plane] = s0 ? s0[plane] : 0.f;
                slot0[e + 2 * plane] = s0 ? s0[2 * plane] : kEmptyScale;
            }
        } else if (p.ws) {
            // the initial state, then each earlier segment: decayed over that
            // segment's tokens, plus the segment's own state (max-shifted add)
            aa[e] = slot0[e];
            bb[e] = slot0[e + plane];
            P[e] = slot0[e + 2 * plane] * kLog2e;
            for (int j = 0; j < seg; ++j) {
                const float* sj = slot0 + e + static_cast<size_t>(j + 1) * 3 * plane;
                const float Pd = P[e] + W[e] * static_cast<float>(p.seg_len);
                const float Pj = sj[2 * plane] * kLog2e;
                float fa, fb;
                shifted_pair(Pd, Pj, fa, fb);
                aa[e] = fmaf(fa, aa[e], fb * sj[0]);
                bb[e] = fmaf(fa, bb[e], fb * sj[plane]);
                P[e] = fmaxf(Pd, Pj);
            }
        } else if (p.init_state) {
            const float* s0 = p.init_state + static_cast<size_t>(b) * 3 * plane + c + e;
            aa[e] = s0[0];
            bb[e] = s0[plane];
            P[e] = s0[2 * plane] * kLog2e;
        }
    }
    E* o = static_cast<E*>(p.out) + (static_cast<size_t>(b) * T + t0) * C + c;
    // One token on both channels: read-out (the state at log weight P, this
    // token at U + K), then update (the state decayed to W + P, this token at
    // K).  Adds, multiplies and fmas in packed fp32x2 arithmetic (each lane
    // rounded as its scalar form would be); exponentials, compares and
    // maxima per channel.
    const float2 W2 = make_float2(W[0], W[1]), U2 = make_float2(U[0], U[1]);
    const float2 m1 = make_float2(-1.f, -1.f), l2e = make_float2(kLog2e, kLog2e);
    float2 aa2 = make_float2(aa[0], aa[1]), bb2 = make_float2(bb[0], bb[1]), P2 = make_float2(P[0], P[1]);
    auto update = [&](float2 K, float2 v) {
        const float2 d = __fadd2_rn(W2, P2);
        const float2 x = __ffma2_rn(K, m1, d);  // d - K
        float2 f1, f2;
        shifted_diff(x.x, f1.x, f2.x);
        shifted_diff(x.y, f1.y, f2.y);
        aa2 = __ffma2_rn(f1, aa2, __fmul2_rn(f2, v));
        bb2 = __ffma2_rn(f1, bb2, f2);
        P2 = make_float2(fmaxf(d.x, K.x), fmaxf(d.y, K.y));
    };
    auto step = [&](float2 K, float2 v) -> float2 {
        const float2 x = __ffma2_rn(__fadd2_rn(U2, K), m1, P2);  // P - (U + K)
        float2 e1, e2;
        shifted_diff(x.x, e1.x, e2.x);
        shifted_diff(x.y, e1.y, e2.y);
        const float2 num = __ffma2_rn(e1, aa2, __fmul2_rn(e2, v)), den = __ffma2_rn(e1, bb2, e2);
        update(K, v);
        return make_float2(__fdividef(num.x, den.x), __fdividef(num.y, den.y));
    };
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j % kStages;
        // whole-warp bounded wait on the tile
        bool got = mbar_try_wait(&full[s], (j / kStages) & 1);
        if (!__all_sync(0xffffffffu, got)) {
            const uint64_t tw = global_timer_ns();
            while (true) {
                if (!got) got = mbar_try_wait_sleep(&full[s], (j / kStages) & 1, 20000);
                if (__all_sync(0xffffffffu, got)) break;
                bool give_up = *abort != 0 || global_timer_ns() - tw > kWaitLimitNs;
                if (__any_sync(0xffffffffu, give_up)) {
                    if (lane == 0) {
                        *abort = 1;
                        if (p.err) atomicCAS(p.err, 0, kErrTmaWait);
                    }
                    ok = false;
                    break;
                }
            }
            if (!ok) break;
        }
        const E* tk = reinterpret_cast<const E*>(sm + s * G::STAGE) + 2 * threadIdx.x;
        const E* tv = reinterpret_cast<const E*>(sm + s * G::STAGE + G::BYTES) + 2 * threadIdx.x;
        const int n = min(G::TT, t1 - (j0 + j) * G::TT);
        if (live && p.state_pass) {
#pragma unroll 8
            for (int i = 0; i < n; ++i) update(__fmul2_rn(load_f2(tk + i * kCW), l2e), load_f2(tv + i * kCW));
        } else if (live) {
            // batches of 8 tokens: the next batch's tile reads are issued
            // before this batch's dependent steps, the outputs stored after
            // them, so that memory latency stays off the recurrence's path
            const int nb = n / 8;
            float2 kk[8], vv[8];
            if (nb > 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kk[e] = load_f2(tk + e * kCW);
                    vv[e] = load_f2(tv + e * kCW);
                }
            }
            for (int bi = 0; bi < nb; ++bi) {
                float2 kn[8], vn[8], yy[8];
                const int nxt = bi + 1 < nb ? (bi + 1) * 8 : bi * 8;  // (a harmless re-read at the end)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kn[e] = load_f2(tk + (nxt + e) * kCW);
                    vn[e] = load_f2(tv + (nxt + e) * kCW);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) yy[e] = step(__fmul2_rn(kk[e], l2e), vv[e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) store_e2(o + static_cast<size_t>(e) * C, yy[e]);
                o += static_cast<size_t>(8) * C;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kk[e] = kn[e];
                    vv[e] = vn[e];
                }
            }
            for (int i = nb * 8; i < n; ++i) {
                store_e2(o, step(__fmul2_rn(load_f2(tk + i * kCW), l2e), load_f2(tv + i * kCW)));
                o += C;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!ok || !live) return;
    float* dst = nullptr;
    if (p.state_pass)
        dst = slot0 + static_cast<size_t>(seg + 1) * 3 * plane;
    else if (seg == p.nseg - 1 && p.final_state)
        dst = p.final_state + static_cast<size_t>(b) * 3 * plane + c;
    if (dst) {
        dst[0] = aa2.x;
        dst[1] = aa2.y;
        dst[plane] = bb2.x;
        dst[plane + 1] = bb2.y;
        dst[2 * plane] = P2.x * (1.f / kLog2e);
        dst[2 * plane + 1] = P2.y * (1.f / kLog2e);
    }
}

bool make_wkv_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int es, int B, int T, int C, int TT) {
    return make_btc_map(map, base, dt, es, B, T, C, kCW, TT);
}

int sm_count_wkv() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || v <= 0)
        v = 148;
    return v;
}

// Segments per sequence: doubled while every segment's CTAs still fit on the
// GPU at once (kCtasPerSm per SM) and segments keep >= kMinSegTokens tokens;
// the segment length is a whole number of tiles.
struct WkvLayout {
    int nseg, seg_len;
};

WkvLayout wkv_layout(int B, int T, int C, int tt, bool segments) {
    const long long ctas = static_cast<long long>(B) * ((C + kCW - 1) / kCW);
    const long long resident = static_cast<long long>(sm_count_wkv()) * kCtasPerSm;
    int nseg = 1;
    if (segments)
        while (ctas * nseg * 2 <= resident && T / (nseg * 2) >= kMinSegTokens) nseg *= 2;
    int seg_len = (T + nseg - 1) / nseg;
    seg_len = (seg_len + tt - 1) / tt * tt;
    if (seg_len < 1) seg_len = tt;
    return WkvLayout{(T + seg_len - 1) / seg_len, seg_len};
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
    // all of the SM's shared memory, so that kCtasPerSm CTAs stay resident
    e = cudaFuncSetAttribute(wkv4_kernel<E>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    WkvLayout L = wkv_layout(a.B, a.T, a.C, G::TT, a.workspace != nullptr);
    const size_t need = sizeof(float) * static_cast<size_t>(a.B) * L.nseg * 3 * a.C;
    if (L.nseg > 1 && a.workspace_bytes < need) L = wkv_layout(a.B, a.T, a.C, G::TT, false);
    WkvParams p{};
    p.w = a.w;
    p.u = a.u;
    p.init_state = a.init_state;
    p.out = a.out;
    p.final_state = a.final_state;
    p.T = a.T;
    p.C = a.C;
    p.seg_len = L.seg_len;
    p.nseg = L.nseg;
    p.err = a.err_word;
    const int tiles = (a.C + kCW - 1) / kCW;
    if (L.nseg > 1) {
        p.ws = static_cast<float*>(a.workspace);
        WkvParams ps = p;
        ps.state_pass = 1;
        wkv4_kernel<E><<<dim3(tiles, a.B, L.nseg - 1), kThreads, G::SMEM, a.stream>>>(tmk, tmv, ps);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    wkv4_kernel<E><<<dim3(tiles, a.B, L.nseg), kThreads, G::SMEM, a.stream>>>(tmk, tmv, p);
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

// [B, T, C] tensor, boxes of [1, box_t tokens, box_c channels], no swizzle.
bool make_btc_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int es, int B, int T, int C, int box_c,
                  int box_t) {
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(C) * es, static_cast<cuuint64_t>(C) * es * T};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_c), static_cast<cuuint32_t>(box_t), 1};
    const cuuint32_t elem[3] = {1, 1, 1};
    return f(map, dt, 3, const_cast<void*>(base), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t wkv4_workspace_bytes(int B, int T, int C, la_dtype dtype) {
    if (B < 1 || T < 1 || C < 1) return 0;
    const WkvLayout L = wkv_layout(B, T, C, dtype == LA_BF16 ? Tile<__nv_bfloat16>::TT : Tile<float>::TT, true);
    if (L.nseg < 2) return 0;
    const size_t b = sizeof(float) * static_cast<size_t>(B) * L.nseg * 3 * C;
    return (b + 255) / 256 * 256;
}

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
