// la_fwd_tc.cuh - chunked forward of causal linear attention for bf16 inputs
// on tcgen05 tensor cores (sm_100a).  Included by the per-Dk instantiation
// files la_fwd_tc_dk*.cu.
//
// The sequence is cut into chunks of C = 128 tokens.  With Lambda_t the
// chunk-local prefix sum of log g up to token t (log2 units below) and S the
// state carried into the chunk, each chunk computes (RetNet issue 21: the scan
// equals (Q K^T * D) V with the causal decay mask D; flash-linear-attention
// issue 268: the carried state and key sum enter as cache terms):
//
//   A      = Q K^T                                   (MMA, 128 x 128, TMEM)
//   P[t,s] = A[t,s] exp(Lambda_t - Lambda_s), s <= t (threads; bf16 to smem)
//   O      = P V  +  diag(exp(Lambda_t)) (Q S)       (two MMAs, TMEM)
//   den_t  = sum_s P[t,s] + exp(Lambda_t) q_t . z    (normalised only)
//   y_t    = O_t (/ den_t)
//   S     <- exp(Lambda_C) S + (diag(exp(Lambda_C - Lambda_s)) K)^T V   (MMA)
//   z     <- exp(Lambda_C) z + sum_s exp(Lambda_C - Lambda_s) k_s
//
// Every exponent above is <= 0, so no factor exceeds 1 and nothing
// overflows or needs a NaN fix-up (RWKV-LM discussion 189: work with the
// exponentially weighted parameterisation rather than scaling by w^(t-1)).
//
// One CTA (128 threads, 4 warps) owns one (b, h) and NV of its Dv value
// columns; Dv / NV CTAs share a head and read the same q, k tiles (through
// L2).  Thread t owns TMEM lane t: token row t of A / O, and key row t of S.
//
// Shared memory (1024-byte aligned panels, 128/64/32-byte TMA swizzle):
//   Q, K  [2 stages][128 tokens x DK]   K-major operands; K is also the
//                                       MN-major A operand of K^T V
//   V     [2 stages][128 tokens x NV]   MN-major B operand
//   P     [128 x 128] bf16              K-major A operand (aliases the Q
//                                       stage when DK = 128)
//   Sb    [DK x NV] bf16 copy of S      MN-major B operand of Q S
// TMEM columns: [0,128) A then O_intra, [128,128+NV) Q S, [128+NV,128+2NV) S.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace tc {

constexpr int C = 128;          // tokens per chunk = MMA M
constexpr int kThreads = 128;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per barrier wait
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr int row_bytes_for(int width) { return width >= 64 ? 128 : width * 2; }
__host__ __device__ constexpr int panels_for(int width) { return width >= 64 ? width / 64 : 1; }
__host__ __device__ constexpr int round1k(int x) { return (x + 1023) / 1024 * 1024; }

template <int DK, int NV>
struct Cfg {
    static constexpr int WK = row_bytes_for(DK);  // bytes per swizzled row of a Q / K panel
    static constexpr int PK = panels_for(DK);
    static constexpr int WV = row_bytes_for(NV);
    static constexpr int PV = panels_for(NV);
    static constexpr int Q_BYTES = C * DK * 2;
    static constexpr int V_BYTES = C * NV * 2;
    static constexpr int P_BYTES = C * C * 2;
    static constexpr int SB_BYTES = DK * NV * 2;
    static constexpr bool P_IN_Q = (DK == 128);
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + 2 * Q_BYTES;
    static constexpr int OFF_P = OFF_V + 2 * V_BYTES;
    static constexpr int OFF_SB = OFF_P + (P_IN_Q ? 0 : P_BYTES);
    static constexpr int OFF_LAM = OFF_SB + round1k(SB_BYTES);  // float[C], log2 units
    static constexpr int OFF_Z = OFF_LAM + C * 4;                // float[128]
    static constexpr int OFF_WTOT = OFF_Z + 128 * 4;             // float[4]
    static constexpr int OFF_BAR = OFF_WTOT + 16;                // u64 tma[2], mma
    static constexpr int OFF_TMEM = OFF_BAR + 24;                // u32
    static constexpr int BYTES = OFF_TMEM + 4;
    static constexpr int SMEM = BYTES + 1024;                    // + base alignment slack
    static constexpr int COL_O = 0, COL_QS = C, COL_S = C + NV;
    static constexpr int TMEM_COLS = (C + 2 * NV) <= 256 ? 256 : 512;
    static constexpr uint32_t TX_BYTES = 2 * Q_BYTES + V_BYTES;
    static constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0, 0);
    static constexpr uint32_t IDESC_QS = make_idesc_bf16(128, NV, 0, 1);
    static constexpr uint32_t IDESC_PV = make_idesc_bf16(128, NV, 0, 1);
    static constexpr uint32_t IDESC_KV = make_idesc_bf16(128, NV, 1, 1);
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(NV % 16 == 0 && NV >= 16 && NV <= 128, "value slice");
    static_assert(DK == 16 || DK == 32 || DK == 64 || DK == 128, "key width");
};

struct Params {
    const float* log_g;
    int decay_kind;
    int normalize;
    const float* init_state;
    const float* init_z;
    __nv_bfloat16* out;
    float* final_state;
    float* final_z;
    int H, T, Dv, split, nchunks;
    int* err;
};

// K-major operand: 16-element K step `kk` of a tile with `rows` rows whose
// K extent is split into panels of row_bytes / 2 elements.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk, int row_bytes, int rows) {
    const int e0 = kk * 16;
    const int per_panel = row_bytes / 2;
    const uint32_t start = tile + (e0 / per_panel) * rows * row_bytes + (e0 % per_panel) * 2;
    return make_smem_desc(start, 16, 8 * row_bytes, row_bytes);
}

// MN-major operand: 16-row K step `kk`; `lbo` = distance between panels
// along MN (0 repeats the first panel).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk, int row_bytes, uint32_t lbo) {
    return make_smem_desc(tile + kk * 16 * row_bytes, lbo, 8 * row_bytes, row_bytes);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b, float& rsum) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 back = __bfloat1622float2(h);
    rsum += back.x + back.y;
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// A wait that gave up: remember it in this thread and in the device error
// word.  Threads agree on stopping through __syncthreads_or, so every thread
// leaves the chunk loop at the same barrier.
__device__ __forceinline__ void record_error(int* err, bool& failed, int code) {
    failed = true;
    if (err) atomicCAS(err, 0, code);
}

template <int DK, int NV>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const Params p) {
    using G = Cfg<DK, NV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float* lam2 = reinterpret_cast<float*>(sm + G::OFF_LAM);
    float* zs = reinterpret_cast<float*>(sm + G::OFF_Z);
    float* wtot = reinterpret_cast<float*>(sm + G::OFF_WTOT);
    uint64_t* tma_bar = reinterpret_cast<uint64_t*>(sm + G::OFF_BAR);
    uint64_t* mma_bar = tma_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + G::OFF_TMEM);
    bool failed = false, aborted = false;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int bh = blockIdx.x / p.split, slice = blockIdx.x % p.split;
    const int h = bh % p.H;
    const int j0 = slice * NV;
    const int T = p.T, nchunks = p.nchunks;
    const bool has_init = p.init_state != nullptr;
    const int kind = p.decay_kind;

    if (tid == 0) {
        prefetch_tensormap(&tmq);
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
        mbar_init(&tma_bar[0], 1);
        mbar_init(&tma_bar[1], 1);
        mbar_init(mma_bar, 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, G::TMEM_COLS);
    for (int i = tid; i < DK; i += kThreads)
        zs[i] = (p.normalize && p.init_z) ? p.init_z[static_cast<size_t>(bh) * DK + i] : 0.f;
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);

    const uint32_t q_base = sbase + G::OFF_Q, k_base = sbase + G::OFF_K, v_base = sbase + G::OFF_V;
    const uint32_t sb_addr = sbase + G::OFF_SB;
    uint8_t* const sb_ptr = sm + G::OFF_SB;

    // thread 0 issues every TMA load and MMA; it alone tracks what is in flight
    int loads_issued = 0, mma_commits = 0;
    auto issue_loads = [&](int cc) {
        const int st = cc & 1;
        mbar_arrive_expect_tx(&tma_bar[st], G::TX_BYTES);
        uint8_t* qd = sm + G::OFF_Q + st * G::Q_BYTES;
        uint8_t* kd = sm + G::OFF_K + st * G::Q_BYTES;
        uint8_t* vd = sm + G::OFF_V + st * G::V_BYTES;
        for (int pp = 0; pp < G::PK; ++pp) {
            tma_load_3d(qd + pp * C * G::WK, &tmq, &tma_bar[st], pp * 64, cc * C, bh);
            tma_load_3d(kd + pp * C * G::WK, &tmk, &tma_bar[st], pp * 64, cc * C, bh);
        }
        for (int pp = 0; pp < G::PV; ++pp)
            tma_load_3d(vd + pp * C * G::WV, &tmv, &tma_bar[st], j0 + pp * 64, cc * C, bh);
        ++loads_issued;
    };
    if (tid == 0)
        for (int cc = 0; cc < 2 && cc < nchunks; ++cc) issue_loads(cc);

    // carried state: fp32 into TMEM (rows = key index), bf16 copy into Sb
    if (has_init && warp * 32 < DK) {
        const bool row_ok = tid < DK;
        const float* src = p.init_state + (static_cast<size_t>(bh) * DK + (row_ok ? tid : 0)) * p.Dv + j0;
#pragma unroll
        for (int cb = 0; cb < NV / 16; ++cb) {
            float r[16];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 x = row_ok ? *reinterpret_cast<const float4*>(src + cb * 16 + e)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                r[e] = x.x; r[e + 1] = x.y; r[e + 2] = x.z; r[e + 3] = x.w;
            }
            tmem_st16(lane_addr + G::COL_S + cb * 16, r);
            if (row_ok) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int j = cb * 16 + half * 8;
                    const uint4 w = make_uint4(pack_bf16(r[half * 8 + 0], r[half * 8 + 1]),
                                               pack_bf16(r[half * 8 + 2], r[half * 8 + 3]),
                                               pack_bf16(r[half * 8 + 4], r[half * 8 + 5]),
                                               pack_bf16(r[half * 8 + 6], r[half * 8 + 7]));
                    const int per_panel = G::WV / 2;
                    *reinterpret_cast<uint4*>(sb_ptr + (j / per_panel) * DK * G::WV +
                                              swz(tid, (j % per_panel) * 2, G::WV)) = w;
                }
            }
        }
        tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    uint32_t mma_phase = 0;
    const size_t lg_row = static_cast<size_t>(bh) * T;
    float ell_next = 0.f;
    if (kind == LA_DECAY_PER_STEP && tid < T) ell_next = p.log_g[lg_row + tid];
    const float ell_head = (kind == LA_DECAY_PER_HEAD) ? p.log_g[h] * kLog2e : 0.f;

    int c = 0;
    for (; c < nchunks; ++c) {
        const int st = c & 1;
        const int rem = min(C, T - c * C);
        const bool live = has_init || c > 0;
        const uint32_t q_tile = q_base + st * G::Q_BYTES;
        const uint32_t k_tile = k_base + st * G::Q_BYTES;
        const uint32_t v_tile = v_base + st * G::V_BYTES;
        uint8_t* const q_ptr = sm + G::OFF_Q + st * G::Q_BYTES;
        uint8_t* const k_ptr = sm + G::OFF_K + st * G::Q_BYTES;
        const uint32_t p_tile = G::P_IN_Q ? q_tile : sbase + G::OFF_P;
        uint8_t* const p_ptr = G::P_IN_Q ? q_ptr : sm + G::OFF_P;

        // chunk-local prefix of log2 decay, row tid
        float lam_t = 0.f;
        if (kind == LA_DECAY_PER_STEP) {
            float x = ell_next * kLog2e;
            const int tn = (c + 1) * C + tid;
            ell_next = (tn < T) ? p.log_g[lg_row + tn] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane == 31) wtot[warp] = x;
            lam_t = x;
        } else if (kind == LA_DECAY_PER_HEAD) {
            lam_t = static_cast<float>(min(tid + 1, rem)) * ell_head;
        }

        if (!mbar_wait_bounded(&tma_bar[st], (c >> 1) & 1, kWaitLimitNs))
            record_error(p.err, failed, kErrTmaWait);
        if (__syncthreads_or(failed)) {
            aborted = true;
            break;
        }
        if (kind == LA_DECAY_PER_STEP)
            for (int w = 0; w < warp; ++w) lam_t += wtot[w];
        lam2[tid] = lam_t;

        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma_bf16(tmem + G::COL_O, desc_kmajor(q_tile, kk, G::WK, C), desc_kmajor(k_tile, kk, G::WK, C),
                          G::IDESC_QK, kk > 0);
            if (live) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    umma_bf16(tmem + G::COL_QS, desc_kmajor(q_tile, kk, G::WK, C),
                              desc_mnmajor(sb_addr, kk, G::WV, DK * G::WV), G::IDESC_QS, kk > 0);
            }
            umma_commit(mma_bar);
            ++mma_commits;
        }
        __syncthreads();  // lam2 complete
        const float lam_c = lam2[C - 1];

        // q_t . z (read before P may overwrite the Q tile)
        float qz = 0.f;
        if (p.normalize) {
#pragma unroll
            for (int pp = 0; pp < G::PK; ++pp) {
#pragma unroll
                for (int ch = 0; ch < G::WK / 16; ++ch) {
                    const uint4 w = *reinterpret_cast<const uint4*>(q_ptr + pp * C * G::WK + swz(tid, ch * 16, G::WK));
                    const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&w);
                    const int d0 = pp * (G::WK / 2) + ch * 8;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(hv[e]);
                        qz = fmaf(f.x, zs[d0 + 2 * e], qz);
                        qz = fmaf(f.y, zs[d0 + 2 * e + 1], qz);
                    }
                }
            }
        }

        if (!mbar_wait_bounded(mma_bar, mma_phase, kWaitLimitNs)) record_error(p.err, failed, kErrMmaWait);
        mma_phase ^= 1;
        tc_fence_after_sync();

        // P row tid: mask, decay, bf16 into the K-major P tile; fp32 row sum of the rounded values
        float rsum = 0.f;
#pragma unroll
        for (int cb = 0; cb < C / 32; ++cb) {
            float a[32];
            tmem_ld16(lane_addr + G::COL_O + cb * 32, *reinterpret_cast<float(*)[16]>(&a[0]));
            tmem_ld16(lane_addr + G::COL_O + cb * 32 + 16, *reinterpret_cast<float(*)[16]>(&a[16]));
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = cb * 32 + e;
                float f = (s <= tid) ? 1.f : 0.f;
                if (kind != LA_DECAY_NONE && s <= tid) f = exp2f(lam_t - lam2[s]);
                a[e] *= f;
            }
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int s0 = cb * 32 + ch * 8;
                const uint4 w = make_uint4(pack_bf16(a[ch * 8 + 0], a[ch * 8 + 1], rsum),
                                           pack_bf16(a[ch * 8 + 2], a[ch * 8 + 3], rsum),
                                           pack_bf16(a[ch * 8 + 4], a[ch * 8 + 5], rsum),
                                           pack_bf16(a[ch * 8 + 6], a[ch * 8 + 7], rsum));
                *reinterpret_cast<uint4*>(p_ptr + (s0 / 64) * C * 128 + swz(tid, (s0 % 64) * 2, 128)) = w;
            }
        }

        if (kind != LA_DECAY_NONE) {
            // decayed keys in place: row tid of K times exp(Lambda_C - Lambda_t)
            const float wk = exp2f(lam_c - lam_t);
#pragma unroll
            for (int pp = 0; pp < G::PK; ++pp) {
#pragma unroll
                for (int ch = 0; ch < G::WK / 16; ++ch) {
                    uint4* ptr = reinterpret_cast<uint4*>(k_ptr + pp * C * G::WK + swz(tid, ch * 16, G::WK));
                    uint4 w = *ptr;
                    __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(hv[e]);
                        hv[e] = __floats2bfloat162_rn(f.x * wk, f.y * wk);
                    }
                    *ptr = w;
                }
            }
            // carried state decays by the chunk total before the K^T V update
            if (live && warp * 32 < DK) {
                const float ec = exp2f(lam_c);
#pragma unroll
                for (int cb = 0; cb < NV / 16; ++cb) {
                    float r[16];
                    tmem_ld16(lane_addr + G::COL_S + cb * 16, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) r[e] *= ec;
                    tmem_st16(lane_addr + G::COL_S + cb * 16, r);
                }
                tmem_wait_st();
            }
        }
        const float et = exp2f(lam_t);
        const float den = rsum + et * qz;

        fence_async_smem();
        tc_fence_before_sync();
        if (__syncthreads_or(failed)) {
            aborted = true;
            break;
        }
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem + G::COL_O, desc_kmajor(p_tile, kk, 128, C),
                          desc_mnmajor(v_tile, kk, G::WV, C * G::WV), G::IDESC_PV, kk > 0);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem + G::COL_S, desc_mnmajor(k_tile, kk, G::WK, DK == 128 ? C * G::WK : 0),
                          desc_mnmajor(v_tile, kk, G::WV, C * G::WV), G::IDESC_KV, (kk > 0) || live);
            umma_commit(mma_bar);
            ++mma_commits;
        }

        // key sum, overlapping the MMAs (both only read the K tile)
        if (p.normalize && tid < DK) {
            const int per_panel = G::WK / 2;
            const uint8_t* col = k_ptr + (tid / per_panel) * C * G::WK;
            const int byte = (tid % per_panel) * 2;
            float acc = 0.f;
#pragma unroll 8
            for (int s = 0; s < C; ++s)
                acc += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(col + swz(s, byte, G::WK)));
            zs[tid] = fmaf(exp2f(lam_c), zs[tid], acc);
        }

        if (!mbar_wait_bounded(mma_bar, mma_phase, kWaitLimitNs)) record_error(p.err, failed, kErrMmaWait);
        mma_phase ^= 1;
        tc_fence_after_sync();

        // epilogue: y_t = O_intra + exp(Lambda_t) (q_t S)  (/ den_t)
        {
            const int t_glob = c * C + tid;
            __nv_bfloat16* dst = p.out + (static_cast<size_t>(bh) * T + t_glob) * p.Dv + j0;
            const float inv = p.normalize ? 1.f / den : 1.f;
#pragma unroll
            for (int cb = 0; cb < NV / 16; ++cb) {
                float o[16], oi[16];
                tmem_ld16(lane_addr + G::COL_O + cb * 16, o);
                if (live) tmem_ld16(lane_addr + G::COL_QS + cb * 16, oi);
                tmem_wait_ld();
                float y[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float val = live ? fmaf(et, oi[e], o[e]) : o[e];
                    y[e] = p.normalize ? val * inv : val;
                }
                if (tid < rem) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + cb * 16);
                    d4[0] = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                                       pack_bf16(y[6], y[7]));
                    d4[1] = make_uint4(pack_bf16(y[8], y[9]), pack_bf16(y[10], y[11]), pack_bf16(y[12], y[13]),
                                       pack_bf16(y[14], y[15]));
                }
            }
        }

        // state refresh: bf16 copy for the next chunk's Q S; fp32 final state
        if (warp * 32 < DK) {
            const bool row_ok = tid < DK;
            const bool last = (c == nchunks - 1);
#pragma unroll
            for (int cb = 0; cb < NV / 16; ++cb) {
                float r[16];
                tmem_ld16(lane_addr + G::COL_S + cb * 16, r);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int j = cb * 16 + half * 8;
                        const int per_panel = G::WV / 2;
                        const uint4 w = make_uint4(pack_bf16(r[half * 8 + 0], r[half * 8 + 1]),
                                                   pack_bf16(r[half * 8 + 2], r[half * 8 + 3]),
                                                   pack_bf16(r[half * 8 + 4], r[half * 8 + 5]),
                                                   pack_bf16(r[half * 8 + 6], r[half * 8 + 7]));
                        *reinterpret_cast<uint4*>(sb_ptr + (j / per_panel) * DK * G::WV +
                                                  swz(tid, (j % per_panel) * 2, G::WV)) = w;
                    }
                    if (last && p.final_state) {
                        float* fs = p.final_state + (static_cast<size_t>(bh) * DK + tid) * p.Dv + j0 + cb * 16;
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *reinterpret_cast<float4*>(fs + e) = make_float4(r[e], r[e + 1], r[e + 2], r[e + 3]);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (tid == 0 && c + 2 < nchunks) issue_loads(c + 2);
    }

    // every thread reaches this barrier once, whether the loop ran out or broke
    aborted = __syncthreads_or(failed);
    if (!aborted) {
        if (p.normalize && p.final_z && slice == 0)
            for (int i = tid; i < DK; i += kThreads) p.final_z[static_cast<size_t>(bh) * DK + i] = zs[i];
    } else if (tid == 0) {
        // drain what this CTA still has in flight before TMEM is released
        for (int cc = c; cc < loads_issued; ++cc)
            mbar_wait_bounded(&tma_bar[cc & 1], (cc >> 1) & 1, kWaitLimitNs);
        if ((mma_commits & 1) != static_cast<int>(mma_phase))
            mbar_wait_bounded(mma_bar, mma_phase, kWaitLimitNs);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, G::TMEM_COLS);
}

// Host side: launch one instantiation.  The tensor maps are built by the
// caller (la_fwd_tc.cu).
template <int DK, int NV>
cudaError_t launch_instance(const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                            const Params& p, int grid, cudaStream_t stream) {
    using G = Cfg<DK, NV>;
    // Request enough shared memory that no more CTAs share an SM than its
    // TMEM columns can hold at once (512 columns per SM).
    const int min_smem = G::TMEM_COLS == 512 ? 116 * 1024 : 78 * 1024;
    const int smem = G::SMEM > min_smem ? G::SMEM : min_smem;
    cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<DK, NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fwd_tc_kernel<DK, NV><<<grid, kThreads, smem, stream>>>(tmq, tmk, tmv, p);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace la
