// la_fwd_ws.cuh - warp-specialised chunked forward of causal linear attention
// for bf16 inputs on tcgen05 tensor cores (sm_100a).  Included by the
// instantiation files la_fwd_ws_*.cu.
//
// Math (per (b, h); chunks of C = 128 tokens; L_t = chunk-local prefix sum of
// log2 g up to token t, L_C its chunk total; S, z = state and key sum carried
// into the chunk):
//
//   y_t   = sum_{s<=t} 2^(L_t - L_s) (q_t . k_s) v_s + 2^(L_t) q_t^T S     (RetNet
//           issue 21: the scan is (Q K^T * D) V; flash-linear-attention issue
//           268: the carried state adds q^T S, the carried key sum q . z)
//   den_t = sum_{s<=t} 2^(L_t - L_s) (q_t . k_s)     + 2^(L_t) q_t . z
//   S'    = 2^(L_C) S + sum_s 2^(L_C - L_s) k_s v_s^T,  z' likewise with v = 1
//
// Folded decay.  With v'_s = 2^(-L_s) v_s (the value rows scaled in place) the
// decay leaves the score tile:
//   O = causal_mask(Q K^T) V' + Q S,   y_t = 2^(L_t) O_t,
//   S' = 2^(L_C) (S + K^T V').
// Each factor is bounded by 2^|L_C|; a chunk whose total decay exceeds
// kFoldLimit (log2 units) is computed in "direct" form instead:
// P = mask(Q K^T) * 2^(L_t - L_s) per element, Q~ = 2^(L_t) Q,
// K~ = 2^(L_C - L_s) K, O = P V + Q~ S, S' = 2^(L_C) S + K~^T V.  In both
// forms no exponent exceeds kFoldLimit and no factor can overflow (RWKV-LM
// discussion 189: use an exponentially weighted representation, never an
// unbounded w^(t-1) scale).
//
// Normaliser.  Two extra 16-column MMAs give the denominator in TMEM:
// P [w_hi w_lo 0 ..] plus Q [z_hi z_lo 0 ..], where w_s = 2^(-L_s) (1 in the
// direct form, whose P already holds the decay) and z are split into two
// bf16 parts (about 16 bits).  In the folded form numerator and denominator
// share the factor 2^(L_t), which cancels.  The key-sum update uses
// K^T [w_hi w_lo 0 ..].
//
// Roles (one CTA = one (b, h) and NV of its Dv columns; Dv / NV CTAs share a
// head and read its q, k through L2):
//   warp 0       TMA producer: Q, K, V tiles into an NSTG-deep stage ring
//   warp 1       MMA issuer (one thread) and TMEM owner
//   warps 2-9    two warpgroups: prep (decay prefix, in-place Q'/K' scaling)
//                and mask (A -> P, bf16, shared memory); warpgroup 0 owns
//                score columns 0-63 and the Q rows, warpgroup 1 columns
//                64-127 and the K rows
//   warps 10-..  state and epilogue (one warpgroup per 64 value columns):
//                S, z in fp32 registers, S' from the K'^T V tile, bf16 copy
//                of S for the next chunk's Q S; then y = O / den of the
//                previous chunk, bf16, stored to global memory
// Every hand-off is an mbarrier; every wait gives up after kWaitLimitNs (then
// the CTA sets the device error word and unwinds).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace ws {

constexpr int C = 128;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kFoldLimit = 64.f;
constexpr int kSmemLimit = 232448;
constexpr int B_COUNT_MAX = 31;  // barrier slots used (see Bar)

enum Mode : int { kModeNone = 0, kModeFolded = 1, kModeDirect = 2 };

__host__ __device__ constexpr int row_bytes_for(int width) { return width >= 64 ? 128 : width * 2; }
__host__ __device__ constexpr int panels_for(int width) { return width >= 64 ? width / 64 : 1; }
__host__ __device__ constexpr int round1k(int x) { return (x + 1023) / 1024 * 1024; }

template <int DK, int NV, bool NORM>
struct Plan {
    static constexpr int WK = row_bytes_for(DK), PK = panels_for(DK);
    static constexpr int WV = row_bytes_for(NV), PV = panels_for(NV);
    static constexpr int Q_BYTES = C * DK * 2;
    static constexpr int V_BYTES = C * NV * 2;
    // one stage: Q | K | V | W (normaliser weights) | L (float[C], log2 units) | meta
    static constexpr int ST_Q = 0, ST_K = Q_BYTES, ST_V = 2 * Q_BYTES;
    static constexpr int ST_W = 2 * Q_BYTES + V_BYTES;                  // [C x 16] bf16, 32-byte swizzle
    static constexpr int ST_LAM = ST_W + (NORM ? C * 32 : 0);
    static constexpr int ST_META = ST_LAM + C * 4;  // float L_C, int mode
    static constexpr int STAGE = round1k(ST_META + 64);
    static constexpr int P_BYTES = C * C * 2;
    static constexpr int SB_BYTES = round1k(DK * NV * 2);
    static constexpr int ZB_BYTES = NORM ? round1k(DK * 32) : 0;
    // barriers and flags, then the output row factors of the last kRowfRing chunks.
    // prep(c + R) may run once state(c + R - NSTG) is done, and the epilogue
    // of chunk c runs before that, so R = NSTG + 1 slots would do; 8 covers NSTG <= 4.
    static constexpr int kRowfRing = 8;
    static constexpr int MISC = 1024 + (NORM ? 0 : kRowfRing * C * 4);  // normalised: the factor cancels
    static constexpr bool fits(int ns, int np, int nsb) {
        return ns * STAGE + np * P_BYTES + nsb * (SB_BYTES + ZB_BYTES) + MISC + 1024 <= kSmemLimit;
    }
    static constexpr int NSTG = fits(4, 2, 2) ? 4 : fits(3, 2, 2) ? 3 : 2;
    static constexpr int NPB = (fits(NSTG, 2, 2) || fits(NSTG, 2, 1)) ? 2 : 1;
    static constexpr int NSB = fits(NSTG, NPB, 2) ? 2 : 1;
    static constexpr bool OK = fits(NSTG, NPB, NSB);
    static constexpr int OFF_P = NSTG * STAGE;
    static constexpr int OFF_SB = OFF_P + NPB * P_BYTES;
    static constexpr int OFF_ZB = OFF_SB + NSB * SB_BYTES;
    static constexpr int OFF_MISC = OFF_ZB + NSB * ZB_BYTES;
    static constexpr int OFF_ROWF = OFF_MISC + 1024;  // float[kRowfRing][C]: 2^(L_t) per token
    static constexpr int SMEM = OFF_MISC + MISC + 1024;
    // TMEM columns
    static constexpr int NDS = (256 + 2 * NV + (NORM ? 64 : 0)) <= 512 ? 2 : 1;
    static constexpr int COL_DS0 = 256;
    static constexpr int COL_ZS0 = 256 + NDS * NV;
    static constexpr int COL_QZ0 = COL_ZS0 + (NORM ? 16 * NDS : 0);
    static constexpr int TMEM_USED = COL_QZ0 + (NORM ? 32 : 0);
    static constexpr int TMEM_COLS = 512;
    // warps
    static constexpr int NSW = NV > 64 ? 2 : 1;
    static constexpr int NVW = NV / NSW;
    static constexpr int W_TMA = 0, W_MMA = 1, W_PM = 2, W_ES = 10;
    static constexpr int NWARPS = W_ES + 4 * NSW;
    static constexpr int THREADS = 32 * NWARPS;
    static constexpr int EMPTY_ARRIVALS = 1 + 8 + 4 * NSW;
    static constexpr uint32_t TX_BYTES = 2 * Q_BYTES + V_BYTES;
    static constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0, 0);
    static constexpr uint32_t IDESC_PV = make_idesc_bf16(128, NV, 0, 1);
    static constexpr uint32_t IDESC_KV = make_idesc_bf16(128, NV, 1, 1);
    static constexpr uint32_t IDESC_N16 = make_idesc_bf16(128, 16, 0, 1);
    static constexpr uint32_t IDESC_KV16 = make_idesc_bf16(128, 16, 1, 1);
    static_assert(TMEM_USED <= TMEM_COLS, "tensor memory budget");
    static_assert(kRowfRing >= NSTG + 1, "row factor ring too shallow");
    static_assert(!OK || OFF_MISC + 8 * B_COUNT_MAX + 8 <= OFF_MISC + 1024, "barrier area");
    static_assert(!OK || NORM || OFF_ROWF + kRowfRing * C * 4 <= SMEM - 1024, "row factor ring inside allocation");
    static_assert(!OK || OFF_MISC + MISC + 1024 <= SMEM, "regions inside allocation");
    static_assert(!OK || SMEM <= kSmemLimit, "shared memory limit");
    static_assert(NV % 16 == 0 && NV >= 16 && NV <= 128, "value slice");
    static_assert(DK == 16 || DK == 32 || DK == 64 || DK == 128, "key width");
};

// Barrier slots (uint64 each) inside the MISC area.
enum Bar : int {
    B_FULL = 0,      // [4] TMA -> consumers
    B_EMPTY = 4,     // [4] stage free
    B_PREP = 8,      // [4] decay prefix and in-place scaling done
    B_AFULL = 12,    // [2] scores in TMEM
    B_OFULL = 14,    // [2] O (and den) in TMEM
    B_OEMPTY = 16,   // [2] epilogue done with a TMEM region
    B_PFULL = 18,    // [2] P in shared memory
    B_PEMPTY = 20,   // [2] MMA done reading P
    B_DSFULL = 22,   // [2] K'^T V in TMEM
    B_DSEMPTY = 24,  // [2] state warps done with it
    B_SBFULL = 26,   // [2] bf16 state copy written
    B_SBEMPTY = 28,  // [2] MMA done reading it
    B_DRAIN = 30,
    B_COUNT = 31
};

struct Params {
    const float* log_g;
    int decay_kind;
    const float* init_state;
    const float* init_z;
    __nv_bfloat16* out;
    float* final_state;
    float* final_z;
    int H, T, Dv, split, nchunks;
    int* err;
};

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void fail(const Params& p, volatile int* abort, int code) {
    *abort = 1;
    if (p.err) atomicCAS(p.err, 0, code);
}

constexpr uint32_t kSleepHintNs = 20000;  // longest single sleep inside a wait

// Single-thread bounded wait; sleeps in the barrier between checks.
__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t parity, volatile int* abort, const Params& p,
                                      int code) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, kSleepHintNs)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            fail(p, abort, code);
            return false;
        }
    }
}

// Whole-warp bounded wait; every lane gets the same answer.
__device__ __forceinline__ bool waitw(uint64_t* bar, uint32_t parity, volatile int* abort, const Params& p,
                                      int code) {
    bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (!ok) ok = mbar_try_wait_sleep(bar, parity, kSleepHintNs);
        if (__all_sync(0xffffffffu, ok)) return true;
        bool give_up = *abort != 0;
        if (!give_up && global_timer_ns() - t0 > kWaitLimitNs) give_up = true;
        if (__any_sync(0xffffffffu, give_up)) {
            if ((threadIdx.x & 31) == 0) fail(p, abort, code);
            return false;
        }
    }
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Multiply the bf16 row `row` of a swizzled [C x width] tile by f, in place.
template <int WIDTH>
__device__ __forceinline__ void scale_row(uint8_t* tile, int row, float f) {
    constexpr int W = row_bytes_for(WIDTH), NP = panels_for(WIDTH), NCH = NP * W / 16;
    constexpr int BATCH = NCH < 4 ? NCH : 4;  // loads in flight before the first store
#pragma unroll
    for (int i0 = 0; i0 < NCH; i0 += BATCH) {
        uint4 w[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int ci = i0 + i;
            w[i] = *reinterpret_cast<const uint4*>(tile + (ci / (W / 16)) * C * W + swz(row, (ci % (W / 16)) * 16, W));
        }
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int ci = i0 + i;
            __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&w[i]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(hv[e]);
                hv[e] = __floats2bfloat162_rn(x.x * f, x.y * f);
            }
            *reinterpret_cast<uint4*>(tile + (ci / (W / 16)) * C * W + swz(row, (ci % (W / 16)) * 16, W)) = w[i];
        }
    }
}

// Columns 16 piece .. 16 piece + 15 of row t of a P panel (128-byte swizzle):
// a[e] where 16 piece + e <= lim, else 0; as bf16.
__device__ __forceinline__ void store_masked16(uint8_t* panel, int t, int piece, const float (&a)[16], int lim) {
    float m[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) m[e] = (16 * piece + e <= lim) ? a[e] : 0.f;
    const uint4 w0 = make_uint4(pack2(m[0], m[1]), pack2(m[2], m[3]), pack2(m[4], m[5]), pack2(m[6], m[7]));
    const uint4 w1 = make_uint4(pack2(m[8], m[9]), pack2(m[10], m[11]), pack2(m[12], m[13]), pack2(m[14], m[15]));
    *reinterpret_cast<uint4*>(panel + swz(t, 32 * piece, 128)) = w0;
    *reinterpret_cast<uint4*>(panel + swz(t, 32 * piece + 16, 128)) = w1;
}

// What every role needs from the kernel prologue (passed by value).
struct Ctx {
    const Params* p;
    uint8_t* sm;
    uint32_t sa, tmem;
    int bh, h, j0, slice;
};

template <int DK, int NV, bool NORM>
__device__ __noinline__ void role_tma(const Ctx x, const CUtensorMap* tmq_p, const CUtensorMap* tmk_p, const CUtensorMap* tmv_p) {
    using G = Plan<DK, NV, NORM>;
    const Params& p = *x.p;
    uint8_t* const sm = x.sm;
    const uint32_t sa = x.sa, tmem = x.tmem;
    uint64_t* const bar = reinterpret_cast<uint64_t*>(sm + G::OFF_MISC);
    volatile int* const abort = reinterpret_cast<volatile int*>(sm + G::OFF_MISC + 8 * B_COUNT + 4);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = x.bh, h = x.h, j0 = x.j0, slice = x.slice;
    const int T = p.T, n = p.nchunks;
    auto stage_ptr = [&](int s) { return sm + s * G::STAGE; };
    auto stage_addr = [&](int s) { return sa + s * G::STAGE; };
    (void)h; (void)j0; (void)slice; (void)T; (void)lane; (void)warp; (void)tmem; (void)stage_addr; (void)stage_ptr;
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
        int issued = 0;
        for (int c = 0; c < n; ++c) {
            const int s = c % G::NSTG;
            if (c >= G::NSTG && !wait1(&bar[B_EMPTY + s], ((c / G::NSTG) - 1) & 1, abort, p, kErrTmaWait))
                break;
            mbar_arrive_expect_tx(&bar[B_FULL + s], G::TX_BYTES);
            uint8_t* st = stage_ptr(s);
            for (int pp = 0; pp < G::PK; ++pp) {
                tma_load_3d(st + G::ST_Q + pp * C * G::WK, tmq_p, &bar[B_FULL + s], pp * 64, c * C, bh);
                tma_load_3d(st + G::ST_K + pp * C * G::WK, tmk_p, &bar[B_FULL + s], pp * 64, c * C, bh);
            }
            for (int pp = 0; pp < G::PV; ++pp)
                tma_load_3d(st + G::ST_V + pp * C * G::WV, tmv_p, &bar[B_FULL + s], j0 + pp * 64, c * C, bh);
            ++issued;
        }
        if (*abort) {
            // let issued copies land before the CTA's shared memory goes away
            const int first = issued > G::NSTG ? issued - G::NSTG : 0;
            for (int c = first; c < issued; ++c)
                mbar_wait_bounded(&bar[B_FULL + c % G::NSTG], (c / G::NSTG) & 1, kWaitLimitNs);
        }
    }
}

template <int DK, int NV, bool NORM>
__device__ __noinline__ void role_mma(const Ctx x) {
    using G = Plan<DK, NV, NORM>;
    const Params& p = *x.p;
    uint8_t* const sm = x.sm;
    const uint32_t sa = x.sa, tmem = x.tmem;
    uint64_t* const bar = reinterpret_cast<uint64_t*>(sm + G::OFF_MISC);
    volatile int* const abort = reinterpret_cast<volatile int*>(sm + G::OFF_MISC + 8 * B_COUNT + 4);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = x.bh, h = x.h, j0 = x.j0, slice = x.slice;
    const int T = p.T, n = p.nchunks;
    auto stage_ptr = [&](int s) { return sm + s * G::STAGE; };
    auto stage_addr = [&](int s) { return sa + s * G::STAGE; };
    (void)h; (void)j0; (void)slice; (void)T; (void)lane; (void)warp; (void)tmem; (void)stage_addr; (void)stage_ptr;
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the schedule (so descriptors stay warp-uniform);
    // one elected lane issues every MMA and commit.
    const bool leader = elect_one();
    int kv_next = 0;  // K'^T V tiles are issued in chunk order
    auto kstep = [](int kk, int W) -> uint32_t {  // byte offset of K step kk in a K-major tile
        return ((kk * 16) / (W / 2)) * C * W + ((kk * 16) % (W / 2)) * 2;
    };
    auto issue_kv = [&](int c) -> bool {
        const int s = c % G::NSTG, b = c % G::NDS;
        if (c >= G::NDS && !waitw(&bar[B_DSEMPTY + b], ((c / G::NDS) - 1) & 1, abort, p, kErrMmaWait))
            return false;
        tc_fence_after_sync();
        // M = 128 key rows; for Dk < 128 a zero panel offset repeats the key panel
        const uint64_t dk = make_smem_desc(stage_addr(s) + G::ST_K, DK == 128 ? C * G::WK : 0, 8 * G::WK, G::WK);
        const uint64_t dv = make_smem_desc(stage_addr(s) + G::ST_V, C * G::WV, 8 * G::WV, G::WV);
        if (leader) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem + G::COL_DS0 + b * NV, dk + ((kk * 16 * G::WK) >> 4), dv + ((kk * 16 * G::WV) >> 4),
                          G::IDESC_KV, kk > 0);
            if (NORM) {
                const uint64_t dw = make_smem_desc(stage_addr(s) + G::ST_W, 0, 8 * 32, 32);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    umma_bf16(tmem + G::COL_ZS0 + b * 16, dk + ((kk * 16 * G::WK) >> 4), dw + ((kk * 16 * 32) >> 4),
                              G::IDESC_KV16, kk > 0);
            }
            umma_commit(&bar[B_DSFULL + b]);
        }
        __syncwarp();
        return true;
    };
    for (int c = 0; c <= n; ++c) {
        int mode_c = kModeNone;
        if (c < n) {
            const int s = c % G::NSTG, r = c & 1;
            if (!waitw(&bar[B_PREP + s], (c / G::NSTG) & 1, abort, p, kErrMmaWait)) break;
            mode_c = *reinterpret_cast<volatile int*>(stage_ptr(s) + G::ST_META + 4);
            if (c >= 2 && !waitw(&bar[B_OEMPTY + r], ((c >> 1) - 1) & 1, abort, p, kErrMmaWait)) break;
            tc_fence_after_sync();
            const uint64_t dq = make_smem_desc(stage_addr(s) + G::ST_Q, 16, 8 * G::WK, G::WK);
            const uint64_t dkk = make_smem_desc(stage_addr(s) + G::ST_K, 16, 8 * G::WK, G::WK);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    umma_bf16(tmem + 128 * r, dq + (kstep(kk, G::WK) >> 4), dkk + (kstep(kk, G::WK) >> 4),
                              G::IDESC_QK, kk > 0);
                umma_commit(&bar[B_AFULL + r]);
            }
            __syncwarp();
            if (kv_next == c && mode_c != kModeDirect) {
                if (!issue_kv(c)) break;
                ++kv_next;
            }
        }
        if (c >= 1) {
            const int cp = c - 1, sp = cp % G::NSTG, rp = cp & 1, pb = cp % G::NPB, sbb = cp % G::NSB;
            if (!waitw(&bar[B_PFULL + pb], (cp / G::NPB) & 1, abort, p, kErrMmaWait)) break;
            tc_fence_after_sync();
            if (kv_next == cp) {  // direct-form chunk: its keys were decayed by the mask warps
                if (!issue_kv(cp)) break;
                ++kv_next;
            }
            if (c < n && kv_next == c && mode_c != kModeDirect) {
                if (!issue_kv(c)) break;
                ++kv_next;
            }
            if (!waitw(&bar[B_SBFULL + sbb], (cp / G::NSB) & 1, abort, p, kErrMmaWait)) break;
            tc_fence_after_sync();
            const uint64_t dp = make_smem_desc(sa + G::OFF_P + pb * G::P_BYTES, 16, 8 * 128, 128);
            const uint64_t dq = make_smem_desc(stage_addr(sp) + G::ST_Q, 16, 8 * G::WK, G::WK);
            const uint64_t dv = make_smem_desc(stage_addr(sp) + G::ST_V, C * G::WV, 8 * G::WV, G::WV);
            const uint64_t dsb =
                make_smem_desc(sa + G::OFF_SB + sbb * G::SB_BYTES, DK * G::WV, 8 * G::WV, G::WV);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    umma_bf16(tmem + 128 * rp, dp + (kstep(kk, 128) >> 4), dv + ((kk * 16 * G::WV) >> 4),
                              G::IDESC_PV, kk > 0);
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    umma_bf16(tmem + 128 * rp, dq + (kstep(kk, G::WK) >> 4), dsb + ((kk * 16 * G::WV) >> 4),
                              G::IDESC_PV, 1);
                if (NORM) {
                    const uint64_t dzb = make_smem_desc(sa + G::OFF_ZB + sbb * G::ZB_BYTES, 0, 8 * 32, 32);
                    const uint64_t dw = make_smem_desc(stage_addr(sp) + G::ST_W, 0, 8 * 32, 32);
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        umma_bf16(tmem + G::COL_QZ0 + 16 * rp, dp + (kstep(kk, 128) >> 4),
                                  dw + ((kk * 16 * 32) >> 4), G::IDESC_N16, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        umma_bf16(tmem + G::COL_QZ0 + 16 * rp, dq + (kstep(kk, G::WK) >> 4),
                                  dzb + ((kk * 16 * 32) >> 4), G::IDESC_N16, 1);
                }
                umma_commit(&bar[B_OFULL + rp]);
                umma_commit(&bar[B_PEMPTY + pb]);
                umma_commit(&bar[B_SBEMPTY + sbb]);
                umma_commit(&bar[B_EMPTY + sp]);
            }
            __syncwarp();
        }
    }
    // everything issued has completed before TMEM is released
    if (leader) umma_commit(&bar[B_DRAIN]);
    __syncwarp();
    mbar_wait_bounded(&bar[B_DRAIN], 0, kWaitLimitNs);
}

template <int DK, int NV, bool NORM>
__device__ __noinline__ void role_prep_mask(const Ctx x) {
    using G = Plan<DK, NV, NORM>;
    const Params& p = *x.p;
    uint8_t* const sm = x.sm;
    const uint32_t sa = x.sa, tmem = x.tmem;
    uint64_t* const bar = reinterpret_cast<uint64_t*>(sm + G::OFF_MISC);
    volatile int* const abort = reinterpret_cast<volatile int*>(sm + G::OFF_MISC + 8 * B_COUNT + 4);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = x.bh, h = x.h, j0 = x.j0, slice = x.slice;
    const int T = p.T, n = p.nchunks;
    auto stage_ptr = [&](int s) { return sm + s * G::STAGE; };
    auto stage_addr = [&](int s) { return sa + s * G::STAGE; };
    (void)h; (void)j0; (void)slice; (void)T; (void)lane; (void)warp; (void)tmem; (void)stage_addr; (void)stage_ptr;
    // ------------------------------------------------------------ prep + mask
    const int wg = (warp - G::W_PM) / 4;  // 0: columns 0-63 and Q rows; 1: columns 64-127 and K rows
    const int wq = warp & 3;
    const int t = 32 * wq + lane;        // TMEM lane = token row
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * wq) << 16);
    const int kind = p.decay_kind;
    const float* lg = p.log_g + static_cast<size_t>(bh) * T;
    const float ell_head = kind == LA_DECAY_PER_HEAD ? p.log_g[h] * kLog2e : 0.f;
    float nxt[4] = {0.f, 0.f, 0.f, 0.f};
    auto fetch = [&](int c) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = c * C + 32 * i + lane;
            nxt[i] = (kind == LA_DECAY_PER_STEP && c < n && row < T) ? lg[row] : 0.f;
        }
    };
    fetch(0);
    // decay prefix of the chunk being prepared (nx_*) and of the chunk being masked (cu_*);
    // scalars, not arrays indexed by chunk parity, so they stay in registers
    float nx_lt = 0.f, nx_lc = 0.f, cu_lt = 0.f, cu_lc = 0.f;
    int nx_md = kModeNone, cu_md = kModeNone;

    auto prep = [&](int c) -> bool {
        const int s = c % G::NSTG, rem = min(C, T - c * C);
        float cur[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
        fetch(c + 1);
        if (!waitw(&bar[B_FULL + s], (c / G::NSTG) & 1, abort, p, kErrTmaWait)) return false;
        float lt = 0.f, lc = 0.f;
        if (kind == LA_DECAY_PER_STEP) {
            float tot[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x = cur[i] * kLog2e;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                tot[i] = x;
            }
            float x = (wq == 0 ? cur[0] : wq == 1 ? cur[1] : wq == 2 ? cur[2] : cur[3]) * kLog2e;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            float off = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < wq) off += tot[i];
            lt = x + off;
            lc = tot[0] + tot[1] + tot[2] + tot[3];
        } else if (kind == LA_DECAY_PER_HEAD) {
            lt = static_cast<float>(min(t + 1, rem)) * ell_head;
            lc = static_cast<float>(rem) * ell_head;
        }
        const int md = kind == LA_DECAY_NONE ? kModeNone : (-lc <= kFoldLimit ? kModeFolded : kModeDirect);
        uint8_t* st = stage_ptr(s);
        if (wg == 0) {
            reinterpret_cast<float*>(st + G::ST_LAM)[t] = lt;
            if (t == 0) {
                *reinterpret_cast<float*>(st + G::ST_META) = lc;
                *reinterpret_cast<int*>(st + G::ST_META + 4) = md;
            }
        }
        if (wg == 0) {
            // output row factor 2^(L_t) of the folded form (1 otherwise); the
            // normalised output does not need it (and has no ring for it)
            if (!NORM)
                reinterpret_cast<float*>(sm + G::OFF_ROWF)[(c % G::kRowfRing) * C + t] =
                    md == kModeFolded ? ex2_approx(lt) : 1.f;
            if (md == kModeFolded) scale_row<NV>(st + G::ST_V, t, ex2_approx(-lt));
        } else if (NORM) {
            // normaliser weights w_t = 2^(-L_t) (1 unless folded), as a bf16 hi/lo pair
            const float w = md == kModeFolded ? ex2_approx(-lt) : 1.f;
            const float hi = __bfloat162float(__float2bfloat16_rn(w));
            *reinterpret_cast<uint4*>(st + G::ST_W + swz(t, 0, 32)) = make_uint4(pack2(hi, w - hi), 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(st + G::ST_W + swz(t, 16, 32)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
        warp_arrive(&bar[B_PREP + s]);
        nx_lt = lt;
        nx_lc = lc;
        nx_md = md;
        return true;
    };

    auto pmask = [&](int c) -> bool {
        const int s = c % G::NSTG, pb = c % G::NPB, r = c & 1;
        if (c >= G::NPB && !waitw(&bar[B_PEMPTY + pb], ((c / G::NPB) - 1) & 1, abort, p, kErrMmaWait))
            return false;
        if (!waitw(&bar[B_AFULL + r], (c >> 1) & 1, abort, p, kErrMmaWait)) return false;
        if (!waitw(&bar[B_PREP + s], (c / G::NSTG) & 1, abort, p, kErrMmaWait)) return false;
        tc_fence_after_sync();
        uint8_t* st = stage_ptr(s);
        uint8_t* pt = sm + G::OFF_P + pb * G::P_BYTES;  // panel wg holds score columns 64 wg .. 64 wg + 63
        const float* lam = reinterpret_cast<const float*>(st + G::ST_LAM);
        const float lt = cu_lt, lc = cu_lc;
        const int md = cu_md;
        const bool all_masked = (32 * wq + 31) < 64 * wg;  // every row of this warp precedes these columns
        uint8_t* prow = pt + wg * C * 128;  // this warpgroup's panel of P
        if (md != kModeDirect) {
            // causal mask only: two loads in flight per wait
            const int lim = all_masked ? -1 : t - 64 * wg;  // keep columns j <= lim of this panel
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float a0[16], a1[16];
                if (!all_masked) {
                    tmem_ld16(lane_addr + 128 * r + 64 * wg + 32 * half, a0);
                    tmem_ld16(lane_addr + 128 * r + 64 * wg + 32 * half + 16, a1);
                    tmem_wait_ld();
                }
                store_masked16(prow, t, 2 * half, a0, lim);
                store_masked16(prow, t, 2 * half + 1, a1, lim);
            }
        } else {
            // direct form: P = mask(A) * 2^(L_t - L_s), one 16-column piece at a time
#pragma unroll 1
            for (int piece = 0; piece < 4; ++piece) {
                float a[16];
                if (!all_masked) {
                    tmem_ld16(lane_addr + 128 * r + 64 * wg + 16 * piece, a);
                    tmem_wait_ld();
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int scol = 64 * wg + 16 * piece + e;
                    a[e] = (scol <= t && !all_masked) ? a[e] * ex2_approx(lt - lam[scol]) : 0.f;
                }
                store_masked16(prow, t, piece, a, 64);
            }
        }
        if (md == kModeDirect) {
            if (wg == 0) scale_row<DK>(st + G::ST_Q, t, ex2_approx(lt));
            else scale_row<DK>(st + G::ST_K, t, ex2_approx(lc - lt));
        }
        tc_fence_before_sync();
        fence_async_smem();
        warp_arrive(&bar[B_PFULL + pb]);
        warp_arrive(&bar[B_EMPTY + s]);
        return true;
    };

    if (n > 0 && prep(0)) {
        for (int c = 0; c < n; ++c) {
            cu_lt = nx_lt;
            cu_lc = nx_lc;
            cu_md = nx_md;
            if (c + 1 < n && !prep(c + 1)) break;
            if (!pmask(c)) break;
        }
    }
}

template <int DK, int NV, bool NORM>
__device__ __noinline__ void role_state_epilogue(const Ctx x) {
    using G = Plan<DK, NV, NORM>;
    const Params& p = *x.p;
    uint8_t* const sm = x.sm;
    const uint32_t sa = x.sa, tmem = x.tmem;
    uint64_t* const bar = reinterpret_cast<uint64_t*>(sm + G::OFF_MISC);
    volatile int* const abort = reinterpret_cast<volatile int*>(sm + G::OFF_MISC + 8 * B_COUNT + 4);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = x.bh, h = x.h, j0 = x.j0, slice = x.slice;
    const int T = p.T, n = p.nchunks;
    auto stage_ptr = [&](int s) { return sm + s * G::STAGE; };
    auto stage_addr = [&](int s) { return sa + s * G::STAGE; };
    (void)h; (void)j0; (void)slice; (void)T; (void)lane; (void)warp; (void)tmem; (void)stage_addr; (void)stage_ptr;
    // ------------------------------------------------------------ state + epilogue
    // Warpgroup wg owns value columns [wg NVW, (wg + 1) NVW) of the slice.
    // Per chunk c: the epilogue of chunk c - 1, then the state update of
    // chunk c (its bf16 copy gates the next chunk's Q S).
    const int wg = (warp - G::W_ES) / 4;
    const int wq = warp & 3;
    const int d = 32 * wq + lane;          // key row of S; also token row t of O
    const bool warp_rows = 32 * wq < DK;   // this warp holds real rows of S
    const bool row_ok = d < DK;
    const int cb = wg * G::NVW;            // first column (within the slice) of this warpgroup
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * wq) << 16);
    float S[G::NVW];
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < G::NVW; ++j) S[j] = 0.f;
    if (row_ok && p.init_state) {
        const float* src = p.init_state + (static_cast<size_t>(bh) * DK + d) * p.Dv + j0 + cb;
#pragma unroll
        for (int j = 0; j < G::NVW; j += 4) {
            const float4 x = *reinterpret_cast<const float4*>(src + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
    }
    if (NORM && row_ok && p.init_z) z = p.init_z[static_cast<size_t>(bh) * DK + d];

    auto write_copy = [&](int k) {  // bf16 copy of S (and z) for production index k
        const int buf = k % G::NSB;
        uint8_t* sb = sm + G::OFF_SB + buf * G::SB_BYTES;
        if (row_ok) {
#pragma unroll
            for (int j = 0; j < G::NVW; j += 8) {
                const int col = cb + j;
                const int per_panel = G::WV / 2;
                *reinterpret_cast<uint4*>(sb + (col / per_panel) * DK * G::WV + swz(d, (col % per_panel) * 2, G::WV)) =
                    make_uint4(pack2(S[j], S[j + 1]), pack2(S[j + 2], S[j + 3]), pack2(S[j + 4], S[j + 5]),
                               pack2(S[j + 6], S[j + 7]));
            }
            if (NORM && wg == 0) {
                const float hi = __bfloat162float(__float2bfloat16_rn(z));
                const float lo = z - hi;
                *reinterpret_cast<uint4*>(sm + G::OFF_ZB + buf * G::ZB_BYTES + swz(d, 0, 32)) =
                    make_uint4(pack2(hi, lo), 0u, 0u, 0u);
            }
        }
        fence_async_smem();
        warp_arrive(&bar[B_SBFULL + buf]);
    };

    auto state = [&](int c) -> bool {
        const int s = c % G::NSTG, b = c % G::NDS;
        if (!waitw(&bar[B_PREP + s], (c / G::NSTG) & 1, abort, p, kErrMmaWait)) return false;
        const uint8_t* st = stage_ptr(s);
        const float lc = *reinterpret_cast<const volatile float*>(st + G::ST_META);
        const int md = *reinterpret_cast<const volatile int*>(st + G::ST_META + 4);
        if (!waitw(&bar[B_DSFULL + b], (c / G::NDS) & 1, abort, p, kErrMmaWait)) return false;
        tc_fence_after_sync();
        // S' from the K'^T V tile, 16 columns at a time
        const float e = md == kModeNone ? 1.f : ex2_approx(lc);
        if (warp_rows) {
#pragma unroll
            for (int j = 0; j < G::NVW; j += 16) {
                float ds[16];
                tmem_ld16(lane_addr + G::COL_DS0 + b * NV + cb + j, ds);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (md == kModeFolded) S[j + i] = e * (S[j + i] + ds[i]);
                    else if (md == kModeDirect) S[j + i] = fmaf(e, S[j + i], ds[i]);
                    else S[j + i] += ds[i];
                }
            }
            if (NORM && wg == 0) {
                float zz[16];
                tmem_ld16(lane_addr + G::COL_ZS0 + 16 * b, zz);
                tmem_wait_ld();
                if (md == kModeFolded) z = e * (z + zz[0]);
                else if (md == kModeDirect) z = fmaf(e, z, zz[0]);
                else z += zz[0];
            }
        }
        tc_fence_before_sync();
        warp_arrive(&bar[B_DSEMPTY + b]);
        warp_arrive(&bar[B_EMPTY + s]);
        if (c == n - 1) return true;
        const int k = c + 1;
        if (k >= G::NSB &&
            !waitw(&bar[B_SBEMPTY + k % G::NSB], ((k / G::NSB) - 1) & 1, abort, p, kErrMmaWait))
            return false;
        write_copy(k);
        return true;
    };

    auto epilogue = [&](int c) -> bool {
        const int r = c & 1, t = d;
        if (!waitw(&bar[B_OFULL + r], (c >> 1) & 1, abort, p, kErrMmaWait)) return false;
        tc_fence_after_sync();
        float inv;  // y = O * inv
        if (NORM) {
            float dd[16];
            tmem_ld16(lane_addr + G::COL_QZ0 + 16 * r, dd);
            tmem_wait_ld();
            inv = 1.f / (dd[0] + dd[1]);
        } else {
            inv = reinterpret_cast<const float*>(sm + G::OFF_ROWF)[(c % G::kRowfRing) * C + t];
        }
        const int rem = min(C, T - c * C);
        __nv_bfloat16* dst =
            p.out + (static_cast<size_t>(bh) * T + static_cast<size_t>(c) * C + t) * p.Dv + j0 + cb;
        constexpr int NB = G::NVW < 64 ? G::NVW / 16 : 4;  // pieces loaded per wait
#pragma unroll
        for (int piece = 0; piece < G::NVW / 16; ++piece) {
            float o[16];
            tmem_ld16(lane_addr + 128 * r + cb + 16 * piece, o);
            if (piece % NB == NB - 1) tmem_wait_ld();
            if (t < rem) {
                uint4* d4 = reinterpret_cast<uint4*>(dst + 16 * piece);
                d4[0] = make_uint4(pack2(o[0] * inv, o[1] * inv), pack2(o[2] * inv, o[3] * inv),
                                   pack2(o[4] * inv, o[5] * inv), pack2(o[6] * inv, o[7] * inv));
                d4[1] = make_uint4(pack2(o[8] * inv, o[9] * inv), pack2(o[10] * inv, o[11] * inv),
                                   pack2(o[12] * inv, o[13] * inv), pack2(o[14] * inv, o[15] * inv));
            }
        }
        tc_fence_before_sync();
        warp_arrive(&bar[B_OEMPTY + r]);
        return true;
    };

    // The epilogue of chunk c - 1 runs before the state update of chunk c:
    // for a direct-form chunk c the MMA warp issues K~^T V(c) only after
    // this warpgroup has released the TMEM region of chunk c - 1.
    write_copy(0);
    bool ok = true;
    for (int c = 0; c < n && ok; ++c) {
        if (c >= 1) ok = epilogue(c - 1);
        if (ok) ok = state(c);
    }
    if (ok && n > 0) ok = epilogue(n - 1);
    if (ok && !*abort && row_ok) {
        if (p.final_state) {
            float* fs = p.final_state + (static_cast<size_t>(bh) * DK + d) * p.Dv + j0 + cb;
#pragma unroll
            for (int j = 0; j < G::NVW; j += 4)
                *reinterpret_cast<float4*>(fs + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        if (NORM && p.final_z && slice == 0 && wg == 0) p.final_z[static_cast<size_t>(bh) * DK + d] = z;
    }
}

template <int DK, int NV, bool NORM>
__global__ void __launch_bounds__(Plan<DK, NV, NORM>::THREADS, 1)
    fwd_ws_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ Params p) {
    using G = Plan<DK, NV, NORM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sa = smem_u32(sm);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + G::OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + G::OFF_MISC + 8 * B_COUNT);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + G::OFF_MISC + 8 * B_COUNT + 4);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int bh = blockIdx.x / p.split, slice = blockIdx.x % p.split;
    const int h = bh % p.H;
    const int j0 = slice * NV;
    const int T = p.T, n = p.nchunks;

    if (tid == 0) {
        prefetch_tensormap(&tmq);
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bar[B_FULL + s], 1);
            mbar_init(&bar[B_EMPTY + s], G::EMPTY_ARRIVALS);
            mbar_init(&bar[B_PREP + s], 8);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[B_AFULL + i], 1);
            mbar_init(&bar[B_OFULL + i], 1);
            mbar_init(&bar[B_OEMPTY + i], 4 * G::NSW);
            mbar_init(&bar[B_PFULL + i], 8);
            mbar_init(&bar[B_PEMPTY + i], 1);
            mbar_init(&bar[B_DSFULL + i], 1);
            mbar_init(&bar[B_DSEMPTY + i], 4 * G::NSW);
            mbar_init(&bar[B_SBFULL + i], 4 * G::NSW);
            mbar_init(&bar[B_SBEMPTY + i], 1);
        }
        mbar_init(&bar[B_DRAIN], 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == G::W_MMA) tmem_alloc(tmem_slot, G::TMEM_COLS);
    if (NORM && warp >= G::W_ES && warp < G::W_ES + 4) {
        // zeroed key-sum tiles (only their first two columns are ever written)
        const int t = tid - 32 * G::W_ES;
        for (int i = t; i < G::NSB * G::ZB_BYTES / 16; i += 128)
            reinterpret_cast<uint4*>(sm + G::OFF_ZB)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const Ctx x{&p, sm, sa, tmem, bh, h, j0, slice};
    if (warp == G::W_TMA) {
        role_tma<DK, NV, NORM>(x, &tmq, &tmk, &tmv);
    } else if (warp == G::W_MMA) {
        role_mma<DK, NV, NORM>(x);
    } else if (warp < G::W_ES) {
        role_prep_mask<DK, NV, NORM>(x);
    } else {
        role_state_epilogue<DK, NV, NORM>(x);
    }

    __syncwarp();  // lanes that idled while lane 0 ran a single-thread role rejoin it
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == G::W_MMA) tmem_dealloc(tmem, G::TMEM_COLS);
}

template <int DK, int NV, bool NORM>
cudaError_t launch_instance(const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                            const Params& p, int grid, cudaStream_t stream) {
    using G = Plan<DK, NV, NORM>;
    if constexpr (!G::OK) {
        return cudaErrorNotSupported;
    } else {
        // at least 116 KB so that one CTA (512 TMEM columns) owns each SM
        const int smem = G::SMEM > 116 * 1024 ? G::SMEM : 116 * 1024;
        cudaError_t e =
            cudaFuncSetAttribute(fwd_ws_kernel<DK, NV, NORM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        fwd_ws_kernel<DK, NV, NORM><<<grid, G::THREADS, smem, stream>>>(tmq, tmk, tmv, p);
        return cudaGetLastError();
    }
}

template <int DK, int NV, bool NORM>
constexpr bool supported() {
    return Plan<DK, NV, NORM>::OK;
}

}  // namespace ws
}  // namespace la
