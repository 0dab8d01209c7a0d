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
//   O = Q S + causal_mask(Q K^T) V',   y_t = 2^(L_t) O_t,
//   S' = 2^(L_C) (S + K^T V').
// Each factor is bounded by 2^|L_C|; a chunk whose total decay exceeds
// kFoldLimit (log2 units) is computed in "direct" form instead:
// P = mask(Q K^T) * 2^(L_t - L_s) per element, Q~ = 2^(L_t) Q,
// K~ = 2^(L_C - L_s) K, O = Q~ S + P V, S' = 2^(L_C) S + K~^T V.  In both
// forms no exponent exceeds kFoldLimit and no factor can overflow (RWKV-LM
// discussion 189: use an exponentially weighted representation, never an
// unbounded w^(t-1) scale).
//
// Normaliser.  Two extra 16-column MMAs give the denominator in TMEM, next to
// O: Q [z_hi z_lo 0 ..] plus P [w_hi w_lo 0 ..], where w_s = 2^(-L_s) (1 in
// the direct form, whose P already holds the decay) and z are split into two
// bf16 parts (about 16 bits).  In the folded form numerator and denominator
// share the factor 2^(L_t), which cancels.  The key-sum update uses
// K^T [w_hi w_lo 0 ..].
//
// Data flow.  Q, K and V tiles (the V stage with the chunk's decay prefix)
// sit in three TMA rings.  A K stage is free once Q K^T and K^T V' have run;
// a Q stage only after Q S, which waits for the state of the previous chunk,
// so the Q ring is the deeper one.  The inter-chunk term Q S is accumulated
// first, long before P V; P lives in tensor memory (the A operand of P V is
// read from TMEM), which keeps shared memory for the rings.
//
// Roles (one CTA = one (b, h) and NV of its Dv columns; Dv / NV CTAs share a
// head and read its q, k through L2):
//   warp 0       MMA issuer B (one elected lane): Q S and P V (a ready P V
//                first: it completes a chunk, and so frees its O buffer)
//   warp 1       MMA issuer A (one elected lane): Q K^T and K^T V'; TMEM owner
//   warps 2-9    two warpgroups: prep (decay prefix, value-row scaling,
//                normaliser weights) and mask (scores -> P in TMEM); warpgroup
//                0 owns score columns 0-63, warpgroup 1 columns 64-127 and
//                writes the outputs (epilogue); with the feature map, the
//                warpgroups map the Q and K tiles
//   warps 10-..  state: fp32 S in registers and its bf16 copy (one warpgroup
//                per 64 value columns)
//   last warp    TMA producer of the Q, K and V rings
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
constexpr unsigned kTmaIdleSleepNs = 64;  // the producer's pause after a pass that issued nothing
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kFoldLimit = 64.f;
constexpr int kSmemLimit = 232448;

enum Mode : int { kModeNone = 0, kModeFolded = 1, kModeDirect = 2 };

__host__ __device__ constexpr int row_bytes_for(int width) { return width >= 64 ? 128 : width * 2; }
__host__ __device__ constexpr int panels_for(int width) { return width >= 64 ? width / 64 : 1; }
__host__ __device__ constexpr int round1k(int x) { return (x + 1023) / 1024 * 1024; }

// Barrier slots (uint64 each) at the start of the MISC area.
enum Bar : int {
    B_QFULL = 0,     // [4] Q tile landed
    B_QEMPTY = 4,    // [4] Q stage free (Q K^T and Q S done)
    B_KFULL = 8,     // [4] K tile landed
    B_KEMPTY = 12,   // [4] K stage free (Q K^T and K^T V' done)
    B_VFULL = 16,    // [4] V tile landed
    B_VEMPTY = 20,   // [4] V stage free (P V done, its prefix read)
    B_PREP = 24,     // [4] decay prefix, value scaling, weights done
    B_AFULL = 28,    // [2] scores in TMEM
    B_AEMPTY = 30,   // [2] scores read by the mask warps
    B_PFULL = 32,    // [2] P in TMEM
    B_PEMPTY = 34,   // [2] P V done reading P
    B_OFULL = 36,    // [2] O (and den) complete
    B_OEMPTY = 38,   // [2] epilogue done with O
    B_DSFULL = 40,   // [2] K^T V' in TMEM
    B_DSEMPTY = 42,  // [2] state warps done with it
    B_SBFULL = 44,   // [2] bf16 state copy written
    B_SBEMPTY = 46,  // [2] Q S done reading it
    B_PHI = 48,      // [4] feature map applied to the chunk's Q and K tiles
    B_DRAIN = 52,    // MMA warp A's issued MMAs complete
    B_DRAINB = 53,   // MMA warp B's
    B_COUNT = 54
};

template <int DK, int NV, bool NORM, bool SP = false>
struct Plan {
    static constexpr int WK = row_bytes_for(DK), PK = panels_for(DK);
    // Value tiles (and the bf16 state copy, whose columns are value columns):
    // with the normaliser, panels of 16 columns (32-byte swizzle), so that the
    // weight panel W (16 columns) continues V and the key-sum panel continues
    // S: one MMA of N = NV + 16 then computes both, reading its A operand once.
    static constexpr int WV = NORM ? 32 : row_bytes_for(NV), PV = NORM ? NV / 16 : panels_for(NV);
    static constexpr int Q_BYTES = C * DK * 2;
    static constexpr int V_BYTES = C * NV * 2;
    // Q and K stages (one tile each)
    static constexpr int Q_STAGE = round1k(Q_BYTES);
    // V stage: V | W (normaliser weights, [C x 16] bf16, 32-byte swizzle) | L (float[C], log2) | meta
    static constexpr int VS_W = V_BYTES;
    static constexpr int VS_LAM = VS_W + (NORM ? C * 32 : 0);
    static constexpr int VS_META = VS_LAM + C * 4;  // float L_C, int mode
    static constexpr int V_STAGE = round1k(VS_META + 64);
    // bf16 state copy: S panels, then (normaliser) the key-sum panel [z_hi z_lo 0 ..]
    static constexpr int SB_ZB = DK * NV * 2;  // offset of the key-sum panel
    static constexpr int SB_BYTES = round1k(DK * NV * 2 + (NORM ? DK * 32 : 0));
    // barriers and flags, then the output row factors of the last kRowfRing
    // chunks (not needed with the normaliser, where the factor cancels).
    static constexpr int kRowfRing = 8;
    static constexpr int MISC = 1024 + (NORM ? 0 : kRowfRing * C * 4);
    static constexpr bool fits(int nq, int nk, int nvs, int nsb) {
        return (nq + nk) * Q_STAGE + nvs * V_STAGE + nsb * SB_BYTES + MISC + 1024 <= kSmemLimit;
    }
    // A ring of depth n whose stages each stay busy for a time L allows one
    // chunk per L / n.  Rough busy times (arbitrary units): a Q stage from its
    // load to the chunk's Q S, which waits for the state chain (40); a V stage
    // to its P V, after Q S (45); a K stage only to K^T V' (25).  A single
    // state copy adds a little.  The fitting plan with the smallest bound wins.
    static constexpr int bound(int nq, int nk, int nvs, int nsb) {
        int b = 400 / nq;
        if (250 / nk > b) b = 250 / nk;
        if (450 / nvs > b) b = 450 / nvs;
        return b + (nsb == 1 ? 20 : 0);
    }
    // A state pass (SP) reads no queries and keeps no state copy: its shared
    // memory holds only K and V rings, as deep as fit (at most 4, the
    // barrier slots per ring).  A K stage stays busy from its load to K^T V'
    // and a V stage a little longer (the state warps read its decay), about
    // equally long, so the deepest balanced rings win.
    static constexpr int bound_sp(int nk, int nvs) {
        const int a = 500 / nk, b = 520 / nvs;
        return a > b ? a : b;
    }
    static constexpr int pick() {
        int best = 0, bb = 1 << 30;
        if (SP) {
            for (int nk = 4; nk >= 2; --nk)
                for (int nvs = 4; nvs >= 2; --nvs)
                    if (fits(0, nk, nvs, 0) && bound_sp(nk, nvs) < bb) {
                        bb = bound_sp(nk, nvs);
                        best = nk * 100 + nvs * 10;
                    }
        } else {
            for (int nq = 4; nq >= 2; --nq)
                for (int nk = 4; nk >= 2; --nk)
                    for (int nvs = 4; nvs >= 2; --nvs)
                        for (int nsb = 2; nsb >= 1; --nsb)
                            if (fits(nq, nk, nvs, nsb) && bound(nq, nk, nvs, nsb) < bb) {
                                bb = bound(nq, nk, nvs, nsb);
                                best = nq * 1000 + nk * 100 + nvs * 10 + nsb;
                            }
        }
        return best;
    }
    static constexpr int PICK = pick();
    static constexpr bool OK = PICK != 0;
    // stages allocated (a state pass allocates no Q stage and no state copy)
    static constexpr int NQA = OK ? PICK / 1000 : 2;
    static constexpr int NSBA = OK ? PICK % 10 : 1;
    // ring lengths for the index arithmetic (at least 1; a state pass never
    // touches the Q ring or the state copy)
    static constexpr int NQ = NQA > 0 ? NQA : 1;
    static constexpr int NK = OK ? (PICK / 100) % 10 : 2;
    static constexpr int NVS = OK ? (PICK / 10) % 10 : 2;
    static constexpr int NSB = NSBA > 0 ? NSBA : 1;
    static constexpr int OFF_K = NQA * Q_STAGE;
    static constexpr int OFF_V = OFF_K + NK * Q_STAGE;
    static constexpr int OFF_SB = OFF_V + NVS * V_STAGE;
    static constexpr int OFF_MISC = OFF_SB + NSBA * SB_BYTES;
    static constexpr int OFF_ROWF = OFF_MISC + 1024;  // float[kRowfRing][C]: 2^(L_t) per token
    static constexpr int SMEM = OFF_MISC + MISC + 1024;
    // TMEM columns: scores 128 per buffer | P (bf16 pairs) 64 per buffer | O | K^T V'.
    // Double buffers in the order P, O, scores, K^T V' while they fit.
    static constexpr int OCOLS = NV + (NORM ? 16 : 0);
    static constexpr int tmem_need(int na, int npb, int no, int nds) {
        return 128 * na + 64 * npb + (no + nds) * OCOLS;
    }
    static constexpr int NPB = tmem_need(1, 2, 2, 1) <= 512 ? 2 : 1;
    static constexpr int NO = tmem_need(1, NPB, 2, 1) <= 512 ? 2 : 1;
    static constexpr int NA = tmem_need(2, NPB, NO, 1) <= 512 ? 2 : 1;
    // a state pass keeps only K^T V' in tensor memory: two buffers from column 0
    static constexpr int NDS = SP ? 2 : (tmem_need(NA, NPB, NO, 2) <= 512 ? 2 : 1);
    static constexpr int COL_P0 = 128 * NA;
    static constexpr int COL_O0 = COL_P0 + 64 * NPB;
    static constexpr int COL_DS0 = SP ? 0 : COL_O0 + NO * OCOLS;
    static constexpr int TMEM_USED = COL_DS0 + NDS * OCOLS;
    static constexpr int TMEM_COLS = 512;
    // warps
    static constexpr int NSW = NV > 64 ? 2 : 1;
    static constexpr int NVW = NV / NSW;
    static constexpr int W_MMAB = 0, W_MMA = 1, W_PM = 2, W_ES = 10;
    static constexpr int W_TMAV = W_ES + 4 * NSW;
    static constexpr int NWARPS = W_TMAV + 1;
    static constexpr int THREADS = 32 * NWARPS;
    static constexpr int VEMPTY_ARRIVALS = 1 + 8 + 4 * NSW;
    static constexpr uint32_t Q_TX = Q_BYTES;
    static constexpr uint32_t V_TX = V_BYTES;
    static constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0, 0);
    static constexpr int NOUT = NV + (NORM ? 16 : 0);  // value columns plus the normaliser panel
    static constexpr uint32_t IDESC_PV = make_idesc_bf16(128, NOUT, 0, 1);
    static constexpr uint32_t IDESC_KV = make_idesc_bf16(128, NOUT, 1, 1);
    static_assert(TMEM_USED <= TMEM_COLS, "tensor memory budget");
    static_assert(NV % 16 == 0 && NV >= 16 && NV <= 128, "value slice");
    static_assert(DK == 16 || DK == 32 || DK == 64 || DK == 128, "key width");
    // the epilogue of chunk c runs before the mask of chunk c + 2, so before
    // the prep of chunk c + 2 + NVS rewrites its row factors
    static_assert(kRowfRing >= NVS + 3, "row factor ring too shallow");
    static_assert(8 * B_COUNT + 8 <= 1024, "barrier area");
    static_assert(!OK || (OFF_K % 1024 == 0 && OFF_V % 1024 == 0), "stages aligned for 128-byte swizzle");
    static_assert(!OK || SMEM <= kSmemLimit, "shared memory limit");
    static_assert(!OK || NORM || OFF_ROWF + kRowfRing * C * 4 <= SMEM - 1024, "row factor ring inside allocation");
};

struct Params {
    const float* log_g;
    int decay_kind;
    const float* init_state;
    const float* init_z;
    __nv_bfloat16* out;
    float* final_state;
    float* final_z;
    // Dk and Dv are the tensors' widths.  The instance's key width DK is the
    // smallest one >= Dk: the key and query tiles' columns past Dk are the
    // TMA's zero fill, and the rows of S past Dk are neither read nor written
    // in global memory.  The value slices divide Dv exactly.
    int H, T, Dk, Dv, split, nchunks;
    int* err;
    // T-segments: each (b, h, slice) is cut into nseg segments of seg_chunks
    // chunks, one CTA each.  The output pass starts segment i from the state
    // after segment i - 1, combined from the workspace; the state pass
    // (state_pass = 1) only writes each segment's own contribution there.
    int nseg, seg_chunks, state_pass;
    float* ws_S;         // [B H][ws_nS][Dk][Dv] state of each state segment, from zero
    float* ws_z;         // [B H][ws_nS][Dk] key sum of each state segment, from zero
    float* ws_L;         // [B H][ws_nS] total log2 decay of each state segment
    int ws_nS;           // state segments per (b, h)
    int ws_per_seg;      // state segments per output segment
    // reverse scan (S_t = g_t S_{t+1} + k_t v_t^T): chunks are visited from
    // the last, and inside a chunk the decay runs from its last token; the
    // kernel works in scan order, mem_chunk maps it to memory.  The kernel
    // takes the direction from its REV template argument (the forward
    // instances carry no reverse-scan code); this field selects the instance.
    int reverse;
    int accumulate;      // reverse or 16-wide key instances: add y to the values in out (fp32 add)
    float q_scale;       // the output of an unnormalised scan is linear in q: y *= q_scale
                         // (the normalised output does not depend on the scale of q)
    int feature_map;     // LA_FEATURE_ELU1: the prep warps replace each landed Q and K tile
                         // by phi(x) = elu(x) + 1 before the chunk's first MMA (forward only)
    int pdl;             // (host) launch with programmatic stream serialisation
};

// What every role needs from the kernel prologue (passed by value).
struct Ctx {
    const Params* p;
    uint8_t* sm;
    uint32_t sa, tmem;
    int bh, h, j0, slice;
    int seg, c0, n;  // segment, its first chunk and its number of chunks
};

__device__ __forceinline__ void fail(const Params& p, volatile int* abort, int code) {
    *abort = 1;
    if (p.err) atomicCAS(p.err, 0, code);
}

constexpr uint32_t kSleepHintNs = 20000;  // longest single sleep inside a wait

// Slow paths of the bounded waits, kept out of line so that the hot loops stay
// small in the instruction cache.
static __device__ __noinline__ bool wait1_slow(uint64_t* bar, uint32_t parity, volatile int* abort, const Params& p,
                                        int code) {
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

static __device__ __noinline__ bool waitw_slow(uint64_t* bar, uint32_t parity, volatile int* abort, const Params& p,
                                        int code, bool ok) {
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

// Single-thread bounded wait; sleeps in the barrier between checks.
__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t parity, volatile int* abort, const Params& p,
                                      int code) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait1_slow(bar, parity, abort, p, code);
}

// Whole-warp bounded wait; every lane gets the same answer.
__device__ __forceinline__ bool waitw(uint64_t* bar, uint32_t parity, volatile int* abort, const Params& p,
                                      int code) {
    const bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    return waitw_slow(bar, parity, abort, p, code, ok);
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
// W: bytes per swizzled panel row (the tile's layout; by default the widest
// swizzle for WIDTH columns).
template <int WIDTH, int W = row_bytes_for(WIDTH)>
__device__ __forceinline__ void scale_row(uint8_t* tile, int row, float f) {
    constexpr int NP = WIDTH * 2 / W, NCH = NP * W / 16;
    constexpr int BATCH = NCH < 4 ? NCH : 4;  // loads in flight before the first store
    // f = f_hi + f_lo (two bf16 parts): fma(v, f_hi, v f_lo) rounds once, so the
    // result is the bf16 rounding of v f up to about 2^-17 relative
    const float fhi = __bfloat162float(__float2bfloat16_rn(f));
    const __nv_bfloat162 f2h = __float2bfloat162_rn(fhi), f2l = __float2bfloat162_rn(f - fhi);
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
            for (int e = 0; e < 4; ++e) hv[e] = __hfma2(hv[e], f2h, __hmul2(hv[e], f2l));
            *reinterpret_cast<uint4*>(tile + (ci / (W / 16)) * C * W + swz(row, (ci % (W / 16)) * 16, W)) = w[i];
        }
    }
}

// Byte offset of 16-element K step kk in a K-major tile (rows of W bytes).
__host__ __device__ constexpr uint32_t kstep(int kk, int W) {
    return ((kk * 16) / (W / 2)) * C * W + ((kk * 16) % (W / 2)) * 2;
}

// Store 16 outputs o * inv as bf16 (32 bytes) at dst: one 32-byte store when
// the output is 32-byte aligned, else two 16-byte stores. With acc the bf16
// values already at dst are added first (in fp32, one rounding to bf16).
__device__ __forceinline__ void store_row16(__nv_bfloat16* dst, const float (&o)[16], float inv, bool wide,
                                            bool acc) {
    uint32_t u[8];
    if (acc) {
        const uint4* s4 = reinterpret_cast<const uint4*>(dst);
        const uint4 h0 = s4[0], h1 = s4[1];
        const uint32_t old[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&old[e]));
            u[e] = pack2(fmaf(o[2 * e], inv, f.x), fmaf(o[2 * e + 1], inv, f.y));
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) u[e] = pack2(o[2 * e] * inv, o[2 * e + 1] * inv);
    }
    if (wide) {
        st_global_v8(dst, u);
    } else {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
        d4[0] = make_uint4(u[0], u[1], u[2], u[3]);
        d4[1] = make_uint4(u[4], u[5], u[6], u[7]);
    }
}

// phi(x) = elu(x) + 1 = max(x, 0) + e^min(x, 0) (flash-linear-attention
// issue 268's feature map) on two bf16 values, in bf16x2 arithmetic: the
// exponential is the tensor-core tile's own precision (ex2.approx on a bf16
// pair, its argument min(x, 0) log2(e) rounded to bf16), within a few bf16
// rounding steps of phi computed in fp32 and then rounded; for x > 0 it is
// exactly the bf16 rounding of x + 1.
__device__ __forceinline__ uint32_t elu1_pair(uint32_t u) {
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&u);
    const __nv_bfloat162 zero = __float2bfloat162_rn(0.f), log2e = __float2bfloat162_rn(kLog2e);
    const __nv_bfloat162 arg = __hmul2(__hmin2(x, zero), log2e);
    uint32_t e;
    asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(e) : "r"(*reinterpret_cast<const uint32_t*>(&arg)));
    const __nv_bfloat162 r = __hadd2(__hmax2(x, zero), *reinterpret_cast<const __nv_bfloat162*>(&e));
    return *reinterpret_cast<const uint32_t*>(&r);
}

// phi on row `row` of a landed [C x DK] Q or K tile (DK / (W / 2) swizzled
// panels of C rows of W bytes), in place; the columns at or past dk (the
// TMA's zero fill of a padded key width) stay zero, since phi(0) = 1.  One
// thread per row, so that the direct-form row scaling of the same thread
// follows it without a barrier.
template <int DK>
__device__ __noinline__ void elu1_row(uint8_t* tile, int row, int dk) {
    constexpr int W = row_bytes_for(DK), NP = DK * 2 / W, NCH = W / 16;
#pragma unroll
    for (int pn = 0; pn < NP; ++pn) {
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
            if (pn * (W / 2) + ch * 8 >= dk) continue;
            uint4* q = reinterpret_cast<uint4*>(tile + pn * C * W + swz(row, ch * 16, W));
            uint4 v = *q;
            v.x = elu1_pair(v.x);
            v.y = elu1_pair(v.y);
            v.z = elu1_pair(v.z);
            v.w = elu1_pair(v.w);
            *q = v;
        }
    }
}

// Ask L2 for the n bf16 values at p (the output row that an accumulating
// epilogue reads back one chunk later).
__device__ __forceinline__ void prefetch_row_l2(const __nv_bfloat16* p, int n) {
    for (int e = 0; e < n; e += 64) asm volatile("prefetch.global.L2 [%0];" ::"l"(p + e));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p + n - 1));
}

#define LA_ROLE_PRELUDE                                                                              \
    using G = Plan<DK, NV, NORM, SP>;                                                                \
    const Params& p = *x.p;                                                                          \
    uint8_t* const sm = x.sm;                                                                        \
    const uint32_t sa = x.sa, tmem = x.tmem;                                                         \
    uint64_t* const bar = reinterpret_cast<uint64_t*>(sm + G::OFF_MISC);                             \
    volatile int* const abort = reinterpret_cast<volatile int*>(sm + G::OFF_MISC + 8 * B_COUNT + 4); \
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;                                      \
    const int T = p.T, n = x.n;                                                                      \
    const auto mem_chunk = [&](int c) { /* memory chunk of the c-th chunk of this segment */         \
        return REV ? p.nchunks - 1 - (x.c0 + c) : x.c0 + c;                                          \
    };                                                                                               \
    (void)mem_chunk;                                                                                 \
    const bool accumulate = (REV || DK == 16) && p.accumulate != 0; /* reverse, or 16-wide keys */   \
    (void)accumulate;                                                                                \
    (void)sa;                                                                                        \
    (void)tmem;                                                                                      \
    (void)warp;                                                                                      \
    (void)T;                                                                                         \
    (void)lane;

// ------------------------------------------------------------ TMA producer
// Q, K and V rings: one thread polls all three, so that none waits behind
// another's free stage (the state pass reads no queries).  K and V run as
// far ahead as their rings allow: the prep of chunk c + 1 (which needs V)
// runs before the mask of chunk c.
template <int DK, int NV, bool NORM, bool REV, bool SP>
__device__ __noinline__ void role_tma(const Ctx x, const CUtensorMap* tmq, const CUtensorMap* tmk,
                                      const CUtensorMap* tmv) {
    LA_ROLE_PRELUDE
    if (lane != 0) return;
    const int nq = SP ? 0 : n;
    int cq = 0, ck = 0, cv = 0;
    uint64_t last = global_timer_ns();
    while (cq < nq || ck < n || cv < n) {
        bool moved = false;
        if (cq < nq && (cq < G::NQ || mbar_test(&bar[B_QEMPTY + cq % G::NQ], ((cq / G::NQ) - 1) & 1))) {
            const int s = cq % G::NQ;
            mbar_arrive_expect_tx(&bar[B_QFULL + s], G::Q_TX);
            uint8_t* st = sm + s * G::Q_STAGE;
            for (int pp = 0; pp < G::PK; ++pp)
                tma_load_3d(st + pp * C * G::WK, tmq, &bar[B_QFULL + s], pp * (G::WK / 2), mem_chunk(cq) * C, x.bh);
            ++cq;
            moved = true;
        }
        if (ck < n &&
            (ck < G::NK || mbar_test(&bar[B_KEMPTY + ck % G::NK], ((ck / G::NK) - 1) & 1))) {
            const int s = ck % G::NK;
            mbar_arrive_expect_tx(&bar[B_KFULL + s], G::Q_TX);
            uint8_t* st = sm + G::OFF_K + s * G::Q_STAGE;
            for (int pp = 0; pp < G::PK; ++pp)
                tma_load_3d(st + pp * C * G::WK, tmk, &bar[B_KFULL + s], pp * (G::WK / 2), mem_chunk(ck) * C, x.bh);
            ++ck;
            moved = true;
        }
        if (cv < n &&
            (cv < G::NVS || mbar_test(&bar[B_VEMPTY + cv % G::NVS], ((cv / G::NVS) - 1) & 1))) {
            const int s = cv % G::NVS;
            mbar_arrive_expect_tx(&bar[B_VFULL + s], G::V_TX);
            uint8_t* st = sm + G::OFF_V + s * G::V_STAGE;
            for (int pp = 0; pp < G::PV; ++pp)
                tma_load_3d(st + pp * C * G::WV, tmv, &bar[B_VFULL + s], x.j0 + pp * (G::WV / 2), mem_chunk(cv) * C,
                            x.bh);
            ++cv;
            moved = true;
        }
        if (moved) {
            last = global_timer_ns();
        } else {
            if (*abort) break;
            if (global_timer_ns() - last > kWaitLimitNs) {
                fail(p, abort, kErrTmaWait);
                break;
            }
            __nanosleep(kTmaIdleSleepNs);
        }
    }
    if (*abort) {  // let issued copies land before the CTA's shared memory goes away
        for (int c = cq > G::NQ ? cq - G::NQ : 0; c < cq; ++c)
            mbar_wait_bounded(&bar[B_QFULL + c % G::NQ], (c / G::NQ) & 1, kWaitLimitNs);
        for (int c = ck > G::NK ? ck - G::NK : 0; c < ck; ++c)
            mbar_wait_bounded(&bar[B_KFULL + c % G::NK], (c / G::NK) & 1, kWaitLimitNs);
        for (int c = cv > G::NVS ? cv - G::NVS : 0; c < cv; ++c)
            mbar_wait_bounded(&bar[B_VFULL + c % G::NVS], (c / G::NVS) & 1, kWaitLimitNs);
    }
}

// ------------------------------------------------------------ MMA issuers
// Two warps issue the MMAs, one elected lane each, so that neither queue
// waits behind the other's blocked issue:
//   warp A (W_MMA):  Q K^T (c)  Q and K tiles of c landed (and mapped), its
//                               score buffer free
//                    K^T V' (c) after Q K^T (c) and the prep of c; a
//                               direct-form chunk also after its mask, which
//                               decays Q and K; K^T V' buffer free;
//                               releases the K stage
//   warp B (W_MMAB): Q S (c)    Q tile of c landed (and mapped); the prep of
//                               c done, and the mask too for a direct-form
//                               chunk (it decays the Q tile); O buffer free;
//                               bf16 state after c - 1 written
//                    P V (c)    after Q S (c), which opened the accumulator;
//                               P (c) written
// A Q stage is free once Q K^T (warp A) and Q S (warp B) of its chunk have
// run: two commits.  Each warp polls its barriers (a snapshot per pass) and
// gives up after kWaitLimitNs without progress.
// State pass: warp A issues K^T V' (and K^T W) in order; each also releases
// its K and V stages.
template <int DK, int NV, bool NORM, bool REV, bool SP>
__device__ __noinline__ void mma_state_pass(const Ctx x) {
    LA_ROLE_PRELUDE
    const bool leader = elect_one();
    for (int kv = 0; kv < n; ++kv) {
        const int b = kv % G::NDS;
        if (!waitw(&bar[B_KFULL + kv % G::NK], (kv / G::NK) & 1, abort, p, kErrMmaWait)) break;
        if (!waitw(&bar[B_PREP + kv % G::NVS], (kv / G::NVS) & 1, abort, p, kErrMmaWait)) break;
        if (kv >= G::NDS && !waitw(&bar[B_DSEMPTY + b], ((kv / G::NDS) - 1) & 1, abort, p, kErrMmaWait)) break;
        tc_fence_after_sync();
        const uint32_t ka = sa + G::OFF_K + (kv % G::NK) * G::Q_STAGE;
        const uint32_t va = sa + G::OFF_V + (kv % G::NVS) * G::V_STAGE;
        const uint64_t dk = make_smem_desc(ka, DK == 128 ? C * G::WK : 0, 8 * G::WK, G::WK);
        const uint64_t dv = make_smem_desc(va, C * G::WV, 8 * G::WV, G::WV);
        const uint32_t d = tmem + G::COL_DS0 + b * G::OCOLS;
        if (leader) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(d, dk + ((kk * 16 * G::WK) >> 4), dv + ((kk * 16 * G::WV) >> 4), G::IDESC_KV, kk > 0);
            umma_commit(&bar[B_DSFULL + b]);
            umma_commit(&bar[B_KEMPTY + kv % G::NK]);
            umma_commit(&bar[B_VEMPTY + kv % G::NVS]);
        }
        __syncwarp();
    }
    if (leader) umma_commit(&bar[B_DRAIN]);
    __syncwarp();
    mbar_wait_bounded(&bar[B_DRAIN], 0, kWaitLimitNs);
}

// One pass without progress: give up after kWaitLimitNs (or on abort);
// returns false when the issuer should stop.
__device__ __forceinline__ bool idle_pass(bool moved, uint64_t& idle_since, volatile int* abort, const Params& p) {
    if (moved) {
        idle_since = 0;
        return true;
    }
    const uint64_t now = global_timer_ns();
    if (idle_since == 0) idle_since = now;
    bool give_up = *abort != 0;
    if (!give_up && now - idle_since > kWaitLimitNs) {
        give_up = true;
        if ((threadIdx.x & 31) == 0) fail(p, abort, kErrMmaWait);
    }
    if (__any_sync(0xffffffffu, give_up)) return false;
    __nanosleep(64);
    return true;
}

template <int DK, int NV, bool NORM, bool REV, bool PHI, bool SP>
__device__ __noinline__ void role_mma_a(const Ctx x) {
    LA_ROLE_PRELUDE
    if constexpr (SP) {
        mma_state_pass<DK, NV, NORM, REV, SP>(x);
        return;
    }
    const bool leader = elect_one();
    const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
    auto mode_of = [&](int j) {
        return *reinterpret_cast<volatile int*>(sm + G::OFF_V + (j % G::NVS) * G::V_STAGE + G::VS_META + 4);
    };
    int m1 = 0, kv = 0, pseen = 0;  // next Q K^T, next K^T V'; P (j) seen for j < pseen
    enum : uint32_t { kP = 1, kQ = 2, kK = 4, kA = 8, kPrep = 16, kDir = 32, kDse = 64, kPhi = 128 };
    auto snapshot = [&]() -> uint32_t {
        uint32_t b = 0;
        if (leader) {
            b |= mbar_test(&bar[B_PFULL + pseen % G::NPB], (pseen / G::NPB) & 1) ? kP : 0u;
            b |= mbar_test(&bar[B_QFULL + m1 % G::NQ], (m1 / G::NQ) & 1) ? kQ : 0u;
            b |= mbar_test(&bar[B_KFULL + m1 % G::NK], (m1 / G::NK) & 1) ? kK : 0u;
            b |= (m1 < G::NA || mbar_test(&bar[B_AEMPTY + m1 % G::NA], ((m1 / G::NA) - 1) & 1)) ? kA : 0u;
            if (PHI) b |= mbar_test(&bar[B_PHI + m1 % 4], (m1 / 4) & 1) ? kPhi : 0u;
            b |= mbar_test(&bar[B_PREP + kv % G::NVS], (kv / G::NVS) & 1) ? kPrep : 0u;
            b |= (kv < G::NDS || mbar_test(&bar[B_DSEMPTY + kv % G::NDS], ((kv / G::NDS) - 1) & 1)) ? kDse : 0u;
            if ((b & kPrep) && mode_of(kv) == kModeDirect) b |= kDir;  // the mode is valid once prep is done
        }
        return __shfl_sync(0xffffffffu, b, leader_lane);
    };
    uint64_t idle_since = 0;
    while (kv < n) {
        bool moved = false;
        const uint32_t bits = snapshot();
        if (pseen < m1 && (bits & kP)) {
            ++pseen;
            moved = true;
        }
        const bool kv_ok = kv < m1 && (bits & kPrep) && (!(bits & kDir) || kv < pseen) && (bits & kDse);
        const bool qk_ok = m1 < n && (bits & kQ) && (bits & kK) && (bits & kA) && (!PHI || (bits & kPhi));
        if (qk_ok) {
            tc_fence_after_sync();
            const uint64_t dq = make_smem_desc(sa + (m1 % G::NQ) * G::Q_STAGE, 16, 8 * G::WK, G::WK);
            const uint64_t dk = make_smem_desc(sa + G::OFF_K + (m1 % G::NK) * G::Q_STAGE, 16, 8 * G::WK, G::WK);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    umma_bf16(tmem + 128 * (m1 % G::NA), dq + (kstep(kk, G::WK) >> 4), dk + (kstep(kk, G::WK) >> 4),
                              G::IDESC_QK, kk > 0);
                umma_commit(&bar[B_AFULL + m1 % G::NA]);
                umma_commit(&bar[B_QEMPTY + m1 % G::NQ]);  // one of the Q stage's two releases
            }
            __syncwarp();
            ++m1;
            moved = true;
        } else if (kv_ok) {
            // DS = K^T V' (and K^T W); M = 128 key rows, a zero panel offset
            // repeats the key panel when Dk < 128
            tc_fence_after_sync();
            const int b = kv % G::NDS;
            const uint64_t dk =
                make_smem_desc(sa + G::OFF_K + (kv % G::NK) * G::Q_STAGE, DK == 128 ? C * G::WK : 0, 8 * G::WK, G::WK);
            const uint64_t dv = make_smem_desc(sa + G::OFF_V + (kv % G::NVS) * G::V_STAGE, C * G::WV, 8 * G::WV, G::WV);
            const uint32_t d = tmem + G::COL_DS0 + b * G::OCOLS;
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    umma_bf16(d, dk + ((kk * 16 * G::WK) >> 4), dv + ((kk * 16 * G::WV) >> 4), G::IDESC_KV, kk > 0);
                umma_commit(&bar[B_DSFULL + b]);
                umma_commit(&bar[B_KEMPTY + kv % G::NK]);  // Q K^T and K^T V' of this chunk have run
            }
            __syncwarp();
            ++kv;
            moved = true;
        }
        if (!idle_pass(moved, idle_since, abort, p)) break;
    }
    // everything issued has completed before TMEM is released
    if (leader) umma_commit(&bar[B_DRAIN]);
    __syncwarp();
    mbar_wait_bounded(&bar[B_DRAIN], 0, kWaitLimitNs);
}

template <int DK, int NV, bool NORM, bool REV, bool PHI, bool SP>
__device__ __noinline__ void role_mma_b(const Ctx x) {
    LA_ROLE_PRELUDE
    if constexpr (SP) return;  // no queries, no outputs
    const bool leader = elect_one();
    const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
    auto mode_of = [&](int j) {
        return *reinterpret_cast<volatile int*>(sm + G::OFF_V + (j % G::NVS) * G::V_STAGE + G::VS_META + 4);
    };
    int qs = 0, pv = 0, pseen = 0;  // next Q S, next P V; P (j) seen for j < pseen
    enum : uint32_t { kP = 1, kQ = 2, kPhi = 4, kPrep = 8, kDir = 16, kOe = 32, kSb = 64 };
    auto snapshot = [&]() -> uint32_t {
        uint32_t b = 0;
        if (leader) {
            b |= mbar_test(&bar[B_PFULL + pseen % G::NPB], (pseen / G::NPB) & 1) ? kP : 0u;
            b |= mbar_test(&bar[B_QFULL + qs % G::NQ], (qs / G::NQ) & 1) ? kQ : 0u;
            if (PHI) b |= mbar_test(&bar[B_PHI + qs % 4], (qs / 4) & 1) ? kPhi : 0u;
            b |= mbar_test(&bar[B_PREP + qs % G::NVS], (qs / G::NVS) & 1) ? kPrep : 0u;
            b |= (qs < G::NO || mbar_test(&bar[B_OEMPTY + qs % G::NO], ((qs / G::NO) - 1) & 1)) ? kOe : 0u;
            b |= mbar_test(&bar[B_SBFULL + qs % G::NSB], (qs / G::NSB) & 1) ? kSb : 0u;
            if ((b & kPrep) && mode_of(qs) == kModeDirect) b |= kDir;
        }
        return __shfl_sync(0xffffffffu, b, leader_lane);
    };
    uint64_t idle_since = 0;
    while (pv < n) {
        bool moved = false;
        const uint32_t bits = snapshot();
        // masks are in order, so P (pseen) is tested only after P (pseen - 1)
        if (pseen < n && (bits & kP)) {
            ++pseen;
            moved = true;
        }
        const bool pv_ok = pv < qs && pv < pseen;
        const bool qs_ok = qs < n && (bits & kQ) && (!PHI || (bits & kPhi)) && (bits & kPrep) &&
                           (!(bits & kDir) || qs < pseen) && (bits & kOe) && (bits & kSb);
        if (pv_ok) {
            // P V (and P W) accumulate into the O that Q S opened
            tc_fence_after_sync();
            const int pb = pv % G::NPB, ro = pv % G::NO;
            const uint64_t dv = make_smem_desc(sa + G::OFF_V + (pv % G::NVS) * G::V_STAGE, C * G::WV, 8 * G::WV, G::WV);
            const uint32_t pa = tmem + G::COL_P0 + 64 * pb;
            const uint32_t d = tmem + G::COL_O0 + ro * G::OCOLS;
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    umma_bf16_ts(d, pa + 8 * kk, dv + ((kk * 16 * G::WV) >> 4), G::IDESC_PV, 1);
                umma_commit(&bar[B_OFULL + ro]);
                umma_commit(&bar[B_PEMPTY + pb]);
                umma_commit(&bar[B_VEMPTY + pv % G::NVS]);
            }
            __syncwarp();
            ++pv;
            moved = true;
        } else if (qs_ok) {
            // O = Q S (and den = Q z), opening the accumulator of chunk qs
            tc_fence_after_sync();
            const int ro = qs % G::NO, sbb = qs % G::NSB;
            const uint64_t dq = make_smem_desc(sa + (qs % G::NQ) * G::Q_STAGE, 16, 8 * G::WK, G::WK);
            // B = [S | z] panels of the bf16 state copy
            const uint64_t dsb = make_smem_desc(sa + G::OFF_SB + sbb * G::SB_BYTES, DK * G::WV, 8 * G::WV, G::WV);
            const uint32_t d = tmem + G::COL_O0 + ro * G::OCOLS;
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    umma_bf16(d, dq + (kstep(kk, G::WK) >> 4), dsb + ((kk * 16 * G::WV) >> 4), G::IDESC_PV, kk > 0);
                umma_commit(&bar[B_QEMPTY + qs % G::NQ]);  // the Q stage's other release
                umma_commit(&bar[B_SBEMPTY + sbb]);
            }
            __syncwarp();
            ++qs;
            moved = true;
        }
        if (!idle_pass(moved, idle_since, abort, p)) break;
    }
    if (leader) umma_commit(&bar[B_DRAINB]);
    __syncwarp();
    mbar_wait_bounded(&bar[B_DRAINB], 0, kWaitLimitNs);
}

// ------------------------------------------------------------ prep + mask
// Mask of a direct-form chunk (total decay beyond the fold limit), out of line
// because it is rare: P = mask(A) * 2^(L_t - L_s), written as bf16 pairs at
// p_addr; then this thread's row of the chunk's Q tile (warpgroup 0) or K tile
// (warpgroup 1), given as `tile`, is decayed in place for its Q S and K^T V.
template <int DK>
__device__ __noinline__ void mask_direct(uint32_t s_addr, uint32_t p_addr, uint64_t* aempty, int wg, int t,
                                         bool all_masked, float lt, float lc, const float* lam, uint8_t* tile,
                                         bool rev) {
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        float a0[16], a1[16];
        if (!all_masked) {
            tmem_ld16(s_addr + 32 * half, a0);
            tmem_ld16(s_addr + 32 * half + 16, a1);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) a0[e] = a1[e] = 0.f;
        }
        if (half == 1) {
            tc_fence_before_sync();
            warp_arrive(aempty);
        }
        const int base = 64 * wg + 32 * half;
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int s0 = base + 2 * e;
            // kept: s <= t (forward) or s >= t (reverse scan)
            const float f0 = (rev ? s0 >= t : s0 <= t) ? a0[2 * e] * ex2_approx(lt - lam[s0]) : 0.f;
            const float f1 = (rev ? s0 + 1 >= t : s0 + 1 <= t) ? a0[2 * e + 1] * ex2_approx(lt - lam[s0 + 1]) : 0.f;
            const float f2 = (rev ? s0 + 16 >= t : s0 + 16 <= t) ? a1[2 * e] * ex2_approx(lt - lam[s0 + 16]) : 0.f;
            const float f3 = (rev ? s0 + 17 >= t : s0 + 17 <= t) ? a1[2 * e + 1] * ex2_approx(lt - lam[s0 + 17]) : 0.f;
            u[e] = pack2(f0, f1);
            u[8 + e] = pack2(f2, f3);
        }
        tmem_st16u(p_addr + 16 * half, u);
    }
    tmem_wait_st();
    scale_row<DK>(tile, t, ex2_approx(wg == 0 ? lt : lc - lt));
    fence_async_smem();
}

template <int DK, int NV, bool NORM, bool REV, bool PHI, bool SP>
__device__ __noinline__ void role_prep_mask(const Ctx x) {
    LA_ROLE_PRELUDE
    const int wg = (warp - G::W_PM) / 4;  // 0: score columns 0-63, V rows; 1: columns 64-127, weights
    const int wq = warp & 3;
    const int t = 32 * wq + lane;        // TMEM lane = token row
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * wq) << 16);
    const int kind = p.decay_kind;
    const float* lg = p.log_g + static_cast<size_t>(x.bh) * T;
    const float ell_head = kind == LA_DECAY_PER_HEAD ? p.log_g[x.h] * kLog2e : 0.f;
    // per-step decays: lane l holds rows 4 l .. 4 l + 3 of the chunk (every
    // warp of warpgroup 0 holds the whole chunk)
    float nxt[4] = {0.f, 0.f, 0.f, 0.f};
    auto fetch = [&](int c) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = mem_chunk(c) * C + 4 * lane + i;
            nxt[i] = (kind == LA_DECAY_PER_STEP && c < n && row < T) ? lg[row] : 0.f;
        }
    };
    if (wg == 0 || NORM) fetch(0);

    // Warpgroup 0 computes the chunk's decay prefix, writes it (and the
    // mode) into the V stage, the output row factors and the scaled value
    // rows; warpgroup 1 writes the normaliser weights, or has nothing to do.
    auto prep = [&](int c) -> bool {
        const int s = c % G::NVS, rem = min(C, T - mem_chunk(c) * C);
        if (PHI && SP && wg == 0) {
            // the state pass has no Q tile and no mask: warpgroup 0 maps the
            // chunk's key rows here (before it decays them, for a direct-form
            // chunk), before the prep arrival that the chunk's K^T V' awaits
            if (!waitw(&bar[B_KFULL + c % G::NK], (c / G::NK) & 1, abort, p, kErrTmaWait)) return false;
            if (t < rem) elu1_row<DK>(sm + G::OFF_K + (c % G::NK) * G::Q_STAGE, t, p.Dk);
            fence_async_smem();
        }
        if (!NORM && wg == 1) {
            // nothing to prepare; in the state pass (no mask to pace this
            // warpgroup) wait for the tile so that its arrivals never run a
            // ring's length ahead
            if (SP && !waitw(&bar[B_VFULL + s], (c / G::NVS) & 1, abort, p, kErrTmaWait)) return false;
            warp_arrive(&bar[B_PREP + s]);
            return true;
        }
        const float cur0 = nxt[0], cur1 = nxt[1], cur2 = nxt[2], cur3 = nxt[3];
        fetch(c + 1);
        if (!waitw(&bar[B_VFULL + s], (c / G::NVS) & 1, abort, p, kErrTmaWait)) return false;
        // chunk-local log2 decay prefix L_t and total L_C
        float lt, lc;
        if (kind == LA_DECAY_PER_STEP) {
            // prefix of the lane's four rows, an exclusive warp scan of the
            // lane totals, then each lane of this warp's 32 rows publishes
            // its four prefixes (rows 32 wq .. 32 wq + 31) and reads its own
            const float a0 = cur0 * kLog2e, a1 = a0 + cur1 * kLog2e, a2 = a1 + cur2 * kLog2e,
                        a3 = a2 + cur3 * kLog2e;
            float incl = a3;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const float excl = incl - a3;
            lc = __shfl_sync(0xffffffffu, incl, 31);
            float* lam = reinterpret_cast<float*>(sm + G::OFF_V + s * G::V_STAGE + G::VS_LAM);
            if ((lane >> 3) == wq) {
                // forward: inclusive prefix of the row; reverse: inclusive
                // suffix (the chunk total minus the exclusive prefix)
                const float4 pre = REV
                                       ? make_float4(lc - excl, lc - excl - a0, lc - excl - a1, lc - excl - a2)
                                       : make_float4(excl + a0, excl + a1, excl + a2, excl + a3);
                *reinterpret_cast<float4*>(lam + 4 * lane) = pre;
            }
            __syncwarp();
            lt = lam[t];
        } else {  // per head (ell_head = L per step), or none (ell_head = 0)
            lt = static_cast<float>(REV ? max(rem - t, 0) : min(t + 1, rem)) * ell_head;
            lc = static_cast<float>(rem) * ell_head;
        }
        const int md = kind == LA_DECAY_NONE ? kModeNone : (-lc <= kFoldLimit ? kModeFolded : kModeDirect);
        uint8_t* st = sm + G::OFF_V + s * G::V_STAGE;
        if (wg == 0) {
            reinterpret_cast<float*>(st + G::VS_LAM)[t] = lt;
            if (t == 0) {
                *reinterpret_cast<float*>(st + G::VS_META) = lc;
                *reinterpret_cast<int*>(st + G::VS_META + 4) = md;
            }
            // output row factor 2^(L_t) of the folded form (1 otherwise); the
            // normalised output does not need it (and has no ring for it)
            if (!NORM)
                reinterpret_cast<float*>(sm + G::OFF_ROWF)[(c % G::kRowfRing) * C + t] =
                    md == kModeFolded ? ex2_approx(lt) : 1.f;
            if (md == kModeFolded) scale_row<NV, G::WV>(st, t, ex2_approx(-lt));
            if (md == kModeDirect && SP) {
                // no mask in the state pass: decay this key row here, K~ = 2^(L_C - L_t) K
                if (!waitw(&bar[B_KFULL + c % G::NK], (c / G::NK) & 1, abort, p, kErrTmaWait)) return false;
                scale_row<DK>(sm + G::OFF_K + (c % G::NK) * G::Q_STAGE, t, ex2_approx(lc - lt));
            }
        } else if (NORM) {
            // normaliser weights w_t = 2^(-L_t) (1 unless folded), as a bf16 hi/lo pair
            const float w = md == kModeFolded ? ex2_approx(-lt) : 1.f;
            const float hi = __bfloat162float(__float2bfloat16_rn(w));
            *reinterpret_cast<uint4*>(st + G::VS_W + swz(t, 0, 32)) = make_uint4(pack2(hi, w - hi), 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(st + G::VS_W + swz(t, 16, 32)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
        warp_arrive(&bar[B_PREP + s]);
        return true;
    };

    auto pmask = [&](int c) -> bool {
        const int s = c % G::NVS, pb = c % G::NPB;
        if (c >= G::NPB && !waitw(&bar[B_PEMPTY + pb], ((c / G::NPB) - 1) & 1, abort, p, kErrMmaWait))
            return false;
        const int ab = c % G::NA;  // score buffer
        if (!waitw(&bar[B_AFULL + ab], (c / G::NA) & 1, abort, p, kErrMmaWait)) return false;
        if (!waitw(&bar[B_PREP + s], (c / G::NVS) & 1, abort, p, kErrMmaWait)) return false;
        tc_fence_after_sync();
        const uint8_t* st = sm + G::OFF_V + s * G::V_STAGE;
        const int md = *reinterpret_cast<const volatile int*>(st + G::VS_META + 4);
        const uint32_t p_addr = lane_addr + G::COL_P0 + 64 * pb + 32 * wg;  // packed pairs of score columns
        if (md == kModeDirect) {
            const float* lam = reinterpret_cast<const float*>(st + G::VS_LAM);
            const float lc = *reinterpret_cast<const volatile float*>(st + G::VS_META);
            // every row of this warp precedes (reverse: follows) these columns
            const bool all_masked = REV ? 32 * wq > 64 * wg + 63 : (32 * wq + 31) < 64 * wg;
            mask_direct<DK>(lane_addr + 128 * ab + 64 * wg, p_addr, &bar[B_AEMPTY + ab], wg, t, all_masked, lam[t], lc, lam,
                            wg == 0 ? sm + (c % G::NQ) * G::Q_STAGE : sm + G::OFF_K + (c % G::NK) * G::Q_STAGE,
                            REV);
        } else {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                // 32 x 32 block (row block wq, column block cb) of the scores:
                // above the diagonal all zero, below it copied, on it masked
                // (the reverse scan keeps the upper triangle instead)
                const int cb = 2 * wg + half;
                constexpr bool rev = REV;
                uint32_t u[16];
                if (rev ? cb < wq : cb > wq) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) u[e] = 0u;
                } else {
                    float a0[16], a1[16];
                    tmem_ld16(lane_addr + 128 * ab + 32 * cb, a0);
                    tmem_ld16(lane_addr + 128 * ab + 32 * cb + 16, a1);
                    tmem_wait_ld();
                    if (rev ? cb > wq : cb < wq) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            u[e] = pack2(a0[2 * e], a0[2 * e + 1]);
                            u[8 + e] = pack2(a1[2 * e], a1[2 * e + 1]);
                        }
                    } else if (!rev) {
                        const int r = lane;  // column s0 of the block is kept when s0 <= r
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            u[e] = pack2(2 * e <= r ? a0[2 * e] : 0.f, 2 * e + 1 <= r ? a0[2 * e + 1] : 0.f);
                            u[8 + e] = pack2(2 * e + 16 <= r ? a1[2 * e] : 0.f, 2 * e + 17 <= r ? a1[2 * e + 1] : 0.f);
                        }
                    } else {
                        const int r = lane;  // column s0 of the block is kept when s0 >= r
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            u[e] = pack2(2 * e >= r ? a0[2 * e] : 0.f, 2 * e + 1 >= r ? a0[2 * e + 1] : 0.f);
                            u[8 + e] = pack2(2 * e + 16 >= r ? a1[2 * e] : 0.f, 2 * e + 17 >= r ? a1[2 * e + 1] : 0.f);
                        }
                    }
                }
                if (half == 1) {  // the score buffer is free for a later Q K^T
                    tc_fence_before_sync();
                    warp_arrive(&bar[B_AEMPTY + ab]);
                }
                tmem_st16u(p_addr + 16 * half, u);
            }
            tmem_wait_st();
        }
        tc_fence_before_sync();
        warp_arrive(&bar[B_PFULL + pb]);
        warp_arrive(&bar[B_VEMPTY + s]);
        return true;
    };

    // Epilogue (warpgroup 1, after its mask of the next chunk): y = O times
    // the row factor 2^(L_t) (or / den_t) for all NV columns of the slice;
    // 16-byte stores of bf16 pairs, rows past the sequence end skipped.
    auto out_row = [&](int c) {
        return p.out + (static_cast<size_t>(x.bh) * T + static_cast<size_t>(mem_chunk(c)) * C + t) * p.Dv + x.j0;
    };
    auto epilogue = [&](int c) -> bool {
        const int ro = c % G::NO;
        if (accumulate) {  // the rows this epilogue and the next read back
            if (c == 0 && t < min(C, T - mem_chunk(0) * C)) prefetch_row_l2(out_row(0), NV);
            if (c + 1 < n && t < min(C, T - mem_chunk(c + 1) * C)) prefetch_row_l2(out_row(c + 1), NV);
        }
        if (!waitw(&bar[B_OFULL + ro], (c / G::NO) & 1, abort, p, kErrMmaWait)) return false;
        tc_fence_after_sync();
        const uint32_t oa = lane_addr + G::COL_O0 + ro * G::OCOLS;
        float inv;  // y = O * inv
        if (NORM) {
            float dd[16];
            tmem_ld16(oa + NV, dd);
            tmem_wait_ld();
            inv = 1.f / (dd[0] + dd[1]);
        } else {
            inv = reinterpret_cast<const float*>(sm + G::OFF_ROWF)[(c % G::kRowfRing) * C + t] * p.q_scale;
        }
        const int rem = min(C, T - mem_chunk(c) * C);
        const bool wide = (reinterpret_cast<uintptr_t>(p.out) & 31) == 0;  // 32-byte stores allowed
        __nv_bfloat16* dst = out_row(c);
#pragma unroll 1
        for (int piece = 0; piece < NV / 16; ++piece) {
            float o[16];
            tmem_ld16(oa + 16 * piece, o);
            tmem_wait_ld();
            if (t < rem) store_row16(dst + 16 * piece, o, inv, wide, accumulate);
        }
        tc_fence_before_sync();
        warp_arrive(&bar[B_OEMPTY + ro]);
        return true;
    };
    if constexpr (SP) {  // prep only; nothing reads the V stage's prefix later
#pragma unroll 1
        for (int c = 0; c < n; ++c) {
            if (!prep(c)) break;
            warp_arrive(&bar[B_VEMPTY + c % G::NVS]);
        }
        return;
    }
    // Feature map (output pass): warpgroup 0 maps the chunk's Q tile and
    // warpgroup 1 its K tile, one row per thread, rows past the sequence end
    // left at the TMA's zero fill (phi(0) = 1 would add them to the key
    // sum); the chunk's Q K^T awaits the arrival.
    auto phi = [&](int c) -> bool {
        const int rem = min(C, T - mem_chunk(c) * C);
        if (wg == 0) {
            if (!waitw(&bar[B_QFULL + c % G::NQ], (c / G::NQ) & 1, abort, p, kErrTmaWait)) return false;
            if (t < rem) elu1_row<DK>(sm + (c % G::NQ) * G::Q_STAGE, t, p.Dk);
        } else {
            if (!waitw(&bar[B_KFULL + c % G::NK], (c / G::NK) & 1, abort, p, kErrTmaWait)) return false;
            if (t < rem) elu1_row<DK>(sm + G::OFF_K + (c % G::NK) * G::Q_STAGE, t, p.Dk);
        }
        fence_async_smem();
        warp_arrive(&bar[B_PHI + c % 4]);
        return true;
    };
    constexpr bool map = PHI;
    // prep runs one chunk ahead of the mask, the epilogue one chunk behind
    // it, and the feature map of the next chunk right after the mask (off the
    // path from a chunk's scores to its mask); one call site each keeps the
    // loop small in the instruction cache
#pragma unroll 1
    for (int c = -1; c <= n; ++c) {
        if (c + 1 < n && !prep(c + 1)) break;
        if (c >= 0 && c < n && !pmask(c)) break;
        if (map && c + 1 < n && !phi(c + 1)) break;
        if (wg == 1 && c >= 1 && !epilogue(c - 1)) break;
    }
}

// ------------------------------------------------------------ state
// Warpgroup wg owns value columns [wg NVW, (wg + 1) NVW) of the slice.  Per
// chunk c: the state update of chunk c, then its bf16 copy, which the next
// chunk's Q S reads.
template <int DK, int NV, bool NORM, bool REV, bool SP>
__device__ __noinline__ void role_state(const Ctx x) {
    LA_ROLE_PRELUDE
    const int wg = (warp - G::W_ES) / 4;
    const int wq = warp & 3;
    const int d = 32 * wq + lane;          // key row of S; also token row t of O
    const bool warp_rows = 32 * wq < DK;   // this warp holds rows of S (past Dk they stay zero)
    // rows of S past Dk (a padded key width) are never read or written in
    // global memory; evaluated at each use (a long-lived predicate here costs
    // registers in the chunk loop)
    auto row_ok = [&]() { return d < p.Dk; };
    const int cb = wg * G::NVW;            // first column (within the slice) of this warpgroup
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * wq) << 16);
    const int bh = x.bh, j0 = x.j0;
    float S[G::NVW];
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < G::NVW; ++j) S[j] = 0.f;
    float ltot = 0.f;  // state pass: total log2 decay of the segment
    if (row_ok() && p.init_state && !SP) {
        const float* src = p.init_state + (static_cast<size_t>(bh) * p.Dk + d) * p.Dv + j0 + cb;
#pragma unroll
        for (int j = 0; j < G::NVW; j += 4) {
            const float4 v4 = *reinterpret_cast<const float4*>(src + j);
            S[j] = v4.x;
            S[j + 1] = v4.y;
            S[j + 2] = v4.z;
            S[j + 3] = v4.w;
        }
    }
    if (NORM && row_ok() && p.init_z && !SP) z = p.init_z[static_cast<size_t>(bh) * p.Dk + d];
    if (row_ok() && !SP && x.seg > 0) {
        // state entering this segment: fold in every earlier state segment j,
        // S <- 2^(L_j) S + S_j (the combination of two consecutive spans)
        for (int j = 0; j < x.seg * p.ws_per_seg; ++j) {
            const size_t sj = static_cast<size_t>(bh) * p.ws_nS + j;
            const float e = ex2_approx(p.ws_L[sj]);
            const float* src = p.ws_S + (sj * p.Dk + d) * p.Dv + j0 + cb;
#pragma unroll
            for (int i = 0; i < G::NVW; i += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(src + i);
                S[i] = fmaf(e, S[i], v4.x);
                S[i + 1] = fmaf(e, S[i + 1], v4.y);
                S[i + 2] = fmaf(e, S[i + 2], v4.z);
                S[i + 3] = fmaf(e, S[i + 3], v4.w);
            }
            if (NORM) z = fmaf(e, z, p.ws_z[sj * p.Dk + d]);
        }
    }

    auto write_copy = [&](int k) {  // bf16 copy of S (and z) for production index k
        const int buf = k % G::NSB;
        uint8_t* sb = sm + G::OFF_SB + buf * G::SB_BYTES;
        // every row of the tile, the zero rows past Dk included: Q S reads
        // them (against zero query columns, but whatever else sat in shared
        // memory there could be an infinity or a NaN)
        if (d < DK) {
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
                *reinterpret_cast<uint4*>(sb + G::SB_ZB + swz(d, 0, 32)) =
                    make_uint4(pack2(hi, z - hi), 0u, 0u, 0u);
            }
        }
        fence_async_smem();
        warp_arrive(&bar[B_SBFULL + buf]);
    };

    auto state = [&](int c) -> bool {
        const int s = c % G::NVS, b = c % G::NDS;
        if (!waitw(&bar[B_PREP + s], (c / G::NVS) & 1, abort, p, kErrMmaWait)) return false;
        const uint8_t* st = sm + G::OFF_V + s * G::V_STAGE;
        const float lc = *reinterpret_cast<const volatile float*>(st + G::VS_META);
        const int md = *reinterpret_cast<const volatile int*>(st + G::VS_META + 4);
        ltot += lc;
        if (!waitw(&bar[B_DSFULL + b], (c / G::NDS) & 1, abort, p, kErrMmaWait)) return false;
        tc_fence_after_sync();
        // S' = ca S + cb DS: folded 2^(L_C) (S + K^T V'), direct 2^(L_C) S + K~^T V, none S + K^T V
        const float e = md == kModeNone ? 1.f : ex2_approx(lc);
        const float ca = e, cbf = md == kModeFolded ? e : 1.f;
        const uint32_t dsa = lane_addr + G::COL_DS0 + b * G::OCOLS;
        if (warp_rows) {
#pragma unroll
            for (int j = 0; j < G::NVW; j += 16) {
                float ds[16];
                tmem_ld16(dsa + cb + j, ds);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) S[j + i] = fmaf(ca, S[j + i], cbf * ds[i]);
            }
            if (NORM && wg == 0) {
                float zz[16];
                tmem_ld16(dsa + NV, zz);
                tmem_wait_ld();
                z = fmaf(ca, z, cbf * (zz[0] + zz[1]));
            }
        }
        tc_fence_before_sync();
        warp_arrive(&bar[B_DSEMPTY + b]);
        warp_arrive(&bar[B_VEMPTY + s]);
        if (c == n - 1 || SP) return true;
        const int k = c + 1;
        if (k >= G::NSB && !waitw(&bar[B_SBEMPTY + k % G::NSB], ((k / G::NSB) - 1) & 1, abort, p, kErrMmaWait))
            return false;
        write_copy(k);
        return true;
    };

    if constexpr (SP) {
        bool ok = true;
#pragma unroll 1
        for (int c = 0; c < n && ok; ++c) ok = state(c);
        if (ok && !*abort) {
            const size_t sj = static_cast<size_t>(bh) * p.ws_nS + x.seg;
            if (row_ok()) {
                float* dst = p.ws_S + (sj * p.Dk + d) * p.Dv + j0 + cb;
#pragma unroll
                for (int j = 0; j < G::NVW; j += 4)
                    *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
                if (NORM && x.slice == 0 && wg == 0) p.ws_z[sj * p.Dk + d] = z;
            }
            if (x.slice == 0 && wg == 0 && d == 0) p.ws_L[sj] = ltot;
        }
        return;
    }

    write_copy(0);
    bool ok = true;
#pragma unroll 1
    for (int c = 0; c < n && ok; ++c) ok = state(c);
    if (ok && !*abort && row_ok() && x.seg == p.nseg - 1) {
        if (p.final_state) {
            float* fs = p.final_state + (static_cast<size_t>(bh) * p.Dk + d) * p.Dv + j0 + cb;
#pragma unroll
            for (int j = 0; j < G::NVW; j += 4)
                *reinterpret_cast<float4*>(fs + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        if (NORM && p.final_z && x.slice == 0 && wg == 0) p.final_z[static_cast<size_t>(bh) * p.Dk + d] = z;
    }
}

template <int DK, int NV, bool NORM, bool REV, bool PHI, bool SP>
__global__ void __launch_bounds__(Plan<DK, NV, NORM, SP>::THREADS, 1)
    fwd_ws_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ Params p) {
    using G = Plan<DK, NV, NORM, SP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sa = smem_u32(sm);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + G::OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + G::OFF_MISC + 8 * B_COUNT);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + G::OFF_MISC + 8 * B_COUNT + 4);

    const int tid = threadIdx.x, warp = tid / 32;
    // blockIdx.x = (bh * nseg + seg) * split + slice
    const int slice = blockIdx.x % p.split, bs = blockIdx.x / p.split;
    const int seg = bs % p.nseg, bh = bs / p.nseg;
    const int c0 = seg * p.seg_chunks;
    const int nloc = max(0, min(p.seg_chunks, p.nchunks - c0));

    if (tid == 0) {
        prefetch_tensormap(&tmq);
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bar[B_QFULL + s], 1);
            mbar_init(&bar[B_QEMPTY + s], 2);  // Q K^T (warp A) and Q S (warp B)
            mbar_init(&bar[B_KFULL + s], 1);
            mbar_init(&bar[B_KEMPTY + s], 1);
            mbar_init(&bar[B_VFULL + s], 1);
            mbar_init(&bar[B_VEMPTY + s], G::VEMPTY_ARRIVALS);
            mbar_init(&bar[B_PREP + s], 8);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[B_OFULL + i], 1);
            mbar_init(&bar[B_OEMPTY + i], 4);  // the epilogue warpgroup
            mbar_init(&bar[B_AFULL + i], 1);
            mbar_init(&bar[B_AEMPTY + i], 8);
            mbar_init(&bar[B_PFULL + i], 8);
            mbar_init(&bar[B_PEMPTY + i], 1);
            mbar_init(&bar[B_DSFULL + i], 1);
            mbar_init(&bar[B_DSEMPTY + i], 4 * G::NSW);
            mbar_init(&bar[B_SBFULL + i], 4 * G::NSW);
            mbar_init(&bar[B_SBEMPTY + i], 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&bar[B_PHI + i], 8);
        mbar_init(&bar[B_DRAIN], 1);
        mbar_init(&bar[B_DRAINB], 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == G::W_MMA) tmem_alloc(tmem_slot, G::TMEM_COLS);
    if (NORM && !SP && warp >= G::W_ES && warp < G::W_ES + 4) {
        // zeroed key-sum tiles (only their first two columns are ever written)
        for (int i = tid - 32 * G::W_ES; i < G::NSB * DK * 2; i += 128)  // 16-byte pieces
            reinterpret_cast<uint4*>(sm + G::OFF_SB + (i / (DK * 2)) * G::SB_BYTES + G::SB_ZB)[i % (DK * 2)] =
                make_uint4(0u, 0u, 0u, 0u);
        fence_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // The prologue above may overlap the previous kernel on the stream (the
    // launch allows programmatic serialisation); no global memory is read or
    // written before that kernel has completed.  Every CTA signals the next
    // launch only after its own wait, so a kernel two launches on still
    // starts after this one's predecessor has finished.
    grid_dependency_wait();
    grid_launch_dependents();

    const Ctx x{&p, sm, sa, tmem, bh, bh % p.H, slice * NV, slice, seg, c0, nloc};
    if (warp == G::W_MMAB) {
        role_mma_b<DK, NV, NORM, REV, PHI, SP>(x);
    } else if (warp == G::W_MMA) {
        role_mma_a<DK, NV, NORM, REV, PHI, SP>(x);
    } else if (warp < G::W_ES) {
        role_prep_mask<DK, NV, NORM, REV, PHI, SP>(x);
    } else if (warp < G::W_TMAV) {
        role_state<DK, NV, NORM, REV, SP>(x);
    } else {
        role_tma<DK, NV, NORM, REV, SP>(x, &tmq, &tmk, &tmv);
    }

    __syncwarp();  // lanes that idled while lane 0 ran a single-thread role rejoin it
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == G::W_MMA) tmem_dealloc(tmem, G::TMEM_COLS);
}

template <int DK, int NV, bool NORM, bool REV, bool PHI, bool SP>
cudaError_t launch_instance(const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                            const Params& p, int grid, cudaStream_t stream) {
    using G = Plan<DK, NV, NORM, SP>;
    if constexpr (!G::OK) {
        return cudaErrorNotSupported;
    } else {
        // at least 116 KB so that one CTA (512 TMEM columns) owns each SM
        const int smem = G::SMEM > 116 * 1024 ? G::SMEM : 116 * 1024;
        cudaError_t e =
            cudaFuncSetAttribute(fwd_ws_kernel<DK, NV, NORM, REV, PHI, SP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        // programmatic serialisation: this grid's prologue (barriers, TMEM,
        // descriptor prefetch) overlaps the tail of the previous kernel
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(G::THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = p.pdl ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, fwd_ws_kernel<DK, NV, NORM, REV, PHI, SP>, tmq, tmk, tmv, p);
    }
}

template <int DK, int NV>
constexpr bool supported(bool norm, bool sp) {
    return norm ? (sp ? Plan<DK, NV, true, true>::OK : Plan<DK, NV, true>::OK)
                : (sp ? Plan<DK, NV, false, true>::OK : Plan<DK, NV, false>::OK);
}

template <int DK, int NV, bool NORM, bool REV, bool PHI>
cudaError_t launch_pass(const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv, const Params& p,
                        int grid, cudaStream_t stream) {
    // a state pass runs its own instance (no Q ring, deeper K and V rings)
    return p.state_pass ? launch_instance<DK, NV, NORM, REV, PHI, true>(tmq, tmk, tmv, p, grid, stream)
                        : launch_instance<DK, NV, NORM, REV, PHI, false>(tmq, tmk, tmv, p, grid, stream);
}

// Dispatch on the value slice and the normaliser for one key width and one
// direction (and feature map); each instantiation file (la_fwd_ws_dk*.cu)
// instantiates these for its key width, so that the build compiles the
// widths in parallel.
template <int DK, bool REV, bool NORM, bool PHI>
cudaError_t launch_nv(int nv, const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                      const Params& p, int grid, cudaStream_t stream) {
    switch (nv) {
        case 16: return launch_pass<DK, 16, NORM, REV, PHI>(tmq, tmk, tmv, p, grid, stream);
        case 32: return launch_pass<DK, 32, NORM, REV, PHI>(tmq, tmk, tmv, p, grid, stream);
        case 64: return launch_pass<DK, 64, NORM, REV, PHI>(tmq, tmk, tmv, p, grid, stream);
        case 128: return launch_pass<DK, 128, NORM, REV, PHI>(tmq, tmk, tmv, p, grid, stream);
        default: return cudaErrorNotSupported;
    }
}

// PHI: the instances that apply the feature map to the Q and K tiles
// (forward scans only; the others carry none of its code).
template <int DK, bool REV, bool PHI>
cudaError_t launch_dk(int nv, bool norm, const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                      const Params& p, int grid, cudaStream_t stream) {
    static_assert(!(REV && PHI), "the feature map applies to forward scans");
    return norm ? launch_nv<DK, REV, true, PHI>(nv, tmq, tmk, tmv, p, grid, stream)
                : launch_nv<DK, REV, false, PHI>(nv, tmq, tmk, tmv, p, grid, stream);
}

// sp: the state-pass instance (its plan fits wider slices: no Q ring)
template <int DK>
bool supported_dk(int nv, bool norm, bool sp) {
    switch (nv) {
        case 16: return supported<DK, 16>(norm, sp);
        case 32: return supported<DK, 32>(norm, sp);
        case 64: return supported<DK, 64>(norm, sp);
        case 128: return supported<DK, 128>(norm, sp);
        default: return false;
    }
}

}  // namespace ws
}  // namespace la
