// la_fwd_tc.cu - host side of the tensor-core forward: tensor maps, the
// choice of how many CTAs share one (b, h), and dispatch to the
// warp-specialised kernel instantiation for (Dk, Dv slice, normaliser).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>

#include "la_fwd_ws.cuh"
#include "la_internal.h"

namespace la {
namespace ws {
// instantiated in la_fwd_ws_dk*.cu (one file per key width and direction)
#define LA_WS_DECL(DK)                                                                                         \
    extern template cudaError_t launch_dk<DK, false, false>(int, bool, const CUtensorMap&, const CUtensorMap&, \
                                                            const CUtensorMap&, const Params&, int, cudaStream_t); \
    extern template cudaError_t launch_dk<DK, true, false>(int, bool, const CUtensorMap&, const CUtensorMap&,  \
                                                           const CUtensorMap&, const Params&, int, cudaStream_t); \
    extern template cudaError_t launch_dk<DK, false, true>(int, bool, const CUtensorMap&, const CUtensorMap&,  \
                                                           const CUtensorMap&, const Params&, int, cudaStream_t); \
    extern template bool supported_dk<DK>(int, bool, bool);
LA_WS_DECL(16)
LA_WS_DECL(32)
LA_WS_DECL(64)
LA_WS_DECL(128)
#undef LA_WS_DECL
}  // namespace ws

EncodeTiledFn encode_tiled() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load();
    if (!f) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f = reinterpret_cast<EncodeTiledFn>(ptr);
        fn.store(f);
    }
    return f;
}

namespace {

// Widths with a kernel instance (key width DK, value slice NV).
bool width_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// The instance key width for a tensor width d (a multiple of 16 up to 128):
// the smallest instance width >= d; the tile columns past d are zero-filled
// by the TMA loads, which contributes nothing to scores or states.
int padded_width(int d) { return d <= 16 ? 16 : d <= 32 ? 32 : d <= 64 ? 64 : 128; }

// Tensor widths the tensor-core path takes.
bool tensor_width_ok(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }

// The widest value slice that divides Dv (a multiple of 16): halving it
// keeps it a divisor, so no slice ever runs past Dv.
int widest_slice(int Dv) {
    for (int w : {128, 64, 32})
        if (Dv % w == 0) return w;
    return 16;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
    return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                            : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

// [BH, T, width] bf16, boxes of [1, 128 tokens, box_inner columns].
bool make_map(CUtensorMap* map, const void* base, int width, int T, int BH, int box_inner) {
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(T),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(width) * 2,
                                   static_cast<cuuint64_t>(width) * 2 * static_cast<cuuint64_t>(T)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(ws::C), 1};
    const cuuint32_t elem[3] = {1, 1, 1};
    return f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(ws::row_bytes_for(box_inner)),
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    static std::atomic<int> n{0};
    int v = n.load();
    if (!v) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        n.store(v);
    }
    return v;
}

// sp: the state-pass instance
bool instance_ok(int Dk, int nv, bool norm, bool sp = false) {
    switch (Dk) {
        case 16: return ws::supported_dk<16>(nv, norm, sp);
        case 32: return ws::supported_dk<32>(nv, norm, sp);
        case 64: return ws::supported_dk<64>(nv, norm, sp);
        case 128: return ws::supported_dk<128>(nv, norm, sp);
        default: return false;
    }
}

// The widest value slice of the state-pass instance: it holds no Q ring, so
// wider slices fit than in the output pass, and each slice reloads K.
int state_slice(int Dk, int Dv, bool norm) {
    int nv = widest_slice(Dv);
    while (!instance_ok(padded_width(Dk), nv, norm, true) && nv / 2 >= 16) nv /= 2;
    return nv;
}

int env_int(const char* name) {
    const char* e = std::getenv(name);
    return e ? std::atoi(e) : 0;
}

// How the (b, h) sequences are spread over CTAs (one CTA per SM).
//  split: CTAs sharing one (b, h, segment), each owning nv value columns
//         (a slice width that divides Dv: Dv is a multiple of 16, and the
//         slices are 16, 32, 64 or 128 wide) and recomputing the 128 x 128
//         score tile;
//  nseg:  output segments per (b, h), of seg_chunks chunks each; segment i
//         starts from the state after segment i - 1, assembled from per_seg
//         state segments per earlier output segment (computed by a state
//         pass into the caller's workspace).
// The split is the smallest one whose tiles fit in shared memory.  While that
// leaves most SMs idle, the sequences are cut into segments (of at least
// kMinSegChunks chunks: a segment pays a second launch and a pipeline fill and
// drain, about as long as a dozen chunks) as long as one wave holds them, and
// only then the value columns are
// split further (slices of at least 16 columns): every extra slice reloads
// and re-multiplies Q and K, a segment only reloads K and V once in the state
// pass.  The state pass cuts each segment further while SMs stay idle.
struct Layout {
    int split, nv, nseg, seg_chunks, per_seg, nS;
    int split_sp, nv_sp;  // the state pass's slices
};

constexpr int kMinSegChunks = 16;

Layout plan_layout(int BH, int nchunks, int Dk, int Dv, bool norm, bool segments) {
    const int sms = sm_count();
    const long long target = sms * 4 / 5;
    const int DK = padded_width(Dk);
    int nv = widest_slice(Dv);
    while (!instance_ok(DK, nv, norm) && nv / 2 >= 16) nv /= 2;
    const int es = env_int("LA_DV_SPLIT");
    const bool fixed_split = es >= 1 && Dv % es == 0 && width_ok(Dv / es) && instance_ok(DK, Dv / es, norm);
    if (fixed_split) nv = Dv / es;
    int s = Dv / nv;
    int nseg = 1;
    if (segments && nchunks >= 2) {
        const int eg = env_int("LA_SEGMENTS");
        if (eg >= 1) {
            nseg = eg < nchunks ? eg : nchunks;
        } else if (static_cast<long long>(BH) * s < target) {
            while (nseg * 2 * kMinSegChunks <= nchunks && static_cast<long long>(BH) * s * nseg * 2 <= sms)
                nseg *= 2;
        }
    }
    if (!fixed_split)
        while (static_cast<long long>(BH) * s * nseg < target && nv / 2 >= 16) {
            nv /= 2;
            s = Dv / nv;
        }
    Layout L{};
    L.split = s;
    L.nv = nv;
    L.seg_chunks = (nchunks + nseg - 1) / (nseg > 0 ? nseg : 1);
    if (L.seg_chunks < 1) L.seg_chunks = 1;
    L.nseg = (nchunks + L.seg_chunks - 1) / L.seg_chunks;
    if (L.nseg < 1) L.nseg = 1;
    L.nv_sp = state_slice(Dk, Dv, norm);
    L.split_sp = Dv / L.nv_sp;
    L.per_seg = 1;
    if (L.nseg > 1)
        while (L.seg_chunks % (2 * L.per_seg) == 0 &&
               static_cast<long long>(BH) * L.split_sp * (L.nseg - 1) * L.per_seg * 2 <= sms)
            L.per_seg *= 2;
    L.nS = (L.nseg - 1) * L.per_seg;
    return L;
}

size_t workspace_bytes_for(int BH, int Dk, int Dv, int nS) {
    const size_t per = static_cast<size_t>(Dk) * Dv + Dk + 1;
    const size_t b = sizeof(float) * static_cast<size_t>(BH) * nS * per;
    return (b + 255) / 256 * 256;
}

}  // namespace

bool fwd_tc_supports(int Dk, int Dv) { return tensor_width_ok(Dk) && tensor_width_ok(Dv); }

int fwd_tc_state_pieces(int B, int H, int T, int Dk, int Dv, bool norm, long long* plan_key) {
    if (!fwd_tc_supports(Dk, Dv) || B <= 0 || H <= 0 || T <= 0) return 0;
    const Layout L = plan_layout(B * H, (T + ws::C - 1) / ws::C, Dk, Dv, norm, true);
    if (plan_key)
        *plan_key = ((static_cast<long long>(L.nseg) * 65536 + L.seg_chunks) * 64 + L.per_seg) * 64 + L.nS;
    return L.nS;
}

size_t fwd_tc_workspace_bytes(int B, int H, int T, int Dk, int Dv, bool norm) {
    if (!fwd_tc_supports(Dk, Dv) || B <= 0 || H <= 0 || T <= 0) return 0;
    const int BH = B * H;
    const Layout L = plan_layout(BH, (T + ws::C - 1) / ws::C, Dk, Dv, norm, true);
    return L.nS > 0 ? workspace_bytes_for(BH, Dk, Dv, L.nS) : 0;
}

namespace {

// Launches with programmatic stream serialisation.  The first launch of a
// call may start its prologue while the previous kernel on the stream ends.
// The output pass after a state pass is launched plainly: launched early, its
// first CTAs land on the SMs the state pass left idle and the wave ends up
// less even (measured: the gated T = 65536 forward 5% slower, the
// B = 4, H = 8, T = 2048 forward with four segments 6% faster).
constexpr int kPdlFirst = 1;
constexpr int kPdlOutput = 0;

template <bool REV, bool PHI>
cudaError_t launch_dir(int Dk, int nv, bool norm, const CUtensorMap& tmq, const CUtensorMap& tmk,
                       const CUtensorMap& tmv, const ws::Params& p, int grid, cudaStream_t stream) {
    switch (Dk) {
        case 16: return ws::launch_dk<16, REV, PHI>(nv, norm, tmq, tmk, tmv, p, grid, stream);
        case 32: return ws::launch_dk<32, REV, PHI>(nv, norm, tmq, tmk, tmv, p, grid, stream);
        case 64: return ws::launch_dk<64, REV, PHI>(nv, norm, tmq, tmk, tmv, p, grid, stream);
        case 128: return ws::launch_dk<128, REV, PHI>(nv, norm, tmq, tmk, tmv, p, grid, stream);
        default: return cudaErrorNotSupported;
    }
}

// The direction and the feature map pick the instance: the forward
// instances carry no code of the reverse scan (its index mapping, mask and
// accumulating epilogue), and only the feature-map instances map tiles.
cudaError_t launch_ws(int Dk, int nv, bool norm, const CUtensorMap& tmq, const CUtensorMap& tmk,
                      const CUtensorMap& tmv, const ws::Params& p, int grid, cudaStream_t stream) {
    if (p.feature_map == LA_FEATURE_ELU1)
        return p.reverse ? cudaErrorNotSupported
                         : launch_dir<false, true>(Dk, nv, norm, tmq, tmk, tmv, p, grid, stream);
    return p.reverse ? launch_dir<true, false>(Dk, nv, norm, tmq, tmk, tmv, p, grid, stream)
                     : launch_dir<false, false>(Dk, nv, norm, tmq, tmk, tmv, p, grid, stream);
}

}  // namespace

// A span's own state from zero (la_chunk_state_ws): the state pass alone, over
// `pieces` consecutive pieces of the span per (b, h) (doubled while the CTAs
// fit on the GPU at once), each writing its state, key sum and total log2
// decay to the workspace; the caller folds the pieces together.
namespace {

struct StatePlan {
    int split, nv, pieces, piece_chunks;
};

StatePlan plan_state(int BH, int nchunks, int Dk, int Dv, bool norm) {
    const int sms = sm_count();
    StatePlan P{};
    const int nv = state_slice(Dk, Dv, norm);
    const int s = Dv / nv;
    P.nv = nv;
    int pieces = 1;
    while (pieces * 2 <= nchunks && static_cast<long long>(BH) * s * pieces * 2 <= sms) pieces *= 2;
    P.split = s;
    P.piece_chunks = (nchunks + pieces - 1) / pieces;
    P.pieces = (nchunks + P.piece_chunks - 1) / P.piece_chunks;  // none empty
    return P;
}

}  // namespace

size_t fwd_state_workspace_bytes(int B, int H, int T, int Dk, int Dv, bool norm) {
    if (!fwd_tc_supports(Dk, Dv) || B <= 0 || H <= 0 || T <= 0) return 0;
    const int BH = B * H;
    return workspace_bytes_for(BH, Dk, Dv, plan_state(BH, (T + ws::C - 1) / ws::C, Dk, Dv, norm).pieces);
}

cudaError_t launch_fwd_state(const FwdArgs& a, int* pieces_used) {
    if (!fwd_tc_supports(a.Dk, a.Dv)) return cudaErrorNotSupported;
    const bool norm = a.normalize != 0;
    const int BH = a.B * a.H;
    const int nchunks = (a.T + ws::C - 1) / ws::C;
    const StatePlan P = plan_state(BH, nchunks, a.Dk, a.Dv, norm);
    const int nv = P.nv, DK = padded_width(a.Dk);
    if (!width_ok(nv) || !instance_ok(DK, nv, norm, true)) return cudaErrorNotSupported;
    if (!a.workspace || a.workspace_bytes < workspace_bytes_for(BH, a.Dk, a.Dv, P.pieces))
        return cudaErrorInvalidValue;
    if (pieces_used) *pieces_used = P.pieces;
    CUtensorMap tmq, tmk, tmv;
    const int box_k = DK < 64 ? DK : 64;
    const int box_v = norm ? 16 : (nv < 64 ? nv : 64);
    // the state pass reads no queries: the key tensor stands in for the map
    if (!make_map(&tmq, a.k, a.Dk, a.T, BH, box_k) || !make_map(&tmk, a.k, a.Dk, a.T, BH, box_k) ||
        !make_map(&tmv, a.v, a.Dv, a.T, BH, box_v))
        return cudaErrorInvalidValue;
    ws::Params p{};
    p.log_g = a.log_g;
    p.decay_kind = a.decay_kind;
    p.H = a.H;
    p.T = a.T;
    p.Dk = a.Dk;
    p.Dv = a.Dv;
    p.split = P.split;
    p.nchunks = nchunks;
    p.err = a.err_word;
    p.q_scale = 1.f;
    p.pdl = kPdlFirst;
    float* base = static_cast<float*>(a.workspace);
    p.ws_S = base;
    p.ws_z = p.ws_S + static_cast<size_t>(BH) * P.pieces * a.Dk * a.Dv;
    p.ws_L = p.ws_z + static_cast<size_t>(BH) * P.pieces * a.Dk;
    p.ws_nS = P.pieces;
    p.ws_per_seg = 1;
    p.state_pass = 1;
    p.nseg = P.pieces;
    p.seg_chunks = P.piece_chunks;
    return launch_ws(DK, nv, norm, tmq, tmk, tmv, p, BH * P.pieces * P.split, a.stream);
}


cudaError_t launch_fwd_tc(const FwdArgs& a, int* split_used, int* segments_used) {
    if (!fwd_tc_supports(a.Dk, a.Dv)) return cudaErrorNotSupported;
    // the reverse instances and the forward ones of 16-wide keys accumulate
    if (a.accumulate && !a.reverse && padded_width(a.Dk) != 16) return cudaErrorNotSupported;
    const bool norm = a.normalize != 0;
    const int BH = a.B * a.H;
    const int nchunks = (a.T + ws::C - 1) / ws::C;
    Layout L = plan_layout(BH, nchunks, a.Dk, a.Dv, norm, a.workspace != nullptr);
    if (L.nS > 0 && a.workspace_bytes < workspace_bytes_for(BH, a.Dk, a.Dv, L.nS))
        L = plan_layout(BH, nchunks, a.Dk, a.Dv, norm, false);  // too small: one segment
    const int split = L.split, nv = L.nv, DK = padded_width(a.Dk);
    if (!width_ok(nv) || !instance_ok(DK, nv, norm)) return cudaErrorNotSupported;
    if (split_used) *split_used = split;
    if (segments_used) *segments_used = L.nseg;

    CUtensorMap tmq, tmk, tmv;
    const int box_k = DK < 64 ? DK : 64;
    const int box_v = norm ? 16 : (nv < 64 ? nv : 64);  // the normaliser instances use 16-column panels
    if (!make_map(&tmq, a.q, a.Dk, a.T, BH, box_k) || !make_map(&tmk, a.k, a.Dk, a.T, BH, box_k) ||
        !make_map(&tmv, a.v, a.Dv, a.T, BH, box_v))
        return cudaErrorInvalidValue;

    ws::Params p{};
    p.log_g = a.log_g;
    p.decay_kind = a.decay_kind;
    p.init_state = a.init_state;
    p.init_z = a.init_z;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.final_state = a.final_state;
    p.final_z = a.final_z;
    p.H = a.H;
    p.T = a.T;
    p.Dk = a.Dk;
    p.Dv = a.Dv;
    p.split = split;
    p.nchunks = nchunks;
    p.err = a.err_word;
    p.reverse = a.reverse;
    p.accumulate = a.accumulate;
    p.q_scale = a.q_scale;
    p.feature_map = a.feature_map;
    p.pdl = kPdlFirst;
    if (a.states_ready && L.nS == 0) return cudaErrorInvalidValue;
    if (L.nS > 0) {
        float* base = static_cast<float*>(a.workspace);
        p.ws_S = base;
        p.ws_z = p.ws_S + static_cast<size_t>(BH) * L.nS * a.Dk * a.Dv;
        p.ws_L = p.ws_z + static_cast<size_t>(BH) * L.nS * a.Dk;
        p.ws_nS = L.nS;
        p.ws_per_seg = L.per_seg;
    }
    if (L.nS > 0 && !a.states_ready) {
        // state pass: the contribution of each state segment before the last output segment
        ws::Params ps = p;
        ps.state_pass = 1;
        ps.nseg = L.nS;
        ps.seg_chunks = L.seg_chunks / L.per_seg;
        ps.split = L.split_sp;
        // the value tiles of the state pass's own slice width
        CUtensorMap tmv_sp;
        if (!make_map(&tmv_sp, a.v, a.Dv, a.T, BH, norm ? 16 : (L.nv_sp < 64 ? L.nv_sp : 64)))
            return cudaErrorInvalidValue;
        const cudaError_t e = launch_ws(DK, L.nv_sp, norm, tmq, tmk, tmv_sp, ps, BH * L.nS * L.split_sp, a.stream);
        if (e != cudaSuccess) return e;
    }
    p.state_pass = 0;
    if (L.nS > 0) p.pdl = kPdlOutput;
    p.nseg = L.nseg;
    p.seg_chunks = L.seg_chunks;
    return launch_ws(DK, nv, norm, tmq, tmk, tmv, p, BH * L.nseg * split, a.stream);
}

}  // namespace la
