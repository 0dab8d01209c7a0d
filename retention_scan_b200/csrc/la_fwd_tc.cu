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
#define LA_WS_DECL(DK)                                                                                        \
    cudaError_t launch_dk##DK(int, bool, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,           \
                              const Params&, int, cudaStream_t);                                              \
    bool supported_dk##DK(int, bool);
LA_WS_DECL(16)
LA_WS_DECL(32)
LA_WS_DECL(64)
LA_WS_DECL(128)
#undef LA_WS_DECL
}  // namespace ws

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

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

bool width_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

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

bool instance_ok(int Dk, int nv, bool norm) {
    switch (Dk) {
        case 16: return ws::supported_dk16(nv, norm);
        case 32: return ws::supported_dk32(nv, norm);
        case 64: return ws::supported_dk64(nv, norm);
        case 128: return ws::supported_dk128(nv, norm);
        default: return false;
    }
}

// How many CTAs share one (b, h): each owns Dv / split value columns and
// recomputes the 128 x 128 score tile.  The split is the smallest one whose
// tiles fit in shared memory, doubled while that leaves most SMs idle
// (keeping slices of at least 16 columns).
int choose_split(int BH, int Dk, int Dv, bool norm) {
    if (const char* env = std::getenv("LA_DV_SPLIT")) {
        const int s = std::atoi(env);
        if (s >= 1 && Dv % s == 0 && width_ok(Dv / s) && instance_ok(Dk, Dv / s, norm)) return s;
    }
    int s = 1;
    while (!instance_ok(Dk, Dv / s, norm) && Dv / (2 * s) >= 16) s *= 2;
    const int target = sm_count() * 4 / 5;
    while (static_cast<long long>(BH) * s < target && Dv / (2 * s) >= 16) s *= 2;
    return s;
}

}  // namespace

bool fwd_tc_supports(int Dk, int Dv) { return width_ok(Dk) && width_ok(Dv); }

cudaError_t launch_fwd_tc(const FwdArgs& a, int dv_split, int* split_used) {
    if (!fwd_tc_supports(a.Dk, a.Dv)) return cudaErrorNotSupported;
    const bool norm = a.normalize != 0;
    const int BH = a.B * a.H;
    const int split = dv_split > 0 ? dv_split : choose_split(BH, a.Dk, a.Dv, norm);
    const int nv = a.Dv / split;
    if (a.Dv % split != 0 || !width_ok(nv) || !instance_ok(a.Dk, nv, norm)) return cudaErrorNotSupported;
    if (split_used) *split_used = split;

    CUtensorMap tmq, tmk, tmv;
    const int box_k = a.Dk < 64 ? a.Dk : 64;
    const int box_v = nv < 64 ? nv : 64;
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
    p.Dv = a.Dv;
    p.split = split;
    p.nchunks = (a.T + ws::C - 1) / ws::C;
    p.err = a.err_word;
    const int grid = BH * split;
    switch (a.Dk) {
        case 16: return ws::launch_dk16(nv, norm, tmq, tmk, tmv, p, grid, a.stream);
        case 32: return ws::launch_dk32(nv, norm, tmq, tmk, tmv, p, grid, a.stream);
        case 64: return ws::launch_dk64(nv, norm, tmq, tmk, tmv, p, grid, a.stream);
        case 128: return ws::launch_dk128(nv, norm, tmq, tmk, tmv, p, grid, a.stream);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace la
