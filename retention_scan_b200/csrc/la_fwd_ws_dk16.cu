// la_fwd_ws_dk16.cu - instantiations of the warp-specialised tensor-core
// forward for Dk = 16 (one file per key width so the build runs in parallel).
#include "la_fwd_ws.cuh"

namespace la {
namespace ws {

template <bool NORM>
static cudaError_t launch_nv(int nv, const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                             const Params& p, int grid, cudaStream_t stream) {
    switch (nv) {
        case 16: return launch_instance<16, 16, NORM>(tmq, tmk, tmv, p, grid, stream);
        case 32: return launch_instance<16, 32, NORM>(tmq, tmk, tmv, p, grid, stream);
        case 64: return launch_instance<16, 64, NORM>(tmq, tmk, tmv, p, grid, stream);
        case 128: return launch_instance<16, 128, NORM>(tmq, tmk, tmv, p, grid, stream);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_dk16(int nv, bool norm, const CUtensorMap& tmq, const CUtensorMap& tmk,
                        const CUtensorMap& tmv, const Params& p, int grid, cudaStream_t stream) {
    return norm ? launch_nv<true>(nv, tmq, tmk, tmv, p, grid, stream)
                : launch_nv<false>(nv, tmq, tmk, tmv, p, grid, stream);
}

bool supported_dk16(int nv, bool norm) {
    switch (nv) {
        case 16: return norm ? supported<16, 16, true>() : supported<16, 16, false>();
        case 32: return norm ? supported<16, 32, true>() : supported<16, 32, false>();
        case 64: return norm ? supported<16, 64, true>() : supported<16, 64, false>();
        case 128: return norm ? supported<16, 128, true>() : supported<16, 128, false>();
        default: return false;
    }
}

}  // namespace ws
}  // namespace la
