// la_fwd_tc_dk32.cu - instantiations of the tensor-core forward for Dk = 32
// (one file per key width so that the build compiles them in parallel).
#include "la_fwd_tc.cuh"

namespace la {
namespace tc {

cudaError_t launch_dk32(int nv, const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                        const Params& p, int grid, cudaStream_t stream) {
    switch (nv) {
        case 16: return launch_instance<32, 16>(tmq, tmk, tmv, p, grid, stream);
        case 32: return launch_instance<32, 32>(tmq, tmk, tmv, p, grid, stream);
        case 64: return launch_instance<32, 64>(tmq, tmk, tmv, p, grid, stream);
        case 128: return launch_instance<32, 128>(tmq, tmk, tmv, p, grid, stream);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace tc
}  // namespace la
