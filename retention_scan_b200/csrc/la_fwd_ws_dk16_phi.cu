// la_fwd_ws_dk16_phi.cu - instantiations of the warp-specialised tensor-core kernel for
// Dk = 16, forward scan with the feature map on the Q and K tiles (one file per key width and variant, so that the build
// compiles them in parallel).
#include "la_fwd_ws.cuh"

namespace la {
namespace ws {

template cudaError_t launch_dk<16, false, true>(int, bool, const CUtensorMap&, const CUtensorMap&,
                                                 const CUtensorMap&, const Params&, int, cudaStream_t);

}  // namespace ws
}  // namespace la
