// la_fwd_ws_dk128_phi.cu - instantiations of the warp-specialised tensor-core kernel for
// Dk = 128, forward scan with the feature map on the Q and K tiles (one file per key width and variant, so that the build
// compiles them in parallel).
#include "la_fwd_ws.cuh"

namespace la {
namespace ws {

template cudaError_t launch_dk<128, false, true>(int, bool, const CUtensorMap&, const CUtensorMap&,
                                                 const CUtensorMap&, const Params&, int, cudaStream_t);

}  // namespace ws
}  // namespace la
