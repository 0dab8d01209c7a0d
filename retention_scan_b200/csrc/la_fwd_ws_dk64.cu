// la_fwd_ws_dk64.cu - instantiations of the warp-specialised tensor-core kernel for
// Dk = 64, forward scan (one file per key width and variant, so that the build
// compiles them in parallel).
#include "la_fwd_ws.cuh"

namespace la {
namespace ws {

template cudaError_t launch_dk<64, false, false>(int, bool, const CUtensorMap&, const CUtensorMap&,
                                                 const CUtensorMap&, const Params&, int, cudaStream_t);
template bool supported_dk<64>(int, bool, bool);

}  // namespace ws
}  // namespace la
