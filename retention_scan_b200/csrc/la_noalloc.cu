// la_noalloc.cu - la_chunk_forward_noalloc: the forward whose T-segment
// scratch comes from a fixed device array of this library (one per device)
// instead of from the caller, so that a call allocates no device memory.
#include <cuda_runtime.h>

#include "la.h"
#include "la_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t{16} << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the array in the current device's context: the symbol
// has a different address on every device, and in host code its name is only
// a host-side stand-in.  Looked up with cudaGetSymbolAddress on the first
// call on each device (and again if that device's context was reset since).
void* static_scratch_for_current_device() {
    return la::device_symbol_address(&g_static_scratch, la::kSymStaticScratch);
}

}  // namespace

extern "C" {

size_t la_chunk_forward_noalloc_capacity(void) { return kStaticScratchBytes; }

la_status la_chunk_forward_noalloc(const void* q, const void* k, const void* v, const la_decay* decay,
                                   int normalize, const float* init_state, const float* init_z, void* out,
                                   float* final_state, float* final_z, int B, int H, int T, int Dk, int Dv,
                                   la_dtype dtype, la_stream_t stream) {
    const size_t need = la_chunk_forward_workspace_size(B, H, T, Dk, Dv, dtype, normalize);
    if (need > kStaticScratchBytes) return LA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = static_scratch_for_current_device();
        if (!scratch) return LA_ERR_CUDA;
    }
    return la_chunk_forward_ws(q, k, v, decay, normalize, init_state, init_z, out, final_state, final_z, B, H, T,
                               Dk, Dv, dtype, scratch, need, stream);
}

}  // extern "C"
