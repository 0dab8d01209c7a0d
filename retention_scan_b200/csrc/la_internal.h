// la_internal.h - launcher interface between the C ABI (la_api.cu) and the
// kernel files.  Not installed; the public interface is include/la.h.
#pragma once
#include <cuda_runtime.h>

#include "la.h"

namespace la {

// Device error codes written by kernels that give up waiting on a barrier.
enum DeviceError : int {
    kErrNone = 0,
    kErrTmaWait = 1,   // a TMA load never completed
    kErrMmaWait = 2,   // a tcgen05 MMA batch never completed
};

struct FwdArgs {
    const void* q;
    const void* k;
    const void* v;
    int decay_kind;           // la_decay_kind
    const float* log_g;
    int normalize;
    const float* init_state;  // may be null
    const float* init_z;      // may be null
    void* out;
    float* final_state;       // may be null
    float* final_z;           // may be null
    int B, H, T, Dk, Dv;
    cudaStream_t stream;
    int* err_word;            // device error word of the current device
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    int decay_kind;
    const float* log_g;
    int normalize;
    float* state;
    float* z;
    void* out;
    int B, H, Dk, Dv;
    cudaStream_t stream;
};

// fp32 inputs: recurrent kernel on fp32 FMA units (la_fwd_f32.cu).
cudaError_t launch_fwd_f32(const FwdArgs& a);

// bf16 inputs: chunked kernel on tcgen05 tensor cores (la_fwd_tc.cu).
// dv_split: number of CTAs sharing one (b, h), each owning Dv / dv_split
// value columns (0 = choose).  Returns cudaErrorNotSupported for shapes
// without a kernel; *split_used receives the split that ran.
cudaError_t launch_fwd_tc(const FwdArgs& a, int dv_split, int* split_used);
bool fwd_tc_supports(int Dk, int Dv);

// Decode step (la_decode.cu).
cudaError_t launch_decode(const DecodeArgs& a, la_dtype dtype);

}  // namespace la
