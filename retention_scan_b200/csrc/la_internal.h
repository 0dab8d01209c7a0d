// la_internal.h - launcher interface between the C ABI (la_api.cu) and the
// kernel files.  Not installed; the public interface is include/la.h.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "la.h"

namespace la {

// cuTensorMapEncodeTiled, looked up once through the runtime (so that
// libcuda is not linked); null if the driver does not provide it.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// Device address of one of this library's __device__ variables in the
// current device's current context (`slot` names the variable: one cache
// entry per slot and device).  The lookup (cudaGetSymbolAddress) runs once per
// device and is repeated only when the device's context has changed since,
// for instance after cudaDeviceReset; null if it fails.
enum SymbolSlot : int { kSymErrWord = 0, kSymStaticScratch = 1, kSymSlots = 2 };
void* device_symbol_address(const void* symbol, int slot);

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
    void* workspace;          // scratch for T-segment states (may be null: no segments)
    size_t workspace_bytes;
    int reverse;              // 1: anti-causal scan, t = T-1 down to 0
    int accumulate;           // 1: add y to the values already in out
    int feature_map;          // la_feature_map on q and k (forward scans)
    float q_scale;            // q <- q_scale * phi(q)
    int states_ready;         // 1: the workspace already holds this call's state
                              // segments (fwd_tc_state_pieces); no state pass
};

// The T-segment state pieces that launch_fwd_tc plans for these sizes with a
// workspace (0: none): their count per (b, h), and the plan's segmentation as
// one number that equal plans share (for reusing one scan's state pieces,
// transposed, in another).
int fwd_tc_state_pieces(int B, int H, int T, int Dk, int Dv, bool norm, long long* plan_key);

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
    int feature_map;          // la_feature_map on q and k
    float q_scale;            // q <- q_scale * phi(q)
    cudaStream_t stream;
};

// fp32 inputs: recurrent kernel on fp32 FMA units (la_fwd_f32.cu).
cudaError_t launch_fwd_f32(const FwdArgs& a);

// bf16 inputs: chunked kernel on tcgen05 tensor cores (la_fwd_tc.cu).
// Returns cudaErrorNotSupported for shapes without a kernel; *split_used and
// *segments_used (may be null) receive the value split and the number of
// T-segments that ran.  Segments need a.workspace of at least
// fwd_tc_workspace_bytes(...) bytes; with less (or none) the sequence runs as
// one segment.
cudaError_t launch_fwd_tc(const FwdArgs& a, int* split_used, int* segments_used);
bool fwd_tc_supports(int Dk, int Dv);
size_t fwd_tc_workspace_bytes(int B, int H, int T, int Dk, int Dv, bool norm);

// A span's own state from zero (la_fwd_tc.cu, la_chunk_state_ws): the state
// pass over consecutive pieces of each (b, h)'s span into a.workspace (at least
// fwd_state_workspace_bytes), laid out [B H][pieces][Dk][Dv] states, then
// [B H][pieces][Dk] key sums, then [B H][pieces] total log2 decays;
// *pieces_used receives the number of pieces.
cudaError_t launch_fwd_state(const FwdArgs& a, int* pieces_used);
size_t fwd_state_workspace_bytes(int B, int H, int T, int Dk, int Dv, bool norm);

// Left fold of n consecutive spans' states (la_state.cu):
//   S <- init (or 0);  for j < n:  S <- exp(L_j) S + S_j   (z likewise),
// out_L = sum_j L_j in natural-log units.  Span j's array for (b, h) starts at
// base + j * span + bh * bh_stride ([Dk][Dv] states, [Dk] key sums, one L).
struct CombineArgs {
    const float* S;
    long long S_span, S_bh;
    const float* z;           // may be null when out_z is
    long long z_span, z_bh;
    const float* L;
    long long L_span, L_bh;
    int n;
    int log2_units;           // L given in log2 units (the state pass's)
    const float* init_S;      // may be null (zero)
    const float* init_z;      // may be null (zero)
    float* out_S;             // [BH][Dk][Dv]
    float* out_z;             // [BH][Dk] or null
    float* out_L;             // [BH] or null
    int BH, Dk, Dv;
    cudaStream_t stream;
};
cudaError_t launch_fold(const CombineArgs& a);
// out[bh] = sum over T of the log decay (natural log), summed in double.
cudaError_t launch_log_total(const float* log_g, int kind, int BH, int H, int T, float* out, cudaStream_t stream);

// Decode step (la_decode.cu).
cudaError_t launch_decode(const DecodeArgs& a, la_dtype dtype);

// Small kernels of the backward pass (la_bwd.cu).  All asynchronous on
// `stream`; each returns the launch status.
//   out[bh] = in[bh]^T for BH matrices of R x C fp32 values.
cudaError_t launch_transpose(const float* in, float* out, int BH, int R, int C, cudaStream_t stream);
//   out[b,h,t] = decay of token t + 1 (log, per step; 0 for the last token),
//   from a per-head ([H]) or per-step ([B,H,T]) log decay.
cudaError_t launch_shift_decay(const float* log_g, int kind, float* out, int B, int H, int T, cudaStream_t stream);
//   s[b,h] *= g_1 (the decay of each sequence's first token), [B,H,n] fp32.
cudaError_t launch_scale_by_first_decay(float* s, const float* log_g, int kind, int B, int H, int T, int n,
                                        cudaStream_t stream);
// Gradient of the log decay: d[b,h,t] = sum_{s >= t} (q_s . dq_s - k_s . dk_s)
// + <dSf[b,h], S_T[b,h]> (S_T given transposed, [Dv, Dk]); per step it is
// written to d_log_g [B,H,T], per head summed into d_log_g [H].
struct DlogArgs {
    const void* q;
    const void* k;
    const void* dq;
    const void* dk;
    const float* d_final_state;   // may be null
    const float* st;              // S_T[i][j] at st[bh * st_bh + i * st_i + j * st_j] (when d_final_state)
    long long st_bh;
    int st_i, st_j;
    const float* d_final_z;       // may be null (normalised forward only)
    const float* zt;              // z_T[i] at zt[bh * zt_bh + i * zt_i] (when d_final_z)
    long long zt_bh;
    int zt_i;
    float* d_log_g;
    int kind;                     // LA_DECAY_PER_HEAD or LA_DECAY_PER_STEP
    int B, H, T, Dk, Dv;
    la_dtype dtype;
    double* scratch;              // dlog_scratch_doubles(B, H, T) doubles
    cudaStream_t stream;
};
size_t dlog_scratch_doubles(int B, int H, int T);
cudaError_t launch_dlog(const DlogArgs& a);
// Normalised backward helpers (la_bwd.cu):
//   [n][16] panel, column 0 = 1, the rest 0 (`dtype`)
cudaError_t launch_ones_panel(void* out, long long n, la_dtype dtype, cudaStream_t stream);
//   per (b, h) the Dk vector x (null: zeros) into column 0 of [Dk][16]
//   (rows = true) or row 0 of [16][Dk] (rows = false), fp32
cudaError_t launch_vec_panel(const float* x, float* out, int BH, int Dk, bool rows, cudaStream_t stream);
//   dn = dy / den, dden panel column 0 = -(dy . y) / den, per token (y the
//   normalised output n / den)
cudaError_t launch_norm_grad(const void* dy, const void* y, const void* den_panel, void* dn, void* dden_panel,
                             int Dv, long long ntok, la_dtype dtype, cudaStream_t stream);
//   out[b,h,:] = g_1 * row `row` of panel [B,H,rows,Dk]
cudaError_t launch_panel_row_scaled(const float* panel, float* out, const float* log_g, int kind, int B, int H,
                                    int T, int Dk, int rows, int row, cudaStream_t stream);
//   PK[t] = [v_t | 1 | 0 ...], W wide (`dtype`)
cudaError_t launch_pack_value_panel(const void* v, void* pk, int Dv, int W, long long ntok, la_dtype dtype,
                                    cudaStream_t stream);
//   [S | z | 0] as [Dk][W] fp32 per (b, h); S, z may be null (zeros)
cudaError_t launch_pack_state_panel(const float* S, const float* z, float* out, int BH, int Dk, int Dv, int W,
                                    cudaStream_t stream);
//   from [n | den | ..] (W wide): PQ = [dn | dden | 0 ..] (W wide) and dn (Dv wide)
cudaError_t launch_norm_grad_panel(const void* dy, const void* nd, void* pq, void* dn, int Dv, int W, long long ntok,
                                   la_dtype dtype, cudaStream_t stream);

// RWKV-4 WKV recurrence (la_wkv4.cu).
struct Wkv4Args {
    const void* k;
    const void* v;
    const float* w;
    const float* u;
    const float* init_state;  // [B,3,C] or null (empty state)
    void* out;
    float* final_state;       // [B,3,C] or null
    int B, T, C;
    la_dtype dtype;
    int* err_word;
    void* workspace;          // T-segment states (may be null: one segment)
    size_t workspace_bytes;
    cudaStream_t stream;
};
cudaError_t launch_wkv4(const Wkv4Args& a);
// [B, T, C] tensor map (la_wkv4.cu), boxes of [1, box_t, box_c], no swizzle.
bool make_btc_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int es, int B, int T, int C, int box_c,
                  int box_t);

// Cumulative EMA along T (la_ema.cu).
struct EmaArgs {
    const void* x;            // values [B, T, C]
    const void* f;            // factors [B, T, C]
    const float* init_state;  // [B, C] or null (0)
    void* out;                // [B, T, C]
    float* final_state;       // [B, C] or null
    int B, T, C;
    la_dtype dtype;
    int reverse;
    int* err_word;
    cudaStream_t stream;
};
cudaError_t launch_ema(const EmaArgs& a);
size_t wkv4_workspace_bytes(int B, int T, int C, la_dtype dtype);

}  // namespace la
