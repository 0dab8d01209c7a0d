/*
 * la.h - C ABI of the retention_scan_b200 library: causal linear attention
 * with an optional decay, on NVIDIA B200 (sm_100a), one GPU.
 *
 * What is computed (per batch b and head h, tokens t = 1..T):
 *
 *     S_t = g_t * S_{t-1} + k_t v_t^T          state, [Dk, Dv], fp32
 *     z_t = g_t * z_{t-1} + k_t                key sum, [Dk], fp32 (normalised only)
 *     y_t = q_t^T S_t                          unnormalised output
 *     y_t = (q_t^T S_t) / (q_t^T z_t)          normalised output
 *
 * Sources:
 *   - The recurrence with g = 1, a zero start and the current token included
 *     in y_t: "CS336 L04 linear attention duality" exercise page (tensortonic),
 *     problem statement and its three worked examples.
 *   - g_t as a per-step decay factor, state <- state * factor + value, and
 *     g = gamma (per-head constant) for retention: Jamie-Stirling/RetNet
 *     issue 21, "Proposed improvement/collaboration: removing the O(T^2)
 *     training cost", the cumulative_ema listing and the retention(Q,K,gamma,V)
 *     listing that follows it.
 *   - Decays kept as log values so that every factor is exp(x) with x <= 0:
 *     BlinkDL/RWKV-LM discussion 189, "Numerically stable parallel
 *     cumsum-based WKV", second bullet (exponentially weighted
 *     parameterisation).
 *   - The normaliser QKV / QK1, the carried KV state ("cache") and the carried
 *     key sum ("Z-state", cum_k, shape [B,H,1,D]): flash-linear-attention
 *     issue 268, "[Linear Attention] Update fused_recurrent.py for inference
 *     with nomalization=true", the opening comment and yiyousong's two
 *     explanations (the cache identity and the cum_k argument), and the reply
 *     recommending that the Z-state stay separate from the memory state.
 *
 * Readings where the pages are silent (each is fixed here, not guessed per
 * call):
 *   - g_1 decays the initial state: S_1 = g_1 S_0 + k_1 v_1^T.
 *   - z decays with the same g_t as S.
 *   - The denominator has no epsilon: IEEE division.  The caller keeps
 *     q^T z positive (for instance with the feature map elu(x)+1).
 *   - Feature maps and the q scale are applied by the caller.
 *   - out has the dtype of q; state and key sum are always fp32.
 *
 * Layouts (all dense, row-major, innermost index last):
 *   q, k            [B, H, T, Dk]   dtype
 *   v, out          [B, H, T, Dv]   dtype
 *   state           [B, H, Dk, Dv]  fp32  (Dv fastest)
 *   z               [B, H, Dk]      fp32
 *   decode q, k     [B, H, Dk]      dtype
 *   decode v, out   [B, H, Dv]      dtype
 *
 * Ownership: every pointer is a device pointer owned by the caller.  The
 * library allocates no device memory, keeps no per-call state and never
 * prints.  It may be called from several host threads.
 *
 * Execution: every entry point enqueues its work on `stream` and returns; a
 * device-side failure surfaces at the caller's next synchronisation.  A
 * kernel that gives up waiting on one of its own barriers sets a device
 * error word, which la_device_error() reads and clears.
 */
#ifndef RETENTION_SCAN_B200_LA_H
#define RETENTION_SCAN_B200_LA_H

#include <stddef.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so that this header needs no
 * CUDA header.  NULL is the legacy default stream. */
typedef struct CUstream_st* la_stream_t;

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,   /* null required pointer, bad size, misaligned pointer, bad decay kind */
    LA_ERR_UNSUPPORTED = 2,   /* valid request that this build has no kernel for */
    LA_ERR_CUDA = 3           /* a CUDA call or kernel launch failed */
} la_status;

typedef enum {
    LA_F32 = 0,               /* q, k, v, out are float32 */
    LA_BF16 = 1               /* q, k, v, out are bfloat16 */
} la_dtype;

typedef enum {
    LA_DECAY_NONE = 0,        /* g = 1: plain linear attention; log_g ignored */
    LA_DECAY_PER_HEAD = 1,    /* g_t = exp(log_g[h]) for every t; log_g is [H] */
    LA_DECAY_PER_STEP = 2     /* g_t = exp(log_g[b,h,t]); log_g is [B,H,T] ([B,H] for decode) */
} la_decay_kind;

/* Decay descriptor.  log_g holds natural logs of the decay factors, finite
 * and <= 0, fp32, on the device.  A NULL descriptor means LA_DECAY_NONE.
 * The page's per-head retention decay gamma_h enters as log(gamma_h). */
typedef struct {
    int kind;                 /* an la_decay_kind value */
    const float* log_g;       /* device pointer, see kind for the shape */
} la_decay;

/* Input prologue: a feature map on q and k and a scale on q, applied by the
 * kernels as they read their inputs instead of by a separate pass over
 * memory.  The normalised linear attention of flash-linear-attention issue
 * 268 feeds elu(x) + 1 of the queries and keys, and its sequence diagram
 * passes q * scale; with a prologue the caller hands over the raw q and k.
 * A NULL prologue, or {LA_FEATURE_NONE, 1.0f}, reads the inputs as they are. */
typedef enum {
    LA_FEATURE_NONE = 0,      /* phi(x) = x */
    LA_FEATURE_ELU1 = 1       /* phi(x) = elu(x) + 1 = (x > 0 ? x + 1 : e^x), in fp32 */
} la_feature_map;

typedef struct {
    int feature_map;          /* an la_feature_map value, applied to q and k */
    float q_scale;            /* q <- q_scale * phi(q); finite */
} la_prologue;

/*
 * la_chunk_forward - the whole sequence forward pass.
 *
 * Computes out[b,h,t,:] = y_t for t = 1..T from the recurrence above, and
 * optionally the state and key sum after token T.
 *
 *   q, k, v        inputs, layouts above, `dtype`.  Required (for T > 0).
 *   decay          NULL or a descriptor (see la_decay).
 *   normalize      0: y_t = q_t^T S_t.  1: y_t = q_t^T S_t / q_t^T z_t.
 *   init_state     NULL (zeros) or S_0, [B,H,Dk,Dv] fp32.
 *   init_z         NULL (zeros) or z_0, [B,H,Dk] fp32; read only if normalize.
 *   out            output y, [B,H,T,Dv], `dtype`.  Required (for T > 0).
 *   final_state    NULL (not written) or S_T, [B,H,Dk,Dv] fp32.
 *   final_z        NULL (not written) or z_T, [B,H,Dk] fp32; written only if normalize.
 *   B, H, T        batch, heads, tokens; each >= 0.  B*H == 0 is a no-op.
 *                  T == 0 writes final_state = S_0 and final_z = z_0.
 *   Dk, Dv         key and value widths, >= 1.
 *   stream         CUDA stream.
 *
 * Aliasing: outputs must not overlap inputs; final_state must not overlap
 * init_state, nor final_z init_z.
 *
 * Errors (returned synchronously, nothing is enqueued):
 *   LA_ERR_INVALID_ARG  a required pointer is NULL; a size is negative or
 *                       Dk, Dv < 1; a pointer is not 16-byte aligned; decay
 *                       kind out of range or its log_g NULL; normalize with
 *                       init_state given but init_z NULL (a carried state
 *                       without its key sum gives a wrong denominator: the
 *                       defect described in flash-linear-attention issue 268).
 *   LA_ERR_UNSUPPORTED  LA_F32 with Dk or Dv > 128; LA_BF16 with Dk or Dv not
 *                       a multiple of 16 in [16, 128].
 *   LA_ERR_CUDA         a launch or CUDA runtime call failed.
 *
 * bf16 runs on tcgen05 tensor cores with fp32 accumulation (chunks of 128
 * tokens); fp32 runs a recurrent kernel on fp32 FMA units (no TF32).  The
 * bf16 kernels exist for key widths 16, 32, 64 and 128 and value slices of
 * 16, 32, 64 or 128 columns; other key widths run on the next larger one,
 * the tile columns past Dk read as zeros (the TMA loads' fill), and the
 * value columns run in slices of a width that divides Dv.
 */
LA_API la_status la_chunk_forward(const void* q, const void* k, const void* v,
                           const la_decay* decay, int normalize,
                           const float* init_state, const float* init_z,
                           void* out, float* final_state, float* final_z,
                           int B, int H, int T, int Dk, int Dv,
                           la_dtype dtype, la_stream_t stream);

/*
 * la_chunk_forward_workspace_size - scratch bytes that la_chunk_forward_ws
 * can use for these sizes (0 when the sequence would run as one segment).
 *
 * With a workspace, a bf16 forward whose B*H heads would leave most SMs idle
 * cuts each sequence into T-segments that run side by side: a first pass
 * computes every earlier segment's own state contribution S_j (from a zero
 * state) and its total decay G_j, and the main pass starts segment i from
 * the combination of the earlier ones, S <- G_j S + S_j in order: the
 * associative pairing of (state, decay) spans that RetNet issue 21 uses for
 * its cumulative-EMA scan (and RWKV-LM discussion 189 for the parallel WKV
 * form).  Results equal the unsegmented pass up to fp32 summation order.
 * The fp32 path ignores the workspace.  Deterministic for given sizes and
 * environment (LA_SEGMENTS and LA_DV_SPLIT override the choice, for tests).
 */
LA_API size_t la_chunk_forward_workspace_size(int B, int H, int T, int Dk, int Dv,
                                              la_dtype dtype, int normalize);

/*
 * la_chunk_forward_ws - la_chunk_forward with caller-owned scratch.
 *
 *   workspace        NULL, or device memory of workspace_bytes bytes, 16-byte
 *                    aligned, not overlapping any other argument.  Its
 *                    contents on entry do not matter; it is used on `stream`
 *                    only and may be reused once the stream has passed this
 *                    call.  NULL (or a size below
 *                    la_chunk_forward_workspace_size) runs one segment per
 *                    sequence, exactly as la_chunk_forward.
 *   other arguments  as la_chunk_forward.
 *
 * Errors as la_chunk_forward, plus LA_ERR_INVALID_ARG for a non-NULL
 * workspace that is not 16-byte aligned.
 */
LA_API la_status la_chunk_forward_ws(const void* q, const void* k, const void* v,
                              const la_decay* decay, int normalize,
                              const float* init_state, const float* init_z,
                              void* out, float* final_state, float* final_z,
                              int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                              void* workspace, size_t workspace_bytes,
                              la_stream_t stream);

/*
 * la_chunk_reverse_ws - the anti-causal (right-to-left) scan.
 *
 * The recurrence run from the last token back to the first: RetNet issue 21,
 * Details (the cumulative EMA's reverse flag: the forward scan of the
 * time-reversed inputs, reversed back), which gives:
 *
 *   S_{T+1} = init_state (or 0),   z_{T+1} = init_z (or 0)
 *   S_t = g_t S_{t+1} + k_t v_t^T,  z_t = g_t z_{t+1} + k_t,   t = T .. 1
 *   y_t = q_t^T S_t  (normalize: / q_t^T z_t)
 *
 * so y_t sums over s >= t with the weight g_t g_{t+1} ... g_{s-1}; the
 * decay g_t of token t scales everything after it, mirroring the forward
 * scan.  final_state / final_z receive S_1 / z_1.  Arguments, layouts,
 * workspace (sized by la_chunk_forward_workspace_size), aliasing rules and
 * errors as la_chunk_forward_ws.
 */
LA_API la_status la_chunk_reverse_ws(const void* q, const void* k, const void* v,
                              const la_decay* decay, int normalize,
                              const float* init_state, const float* init_z,
                              void* out, float* final_state, float* final_z,
                              int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                              void* workspace, size_t workspace_bytes,
                              la_stream_t stream);

/*
 * la_chunk_state_ws - the state a span of the sequence leaves when it starts
 * from zero, and the span's total log decay (no outputs, no queries).
 *
 *   S_0 = 0, z_0 = 0;  S_t = g_t S_{t-1} + k_t v_t^T,  z_t = g_t z_{t-1} + k_t
 *   state_out = S_T,  z_out = z_T,  log_g_total[b,h] = sum_t log g_t
 *
 * With these, the state entering any later span follows from the associative
 * combination of consecutive spans, RetNet issue 21 (the paragraph on the
 * associative EMA operator): (S_a, G_a) o (S_b, G_b) = (G_b S_a + S_b, G_a G_b)
 * with G = exp(log_g_total) (la_state_combine).  This is the first step of a
 * sequence split along T over GPUs: each span's state, one exchange of them,
 * then each span's forward from the combined state entering it.
 *
 *   k, v, decay, normalize, B, H, T, Dk, Dv, dtype   as la_chunk_forward_ws
 *   state_out    [B, H, Dk, Dv] fp32, required, 16-byte aligned.
 *   z_out        [B, H, Dk] fp32, required (16-byte aligned) when normalize,
 *                else ignored.
 *   log_g_total  [B, H] fp32 natural log, or NULL (not written).
 *   workspace    bf16: at least la_chunk_state_workspace_size(...) bytes,
 *                16-byte aligned, required when T > 0; fp32: unused.
 *
 * T == 0 writes zero states and a zero log total.  Errors: as
 * la_chunk_forward_ws, and LA_ERR_INVALID_ARG for a missing or short bf16
 * workspace.  bf16 runs the chunked kernel's state pass over pieces of the
 * span and folds them; fp32 runs the recurrent kernel without its outputs.
 */
LA_API size_t la_chunk_state_workspace_size(int B, int H, int T, int Dk, int Dv,
                                            la_dtype dtype, int normalize);
LA_API la_status la_chunk_state_ws(const void* k, const void* v, const la_decay* decay,
                                   int normalize, float* state_out, float* z_out,
                                   float* log_g_total, int B, int H, int T, int Dk, int Dv,
                                   la_dtype dtype, void* workspace, size_t workspace_bytes,
                                   la_stream_t stream);

/*
 * la_state_combine - the left fold of n consecutive spans' states with the
 * associative operator above (RetNet issue 21, the associative EMA operator):
 *
 *   S <- init_state (or 0),  z <- init_z (or 0)
 *   for j = 0 .. n-1:  S <- exp(L_j) S + S_j,  z <- exp(L_j) z + z_j
 *   state_out = S,  z_out = z,  log_g_out = sum_j L_j
 *
 * so that state_out is the state after spans 0..n-1 entered with init_state.
 *   seg_state   span j's [B, H, Dk, Dv] fp32 state at seg_state + j * state_stride
 *   seg_z       span j's [B, H, Dk] key sum at seg_z + j * z_stride (needed when
 *               z_out is given and n > 0)
 *   seg_log_g   span j's [B, H] natural-log total decay at seg_log_g + j * log_stride
 *               (strides in floats, >= 0)
 *   init_state, init_z   [B, H, Dk, Dv] / [B, H, Dk] fp32 or NULL (zero)
 *   state_out   [B, H, Dk, Dv] fp32, required; may be init_state (each element
 *               is read before it is written)
 *   z_out, log_g_out     [B, H, Dk] / [B, H] fp32 or NULL (not written)
 * Every pointer 4-byte aligned.  n == 0 copies the initial state (or zeros).
 * Errors: LA_ERR_INVALID_ARG for negative sizes or strides, a missing
 * required pointer or a misaligned one; LA_ERR_CUDA if the launch fails.
 */
LA_API la_status la_state_combine(const float* seg_state, const float* seg_z,
                                  const float* seg_log_g, long long state_stride,
                                  long long z_stride, long long log_stride, int n,
                                  const float* init_state, const float* init_z,
                                  float* state_out, float* z_out, float* log_g_out,
                                  int B, int H, int Dk, int Dv, la_stream_t stream);

/*
 * la_chunk_bidirectional_ws - the bidirectional (encoder) form:
 * out = y_forward + y_reverse, both scans from zero states.
 *
 * RetNet issue 21, Details (closing remark) builds a bidirectional encoder
 * from one forward and one reverse retention of the same sequence.  Both
 * scans include their own token, and the plain reading of that remark -
 * the sum of the two outputs - counts the s = t term q_t^T k_t v_t twice.  That is what
 * this computes; with normalize each direction is normalised by its own key
 * sum before the addition.  Two launches on `stream`: the forward scan
 * writes out, the reverse scan adds to it (bf16: the sum is formed in fp32
 * from the stored bf16 forward value and rounded once more).
 *
 *   q, k, v, decay, normalize, out, B, H, T, Dk, Dv, dtype, workspace,
 *   workspace_bytes, stream   as la_chunk_forward_ws.
 *
 * Errors as la_chunk_forward_ws; on an error nothing is enqueued.
 */
LA_API la_status la_chunk_bidirectional_ws(const void* q, const void* k, const void* v,
                                    const la_decay* decay, int normalize, void* out,
                                    int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                                    void* workspace, size_t workspace_bytes,
                                    la_stream_t stream);

/*
 * la_chunk_backward_workspace_size - scratch bytes that la_chunk_backward_ws
 * needs for these sizes (always > 0 for B*H > 0 and T > 0).
 */
LA_API size_t la_chunk_backward_workspace_size(int B, int H, int T, int Dk, int Dv,
                                               la_dtype dtype, int decay_kind);

/*
 * la_chunk_backward_ws - gradients of the unnormalised forward pass.
 *
 * For L = sum_t dy_t . y_t + <d_final_state, S_T> through la_chunk_forward
 * (normalize = 0), with dS_t = dL/dS_t (every later use of S_t included):
 *
 *   dS_t = q_t dy_t^T + g_{t+1} dS_{t+1},   dS_T = q_T dy_T^T + d_final_state
 *   dq_t = S_t dy_t        dk_t = dS_t v_t        dv_t = dS_t^T k_t
 *   d_init_state = g_1 dS_1
 *   d log g_t = g_t <dS_t, S_{t-1}>  =  sum_{s >= t} (q_s . dq_s - k_s . dk_s)
 *               + <d_final_state, S_T>
 *
 * The gradients of the scan are scans again (BlinkDL/RWKV-LM discussion 189,
 * fourth bullet: the gradient is computed with cumulative sums as well), and
 * the library runs them on its forward and reverse scan kernels:
 *   dq = forward scan of (q', k', v') = (dy, v, k) from S_0^T  (its state is S_t^T);
 *   dk = reverse scan of (v, dy, q) from d_final_state^T        (state dS_t^T);
 *   dv = reverse scan of (k, q, dy) from d_final_state          (state dS_t);
 * the reverse scans take the decay one token later (g_{t+1}, and 1 for the
 * last token).  The decay gradient is the suffix sum on the second line
 * (the identity <dS_t,S_t> - g_t <dS_t,S_{t-1}> = k_t . dk_t, summed from
 * the end).  Its bf16 error grows with the square root of the number of
 * summed tokens: each q . dq and k . dk carries the rounding of the bf16 dq
 * and dk it is formed from.
 *
 *   q, k, v, decay, init_state, B, H, T, Dk, Dv, dtype   as the forward call
 *                  (init_state NULL: zeros).
 *   dy             [B,H,T,Dv] `dtype`: dL/dy.  Required (for T > 0).
 *   d_final_state  NULL (zeros) or [B,H,Dk,Dv] fp32: dL/dS_T.
 *   dq, dk         [B,H,T,Dk] `dtype`; dv [B,H,T,Dv] `dtype`.  Required.
 *   d_log_g        NULL (not computed) or fp32 with the shape of decay->log_g:
 *                  [H] for a per-head decay (summed over b and t), [B,H,T]
 *                  for a per-step decay.  Must be NULL without a decay.
 *   d_init_state   NULL (not written) or [B,H,Dk,Dv] fp32: dL/dS_0.
 *   workspace      device memory of at least
 *                  la_chunk_backward_workspace_size(...) bytes, 16-byte
 *                  aligned, used on `stream` only.  Required (for T > 0).
 *
 * Several launches on `stream`: three scans (each possibly a state pass and
 * an output pass; the dv scan takes the dk scan's state pieces, transposed,
 * when the two scans cut T alike) and small kernels for the transposed
 * carried states, the shifted decay, d_init_state and d_log_g.  Outputs must
 * not overlap inputs or each other.
 *
 * Errors: as la_chunk_forward_ws, plus LA_ERR_INVALID_ARG for a NULL
 * required pointer (dy, dq, dk, dv, workspace), a workspace smaller than
 * la_chunk_backward_workspace_size or misaligned, or d_log_g given without a
 * decay.  The normalised forward's backward is la_chunk_backward_norm_ws.
 */
LA_API la_status la_chunk_backward_ws(const void* q, const void* k, const void* v,
                               const la_decay* decay, const float* init_state,
                               const void* dy, const float* d_final_state,
                               void* dq, void* dk, void* dv, float* d_log_g, float* d_init_state,
                               int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                               void* workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * la_chunk_forward_pro_ws - la_chunk_forward_ws on phi(q) * q_scale and
 * phi(k) (see la_prologue), with the prologue applied inside the kernels.
 *
 * The fp32 path applies both as it stages q and k (phi in fp32).  The bf16
 * tensor-core path applies the feature map to each Q and K tile in shared
 * memory once it has landed, before the tile's first MMA, at the tiles' own
 * precision (bf16 arithmetic; within a bf16 rounding step or two of phi
 * evaluated in fp32 and rounded), leaving the rows past the sequence end and
 * the columns past Dk at zero; it applies q_scale in its epilogue (the output
 * is linear in q, and the normalised output does not depend on the scale of
 * q).  Either way q and k cross HBM once, raw.
 *
 *   prologue        NULL (identity) or a descriptor.
 *   other arguments as la_chunk_forward_ws.
 *
 * Errors as la_chunk_forward_ws, plus LA_ERR_INVALID_ARG for a feature_map
 * out of range or a q_scale that is not finite.
 */
LA_API la_status la_chunk_forward_pro_ws(const void* q, const void* k, const void* v,
                                  const la_decay* decay, int normalize, const la_prologue* prologue,
                                  const float* init_state, const float* init_z,
                                  void* out, float* final_state, float* final_z,
                                  int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                                  void* workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * la_decode_step_pro - la_decode_step on phi(q) * q_scale and phi(k) (see
 * la_prologue), applied as the kernel stages this token's q and k: a
 * generation loop needs no separate feature-map launch per token.
 * Arguments and errors as la_decode_step, plus LA_ERR_INVALID_ARG for a
 * feature_map out of range or a q_scale that is not finite.
 */
LA_API la_status la_decode_step_pro(const void* q, const void* k, const void* v,
                             const la_decay* decay, int normalize, const la_prologue* prologue,
                             float* state, float* z, void* out,
                             int B, int H, int Dk, int Dv,
                             la_dtype dtype, la_stream_t stream);

/*
 * la_wkv4_forward - the RWKV-4 WKV recurrence (a different recurrence from
 * the one above: per channel, exponential key weights, a bonus for the
 * current token, no query).
 *
 * Source: BlinkDL/RWKV-LM issue 167, "Questions about formula 14 and code
 * implementation in the paper", the att_seq time loop in the opening
 * comment.  Per batch b and channel c, with time decay w[c] (natural log of
 * the per-step factor) and bonus u[c]:
 *
 *   wkv_t = ( sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u + k_t}     )
 *
 * (tokens counted from 0, plus the carried state's share).  The state is
 * the loop's (aa, bb, pp): the two sums are e^pp aa and e^pp bb, pp a running
 * log scale, so that only differences <= 0 are exponentiated and no large
 * key overflows.  Per token the loop first reads out (the state against the
 * current token at log weight u + k_t), then updates (the state decayed to
 * w + pp against the token at k_t, the larger log weight the new pp).
 * Computed in fp32 whatever the input type.
 *
 *   k, v, out      [B, T, C], `dtype` (LA_F32 or LA_BF16).  Required (T > 0).
 *   w, u           [C] fp32, finite.  Required.
 *   init_state     NULL (the empty state: aa = bb = 0, pp = -1e38) or
 *                  [B, 3, C] fp32, the planes aa, bb, pp.
 *   final_state    NULL (not written) or [B, 3, C] fp32; may be the same
 *                  buffer as init_state (each channel reads its state before
 *                  it writes it).
 *   B, T, C        batch, tokens, channels: B, T >= 0, C >= 1; B == 0 is a
 *                  no-op, T == 0 copies init_state (or the empty state) to
 *                  final_state.
 *
 * Layout note: channels are the fastest index, as in the page's
 * [T, C]-shaped k[t] and v[t] rows; each channel is an independent scan.
 *
 * Errors (synchronous, nothing enqueued): LA_ERR_INVALID_ARG for a NULL
 * required pointer, negative sizes, C < 1, k, v or out not 16-byte aligned,
 * w, u or a state not 4-byte aligned, a bad dtype; LA_ERR_UNSUPPORTED for C
 * not a multiple of 8 (bf16) or 4 (fp32) (the rows are moved as TMA tiles),
 * or B > 65535; LA_ERR_CUDA if a launch fails.
 */
LA_API la_status la_wkv4_forward(const void* k, const void* v, const float* w, const float* u,
                                 const float* init_state, void* out, float* final_state,
                                 int B, int T, int C, la_dtype dtype, la_stream_t stream);

/*
 * la_wkv4_workspace_size - scratch bytes la_wkv4_forward_ws can use for these
 * sizes (0 when the sequences would run as one segment).
 *
 * la_wkv4_forward_ws - la_wkv4_forward with caller-owned scratch.  Each
 * channel's loop is sequential in t, so B x C channels alone can leave the
 * GPU underused; with a workspace of at least la_wkv4_workspace_size bytes
 * the sequence is cut into T-segments: a first launch computes each earlier
 * segment's own (aa, bb, pp) from the empty state, the second starts every
 * segment from the initial state combined with them in order (decayed over
 * each segment's tokens, then added with the loop's own max-shifted
 * weighting).  Results equal the single pass up to fp32 rounding.
 *   workspace   NULL (one segment) or device memory, 16-byte aligned, used on
 *               `stream` only; a smaller size than la_wkv4_workspace_size
 *               runs one segment.  In place (final_state == init_state)
 *               stays allowed.
 * Other arguments and errors as la_wkv4_forward, plus LA_ERR_INVALID_ARG for
 * a misaligned workspace.
 */
LA_API size_t la_wkv4_workspace_size(int B, int T, int C, la_dtype dtype);
LA_API la_status la_wkv4_forward_ws(const void* k, const void* v, const float* w, const float* u,
                                    const float* init_state, void* out, float* final_state,
                                    int B, int T, int C, la_dtype dtype, void* workspace,
                                    size_t workspace_bytes, la_stream_t stream);

/*
 * la_chunk_backward_norm_workspace_size - scratch bytes that
 * la_chunk_backward_norm_ws needs (always > 0 for B*H > 0 and T > 0).
 */
LA_API size_t la_chunk_backward_norm_workspace_size(int B, int H, int T, int Dk, int Dv,
                                                    la_dtype dtype, int decay_kind);

/*
 * la_chunk_backward_norm_ws - gradients of the normalised forward pass
 * (normalize = 1): y_t = n_t / den_t with n_t = S_t^T q_t, den_t = q_t . z_t,
 * for L = sum_t dy_t . y_t + <d_final_state, S_T> + <d_final_z, z_T>.
 *
 * With dn_t = dy_t / den_t and dden_t = -(dy_t . n_t) / den_t^2:
 *   dq_t = S_t dn_t + dden_t z_t
 *   dS_t = q_t dn_t^T + g_{t+1} dS_{t+1}     dz_t = dden_t q_t + g_{t+1} dz_{t+1}
 *   dk_t = dS_t v_t + dz_t                   dv_t = dS_t^T k_t
 *   d_init_state = g_1 dS_1,  d_init_z = g_1 dz_1
 *   d log g_t = sum_{s >= t} (q_s . dq_s - k_s . dk_s) + <d_final_state, S_T>
 *               + <d_final_z, z_T>
 * All of it runs on the scan kernels, as in la_chunk_backward_ws: the
 * numerator and the denominator are recomputed by two forward scans (the
 * denominator as the scan of a 16-wide value panel whose first column is 1,
 * so that its state's first column is z_t), dn and dden by a small kernel,
 * and the key-sum terms dden_t z_t and dz_t by scans of 16-wide panels (the
 * second adds into dk); dq's two parts are added by a small kernel.
 *
 *   init_z         NULL (zeros) or z_0 [B,H,Dk] fp32; required with init_state.
 *   d_final_z      NULL (zeros) or dL/dz_T [B,H,Dk] fp32.
 *   d_init_z       NULL (not written) or [B,H,Dk] fp32: dL/dz_0.
 *   workspace      at least la_chunk_backward_norm_workspace_size(...) bytes.
 *   other arguments as la_chunk_backward_ws.
 *
 * Errors as la_chunk_backward_ws, plus LA_ERR_INVALID_ARG for init_state
 * without init_z.
 */
LA_API la_status la_chunk_backward_norm_ws(const void* q, const void* k, const void* v,
                                    const la_decay* decay, const float* init_state, const float* init_z,
                                    const void* dy, const float* d_final_state, const float* d_final_z,
                                    void* dq, void* dk, void* dv, float* d_log_g,
                                    float* d_init_state, float* d_init_z,
                                    int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                                    void* workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * la_ema_scan - the cumulative exponential moving average: element-wise
 * values and factors scanned along T per channel.
 *
 * Source: Jamie-Stirling/RetNet issue 21, "Proposed improvement/
 * collaboration: removing the O(T^2) training cost", cumulative_ema(values,
 * factors, reverse): each output is the previous output times this step's
 * factor plus this step's value (the listing's pairing operator
 * (xa, fa) o (xb, fb) = (xa fb + xb, fa fb)); with reverse, the non-reversed
 * scan of the time-reversed arguments, reversed back.  Per batch b and
 * channel c, with s the carried state:
 *
 *   forward:  s <- f_t s + x_t,  out_t = s,   t = 0 .. T-1
 *   reverse:  s <- f_t s + x_t,  out_t = s,   t = T-1 .. 0
 *
 * The page's retention(Q, K, gamma, V) runs this scan over K (x) V with
 * factors gamma; la_chunk_forward is the fused form of that path.  Computed
 * in fp32 whatever the input type.
 *
 *   x, f, out      [B, T, C], `dtype` (LA_F32 or LA_BF16), channels fastest.
 *                  Required (T > 0).
 *   init_state     NULL (0) or [B, C] fp32: the state before the first scanned step.
 *   final_state    NULL (not written) or [B, C] fp32: the state after the
 *                  last scanned step; may be the same buffer as init_state.
 *   reverse        0 forward, 1 reverse.
 *   B, T, C        B, T >= 0, C >= 1; B == 0 is a no-op, T == 0 copies
 *                  init_state (or 0) to final_state.
 *
 * Errors (synchronous, nothing enqueued): LA_ERR_INVALID_ARG for a NULL
 * required pointer, negative sizes, C < 1, x, f or out not 16-byte aligned,
 * a state not 4-byte aligned, a bad dtype; LA_ERR_UNSUPPORTED for C not a
 * multiple of 8 (bf16) or 4 (fp32), or B > 65535; LA_ERR_CUDA if a launch
 * fails.
 */
LA_API la_status la_ema_scan(const void* x, const void* f, const float* init_state, void* out,
                             float* final_state, int B, int T, int C, la_dtype dtype, int reverse,
                             la_stream_t stream);

/*
 * la_chunk_forward_noalloc - la_chunk_forward_ws whose workspace is a fixed
 * device array inside this library (la_chunk_forward_noalloc_capacity()
 * bytes, 16 MiB, one per device, reserved when the library's device code is
 * loaded), so that the call itself allocates no device memory.  The pages
 * have no counterpart: this is a property of this library's interface only.
 *
 * It is meant for callers that cannot allocate device memory at the point
 * of the call: code that runs under a fixed memory budget or behind its own
 * allocator that must not be bypassed, or host code that must not call
 * cudaMalloc at all (it can synchronise the device and is not allowed in
 * some contexts, such as while a stream is being captured).
 *
 * The array is shared by every call on a device and keeps what the last call
 * left in it (every call writes the parts it reads before reading them):
 * calls on one device that overlap in time on the GPU race on it, so issue
 * them on one stream, or synchronise between the streams.  The array's
 * device address is looked up (cudaGetSymbolAddress) by the first call on
 * each device, with that device current, and again only if that device's
 * context has been reset since; make that first call before any stream
 * capture begins.  Arguments, results and errors as la_chunk_forward, plus
 * LA_ERR_UNSUPPORTED (nothing enqueued) when these sizes would need a larger
 * workspace than the array holds (la_chunk_forward_workspace_size), and
 * LA_ERR_CUDA if the array's address cannot be obtained on the current device.
 */
LA_API la_status la_chunk_forward_noalloc(const void* q, const void* k, const void* v,
                                   const la_decay* decay, int normalize,
                                   const float* init_state, const float* init_z,
                                   void* out, float* final_state, float* final_z,
                                   int B, int H, int T, int Dk, int Dv,
                                   la_dtype dtype, la_stream_t stream);

/* Bytes of the fixed device array that la_chunk_forward_noalloc uses. */
LA_API size_t la_chunk_forward_noalloc_capacity(void);

/*
 * la_decode_step - one token of the recurrence, state updated in place.
 *
 *   S <- g S + k v^T;  z <- g z + k (if normalize);  out = q^T S  (/ q^T z).
 *
 * This is the token-by-token inference path that carries the KV state and,
 * with normalisation, the key sum between calls (flash-linear-attention
 * issue 268: the generation case where only the last token is passed).
 *
 *   q, k           [B,H,Dk], `dtype`.  v, out: [B,H,Dv], `dtype`.
 *   decay          NULL, LA_DECAY_PER_HEAD (log_g [H]) or LA_DECAY_PER_STEP
 *                  (log_g [B,H], this token's decay).
 *   state          [B,H,Dk,Dv] fp32, read and written in place.  Required.
 *   z              [B,H,Dk] fp32, read and written in place.  Required if
 *                  normalize, ignored otherwise.
 *
 * Errors as for la_chunk_forward; LA_ERR_UNSUPPORTED if Dk or Dv > 128.
 */
LA_API la_status la_decode_step(const void* q, const void* k, const void* v,
                         const la_decay* decay, int normalize,
                         float* state, float* z, void* out,
                         int B, int H, int Dk, int Dv,
                         la_dtype dtype, la_stream_t stream);

/* A static string naming a status code. */
LA_API const char* la_status_string(la_status status);

/*
 * la_device_error - reads and clears the device error word of the current
 * device.  *code receives 0 if no kernel of this library gave up since the
 * last call, else a nonzero code naming the wait that timed out.  Synchronises
 * with `stream` first.  Returns LA_ERR_CUDA if that fails.
 */
LA_API la_status la_device_error(int* code, la_stream_t stream);

/* Library version, "MAJOR.MINOR.PATCH". */
LA_API const char* la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RETENTION_SCAN_B200_LA_H */
