// la_api.cu - the C ABI (include/la.h): argument validation, dispatch to the
// kernels, the device error word.  Nothing here allocates device memory.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "la.h"
#include "la_internal.h"

namespace {

// Set by a kernel that gave up waiting on one of its barriers (kErr* codes).
__device__ int g_err_word;

constexpr int kMaxDevices = 64;
std::atomic<int*> g_err_ptr[kMaxDevices];

int* err_word_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    int* p = g_err_ptr[dev].load();
    if (!p) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_err_word) != cudaSuccess) return nullptr;
        p = static_cast<int*>(addr);
        g_err_ptr[dev].store(p);
    }
    return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Host-side fault injection for tests: LA_FAULT_INJECT=launch makes every
// compute entry point report a failed launch without enqueuing anything.
bool launch_fault_injected() {
    const char* e = std::getenv("LA_FAULT_INJECT");
    return e && std::strcmp(e, "launch") == 0;
}

bool fits_int(long long x) { return x >= 0 && x <= INT_MAX; }

la_status check_prologue(const la_prologue* pro, int* fmap, float* qscale) {
    *fmap = LA_FEATURE_NONE;
    *qscale = 1.f;
    if (!pro) return LA_OK;
    if (pro->feature_map < LA_FEATURE_NONE || pro->feature_map > LA_FEATURE_ELU1) return LA_ERR_INVALID_ARG;
    if (!std::isfinite(pro->q_scale)) return LA_ERR_INVALID_ARG;
    *fmap = pro->feature_map;
    *qscale = pro->q_scale;
    return LA_OK;
}

la_status check_decay(const la_decay* decay, int* kind, const float** log_g) {
    *kind = LA_DECAY_NONE;
    *log_g = nullptr;
    if (!decay) return LA_OK;
    if (decay->kind < LA_DECAY_NONE || decay->kind > LA_DECAY_PER_STEP) return LA_ERR_INVALID_ARG;
    *kind = decay->kind;
    if (*kind != LA_DECAY_NONE) {
        if (!decay->log_g || !aligned4(decay->log_g)) return LA_ERR_INVALID_ARG;
        *log_g = decay->log_g;
    }
    return LA_OK;
}

// One whole-sequence scan, forward (t = 1..T) or reverse (t = T..1), its
// outputs written to out or (accumulate) added to the values already there.
la_status scan(const void* q, const void* k, const void* v, const la_decay* decay, int normalize,
               const float* init_state, const float* init_z, void* out, float* final_state, float* final_z,
               int B, int H, int T, int Dk, int Dv, la_dtype dtype, void* workspace, size_t workspace_bytes,
               la_stream_t stream, int reverse, int accumulate, const la_prologue* pro = nullptr) {
    if (B < 0 || H < 0 || T < 0 || Dk < 1 || Dv < 1) return LA_ERR_INVALID_ARG;
    int fmap;
    float qscale;
    if (check_prologue(pro, &fmap, &qscale) != LA_OK) return LA_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    int kind;
    const float* log_g;
    if (check_decay(decay, &kind, &log_g) != LA_OK) return LA_ERR_INVALID_ARG;
    normalize = normalize ? 1 : 0;
    if (normalize && init_state && !init_z) return LA_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(B) * H;
    if (!fits_int(BH * 8)) return LA_ERR_INVALID_ARG;
    for (const void* p : {static_cast<const void*>(init_state), static_cast<const void*>(final_state)})
        if (p && !aligned16(p)) return LA_ERR_INVALID_ARG;
    if (normalize)
        for (const void* p : {static_cast<const void*>(init_z), static_cast<const void*>(final_z)})
            if (p && !aligned16(p)) return LA_ERR_INVALID_ARG;
    if (BH > 0 && T > 0) {
        if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    }
    if (dtype == LA_F32 && (Dk > 128 || Dv > 128)) return LA_ERR_UNSUPPORTED;
    if (dtype == LA_BF16 && !la::fwd_tc_supports(Dk, Dv)) return LA_ERR_UNSUPPORTED;
    if (dtype == LA_BF16 && fmap != LA_FEATURE_NONE) return LA_ERR_UNSUPPORTED;  // see la.h
    if (BH == 0) return LA_OK;
    if (launch_fault_injected()) return LA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    if (T == 0) {  // empty sequence: the carried state passes through unchanged
        const size_t sbytes = sizeof(float) * static_cast<size_t>(BH) * Dk * Dv;
        const size_t zbytes = sizeof(float) * static_cast<size_t>(BH) * Dk;
        cudaError_t e = cudaSuccess;
        if (final_state)
            e = init_state ? cudaMemcpyAsync(final_state, init_state, sbytes, cudaMemcpyDeviceToDevice, s)
                           : cudaMemsetAsync(final_state, 0, sbytes, s);
        if (e == cudaSuccess && normalize && final_z)
            e = init_z ? cudaMemcpyAsync(final_z, init_z, zbytes, cudaMemcpyDeviceToDevice, s)
                       : cudaMemsetAsync(final_z, 0, zbytes, s);
        return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
    }

    la::FwdArgs a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.decay_kind = kind;
    a.log_g = log_g;
    a.normalize = normalize;
    a.init_state = init_state;
    a.init_z = normalize ? init_z : nullptr;
    a.out = out;
    a.final_state = final_state;
    a.final_z = normalize ? final_z : nullptr;
    a.B = B;
    a.H = H;
    a.T = T;
    a.Dk = Dk;
    a.Dv = Dv;
    a.stream = s;
    a.err_word = err_word_for_current_device();
    a.reverse = reverse;
    a.accumulate = accumulate;
    a.feature_map = fmap;
    a.q_scale = qscale;
    cudaError_t e;
    if (dtype == LA_F32) {
        e = la::launch_fwd_f32(a);
    } else {
        a.workspace = workspace;
        a.workspace_bytes = workspace ? workspace_bytes : 0;
        e = la::launch_fwd_tc(a, nullptr, nullptr);
        if (e == cudaErrorNotSupported) return LA_ERR_UNSUPPORTED;
    }
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

// Scratch of the backward pass, in 256-byte aligned regions (every optional
// region is reserved, so that the size depends on the sizes only):
//   S_0^T, d_final_state^T, S_T^T   [B,H,Dv,Dk] fp32 each
//   shifted log decay               [B,H,T] fp32 (with a decay)
//   decay-gradient scratch          la::dlog_scratch_doubles doubles
//   T-segment workspace of the scans (the larger of the two key/value widths' orders)
struct BwdLayout {
    size_t s0t, dsft, st, lsh, dlog, scan, scan_bytes, total;
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

BwdLayout bwd_layout(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int kind) {
    const size_t BH = static_cast<size_t>(B) * H;
    const size_t state = round256(sizeof(float) * BH * Dk * Dv);
    BwdLayout L{};
    L.s0t = 0;
    L.dsft = L.s0t + state;
    L.st = L.dsft + state;
    L.lsh = L.st + state;
    L.dlog = L.lsh + (kind != LA_DECAY_NONE ? round256(sizeof(float) * BH * T) : 0);
    L.scan = L.dlog + round256(sizeof(double) * la::dlog_scratch_doubles(B, H, T));
    L.scan_bytes = 0;
    if (dtype == LA_BF16) {
        const size_t a = la::fwd_tc_workspace_bytes(B, H, T, Dv, Dk, false);  // dq, dk scans
        const size_t b = la::fwd_tc_workspace_bytes(B, H, T, Dk, Dv, false);  // dv scan
        L.scan_bytes = round256(a > b ? a : b);
    }
    L.total = L.scan + L.scan_bytes;
    return L;
}

}  // namespace

extern "C" {

const char* la_status_string(la_status status) {
    switch (status) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: no kernel for this shape or dtype";
        case LA_ERR_CUDA: return "LA_ERR_CUDA: a CUDA call or kernel launch failed";
    }
    return "unknown la_status";
}

const char* la_version(void) { return "0.1.0"; }

size_t la_chunk_forward_workspace_size(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int normalize) {
    if (dtype != LA_BF16 || B < 1 || H < 1 || T < 1) return 0;
    if (!fits_int(static_cast<long long>(B) * H * 8)) return 0;
    return la::fwd_tc_workspace_bytes(B, H, T, Dk, Dv, normalize != 0);
}

la_status la_chunk_forward(const void* q, const void* k, const void* v, const la_decay* decay, int normalize,
                           const float* init_state, const float* init_z, void* out, float* final_state,
                           float* final_z, int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                           la_stream_t stream) {
    return la_chunk_forward_ws(q, k, v, decay, normalize, init_state, init_z, out, final_state, final_z, B, H, T,
                               Dk, Dv, dtype, nullptr, 0, stream);
}

la_status la_chunk_forward_ws(const void* q, const void* k, const void* v, const la_decay* decay, int normalize,
                              const float* init_state, const float* init_z, void* out, float* final_state,
                              float* final_z, int B, int H, int T, int Dk, int Dv, la_dtype dtype, void* workspace,
                              size_t workspace_bytes, la_stream_t stream) {
    return scan(q, k, v, decay, normalize, init_state, init_z, out, final_state, final_z, B, H, T, Dk, Dv, dtype,
                workspace, workspace_bytes, stream, 0, 0);
}

la_status la_chunk_forward_pro_ws(const void* q, const void* k, const void* v, const la_decay* decay, int normalize,
                                  const la_prologue* prologue, const float* init_state, const float* init_z, void* out,
                                  float* final_state, float* final_z, int B, int H, int T, int Dk, int Dv,
                                  la_dtype dtype, void* workspace, size_t workspace_bytes, la_stream_t stream) {
    return scan(q, k, v, decay, normalize, init_state, init_z, out, final_state, final_z, B, H, T, Dk, Dv, dtype,
                workspace, workspace_bytes, stream, 0, 0, prologue);
}

la_status la_chunk_reverse_ws(const void* q, const void* k, const void* v, const la_decay* decay, int normalize,
                              const float* init_state, const float* init_z, void* out, float* final_state,
                              float* final_z, int B, int H, int T, int Dk, int Dv, la_dtype dtype, void* workspace,
                              size_t workspace_bytes, la_stream_t stream) {
    return scan(q, k, v, decay, normalize, init_state, init_z, out, final_state, final_z, B, H, T, Dk, Dv, dtype,
                workspace, workspace_bytes, stream, 1, 0);
}

la_status la_chunk_bidirectional_ws(const void* q, const void* k, const void* v, const la_decay* decay,
                                    int normalize, void* out, int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                                    void* workspace, size_t workspace_bytes, la_stream_t stream) {
    // the reverse scan's launch is not enqueued unless the forward one was;
    // the arguments are checked once, by the first call
    const la_status st = scan(q, k, v, decay, normalize, nullptr, nullptr, out, nullptr, nullptr, B, H, T, Dk, Dv,
                              dtype, workspace, workspace_bytes, stream, 0, 0);
    if (st != LA_OK) return st;
    return scan(q, k, v, decay, normalize, nullptr, nullptr, out, nullptr, nullptr, B, H, T, Dk, Dv, dtype,
                workspace, workspace_bytes, stream, 1, 1);
}

size_t la_chunk_backward_workspace_size(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int decay_kind) {
    if ((dtype != LA_F32 && dtype != LA_BF16) || B < 1 || H < 1 || T < 1 || Dk < 1 || Dv < 1) return 0;
    if (decay_kind < LA_DECAY_NONE || decay_kind > LA_DECAY_PER_STEP) return 0;
    if (!fits_int(static_cast<long long>(B) * H * 8)) return 0;
    return bwd_layout(B, H, T, Dk, Dv, dtype, decay_kind).total;
}

// dq, dk, dv by three scans on the forward and reverse scan kernels (the
// header explains the permutations), then d_init_state and d_log_g.
la_status la_chunk_backward_ws(const void* q, const void* k, const void* v, const la_decay* decay,
                               const float* init_state, const void* dy, const float* d_final_state, void* dq,
                               void* dk, void* dv, float* d_log_g, float* d_init_state, int B, int H, int T, int Dk,
                               int Dv, la_dtype dtype, void* workspace, size_t workspace_bytes,
                               la_stream_t stream) {
    if (B < 0 || H < 0 || T < 0 || Dk < 1 || Dv < 1) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    int kind;
    const float* log_g;
    if (check_decay(decay, &kind, &log_g) != LA_OK) return LA_ERR_INVALID_ARG;
    if (d_log_g && (kind == LA_DECAY_NONE || !aligned4(d_log_g))) return LA_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(B) * H;
    if (!fits_int(BH * 8) || BH > 65535) return BH > 65535 ? LA_ERR_UNSUPPORTED : LA_ERR_INVALID_ARG;
    for (const void* p : {static_cast<const void*>(init_state), static_cast<const void*>(d_final_state),
                          static_cast<const void*>(d_init_state)})
        if (p && !aligned16(p)) return LA_ERR_INVALID_ARG;
    const bool work = BH > 0 && T > 0;
    if (work) {
        for (const void* p : {q, k, v, dy, static_cast<const void*>(dq), static_cast<const void*>(dk),
                              static_cast<const void*>(dv), static_cast<const void*>(workspace)})
            if (!p || !aligned16(p)) return LA_ERR_INVALID_ARG;
    }
    if (dtype == LA_F32 && (Dk > 128 || Dv > 128)) return LA_ERR_UNSUPPORTED;
    if (dtype == LA_BF16 && !la::fwd_tc_supports(Dk, Dv)) return LA_ERR_UNSUPPORTED;
    if (work && (T + 255) / 256 > 65535) return LA_ERR_UNSUPPORTED;
    const BwdLayout L = work ? bwd_layout(B, H, T, Dk, Dv, dtype, kind) : BwdLayout{};
    if (work && workspace_bytes < L.total) return LA_ERR_INVALID_ARG;
    if (BH == 0) return LA_OK;
    if (launch_fault_injected()) return LA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t sbytes = sizeof(float) * static_cast<size_t>(BH) * Dk * Dv;

    if (T == 0) {  // S_T = S_0: the state gradient passes through; no decay was applied
        cudaError_t e = cudaSuccess;
        if (d_init_state)
            e = d_final_state ? cudaMemcpyAsync(d_init_state, d_final_state, sbytes, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(d_init_state, 0, sbytes, s);
        if (e == cudaSuccess && d_log_g && kind == LA_DECAY_PER_HEAD)
            e = cudaMemsetAsync(d_log_g, 0, sizeof(float) * H, s);
        return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
    }

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* s0t = init_state ? reinterpret_cast<float*>(ws + L.s0t) : nullptr;
    float* dsft = d_final_state ? reinterpret_cast<float*>(ws + L.dsft) : nullptr;
    const bool need_st = d_log_g && d_final_state;  // <d_final_state, S_T> enters d_log_g
    float* st = need_st ? reinterpret_cast<float*>(ws + L.st) : nullptr;
    float* lsh = kind != LA_DECAY_NONE ? reinterpret_cast<float*>(ws + L.lsh) : nullptr;
    void* scan_ws = L.scan_bytes ? ws + L.scan : nullptr;
    const int bh = static_cast<int>(BH);
    auto cuda_ok = [](cudaError_t e) { return e == cudaSuccess; };

    if (s0t && !cuda_ok(la::launch_transpose(init_state, s0t, bh, Dk, Dv, s))) return LA_ERR_CUDA;
    if (dsft && !cuda_ok(la::launch_transpose(d_final_state, dsft, bh, Dk, Dv, s))) return LA_ERR_CUDA;
    if (lsh && !cuda_ok(la::launch_shift_decay(log_g, kind, lsh, B, H, T, s))) return LA_ERR_CUDA;
    const la_decay shifted{LA_DECAY_PER_STEP, lsh};
    const la_decay* rdecay = lsh ? &shifted : nullptr;

    // dq = forward scan of (dy, v, k) from S_0^T; its final state is S_T^T
    la_status r = scan(dy, v, k, decay, 0, s0t, nullptr, dq, st, nullptr, B, H, T, Dv, Dk, dtype, scan_ws,
                       L.scan_bytes, stream, 0, 0);
    if (r != LA_OK) return r;
    // dk = reverse scan of (v, dy, q) from d_final_state^T, decay one token later
    r = scan(v, dy, q, rdecay, 0, dsft, nullptr, dk, nullptr, nullptr, B, H, T, Dv, Dk, dtype, scan_ws,
             L.scan_bytes, stream, 1, 0);
    if (r != LA_OK) return r;
    // dv = reverse scan of (k, q, dy) from d_final_state; its final state is dS_1
    r = scan(k, q, dy, rdecay, 0, d_final_state, nullptr, dv, d_init_state, nullptr, B, H, T, Dk, Dv, dtype,
             scan_ws, L.scan_bytes, stream, 1, 0);
    if (r != LA_OK) return r;
    if (d_init_state && kind != LA_DECAY_NONE &&
        !cuda_ok(la::launch_scale_by_first_decay(d_init_state, log_g, kind, B, H, T, Dk * Dv, s)))
        return LA_ERR_CUDA;
    if (d_log_g) {
        la::DlogArgs a{};
        a.q = q;
        a.k = k;
        a.dq = dq;
        a.dk = dk;
        a.d_final_state = d_final_state;
        a.final_state_t = st;
        a.d_log_g = d_log_g;
        a.kind = kind;
        a.B = B;
        a.H = H;
        a.T = T;
        a.Dk = Dk;
        a.Dv = Dv;
        a.dtype = dtype;
        a.scratch = reinterpret_cast<double*>(ws + L.dlog);
        a.stream = s;
        if (!cuda_ok(la::launch_dlog(a))) return LA_ERR_CUDA;
    }
    return LA_OK;
}

size_t la_wkv4_workspace_size(int B, int T, int C, la_dtype dtype) {
    if ((dtype != LA_F32 && dtype != LA_BF16) || B < 1 || T < 1 || C < 1 || B > 65535) return 0;
    if (!fits_int(static_cast<long long>(T) * C) || !fits_int(3LL * B * C)) return 0;
    return la::wkv4_workspace_bytes(B, T, C, dtype);
}

la_status la_wkv4_forward(const void* k, const void* v, const float* w, const float* u, const float* init_state,
                          void* out, float* final_state, int B, int T, int C, la_dtype dtype, la_stream_t stream) {
    return la_wkv4_forward_ws(k, v, w, u, init_state, out, final_state, B, T, C, dtype, nullptr, 0, stream);
}

la_status la_wkv4_forward_ws(const void* k, const void* v, const float* w, const float* u, const float* init_state,
                             void* out, float* final_state, int B, int T, int C, la_dtype dtype, void* workspace,
                             size_t workspace_bytes, la_stream_t stream) {
    if (B < 0 || T < 0 || C < 1) return LA_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (!w || !u || !aligned4(w) || !aligned4(u)) return LA_ERR_INVALID_ARG;
    if ((init_state && !aligned4(init_state)) || (final_state && !aligned4(final_state))) return LA_ERR_INVALID_ARG;
    if (B > 0 && T > 0) {
        if (!k || !v || !out) return LA_ERR_INVALID_ARG;
        if (!aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    }
    // rows of k and v are TMA tiles: their byte stride must be a multiple of 16
    if (C % (dtype == LA_BF16 ? 8 : 4) != 0) return LA_ERR_UNSUPPORTED;
    if (B > 65535 || !fits_int(static_cast<long long>(T) * C) ||
        !fits_int(3LL * B * C))
        return LA_ERR_UNSUPPORTED;
    if (B == 0) return LA_OK;
    if (launch_fault_injected()) return LA_ERR_CUDA;
    la::Wkv4Args a{};
    a.k = k;
    a.v = v;
    a.w = w;
    a.u = u;
    a.init_state = init_state;
    a.out = out;
    a.final_state = final_state;
    a.B = B;
    a.T = T;
    a.C = C;
    a.dtype = dtype;
    a.err_word = err_word_for_current_device();
    a.workspace = workspace;
    a.workspace_bytes = workspace ? workspace_bytes : 0;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    return la::launch_wkv4(a) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_decode_step(const void* q, const void* k, const void* v, const la_decay* decay, int normalize,
                         float* state, float* z, void* out, int B, int H, int Dk, int Dv, la_dtype dtype,
                         la_stream_t stream) {
    return la_decode_step_pro(q, k, v, decay, normalize, nullptr, state, z, out, B, H, Dk, Dv, dtype, stream);
}

la_status la_decode_step_pro(const void* q, const void* k, const void* v, const la_decay* decay, int normalize,
                             const la_prologue* prologue, float* state, float* z, void* out, int B, int H, int Dk,
                             int Dv, la_dtype dtype, la_stream_t stream) {
    int fmap;
    float qscale;
    if (check_prologue(prologue, &fmap, &qscale) != LA_OK) return LA_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || Dk < 1 || Dv < 1) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    int kind;
    const float* log_g;
    if (check_decay(decay, &kind, &log_g) != LA_OK) return LA_ERR_INVALID_ARG;
    normalize = normalize ? 1 : 0;
    const long long BH = static_cast<long long>(B) * H;
    if (!fits_int(BH)) return LA_ERR_INVALID_ARG;
    if (BH > 0) {
        if (!q || !k || !v || !out || !state) return LA_ERR_INVALID_ARG;
        if (normalize && !z) return LA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
            return LA_ERR_INVALID_ARG;
        if (normalize && !aligned16(z)) return LA_ERR_INVALID_ARG;
    }
    if (Dk > 128 || Dv > 128) return LA_ERR_UNSUPPORTED;
    if (BH == 0) return LA_OK;
    if (launch_fault_injected()) return LA_ERR_CUDA;
    la::DecodeArgs a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.decay_kind = kind;
    a.log_g = log_g;
    a.normalize = normalize;
    a.state = state;
    a.z = normalize ? z : nullptr;
    a.out = out;
    a.B = B;
    a.H = H;
    a.Dk = Dk;
    a.Dv = Dv;
    a.feature_map = fmap;
    a.q_scale = qscale;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    return la::launch_decode(a, dtype) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_device_error(int* code, la_stream_t stream) {
    if (!code) return LA_ERR_INVALID_ARG;
    *code = 0;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return LA_ERR_CUDA;
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof(int)) != cudaSuccess) return LA_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_err_word, &zero, sizeof(int)) != cudaSuccess) return LA_ERR_CUDA;
    *code = v;
    return LA_OK;
}

}  // extern "C"
