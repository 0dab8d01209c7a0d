// la_api.cu - the C ABI (include/la.h): argument validation, dispatch to the
// kernels, the device error word.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <mutex>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "la.h"
#include "la_internal.h"

namespace la {
namespace {

constexpr int kMaxDevices = 64;

// cuCtxGetCurrent, looked up once through the runtime (libcuda is not linked).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
    static std::atomic<CtxGetCurrentFn> fn{nullptr};
    CtxGetCurrentFn f = fn.load();
    if (!f) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f = reinterpret_cast<CtxGetCurrentFn>(ptr);
        fn.store(f);
    }
    return f;
}

void* current_context() {
    CtxGetCurrentFn f = ctx_get_current();
    CUcontext c = nullptr;
    if (!f || f(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

struct SymbolEntry {
    void* ctx;
    void* addr;
};
std::mutex g_sym_mutex;
SymbolEntry g_sym[kSymSlots][kMaxDevices];

}  // namespace

void* device_symbol_address(const void* symbol, int slot) {
    int dev = 0;
    if (slot < 0 || slot >= kSymSlots || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_sym_mutex);
    SymbolEntry& e = g_sym[slot][dev];
    void* ctx = current_context();
    if (e.addr && ctx && e.ctx == ctx) return e.addr;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, symbol) != cudaSuccess) return nullptr;
    e.ctx = current_context();  // the lookup made the device's primary context current if none was
    e.addr = addr;
    return addr;
}

}  // namespace la

namespace {

// Set by a kernel that gave up waiting on one of its barriers (kErr* codes).
__device__ int g_err_word;

int* err_word_for_current_device() { return static_cast<int*>(la::device_symbol_address(&g_err_word, la::kSymErrWord)); }

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
               la_stream_t stream, int reverse, int accumulate, const la_prologue* pro = nullptr,
               int states_ready = 0) {
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
    a.states_ready = states_ready;
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
    size_t s0t, dsft, st, lsh, dlog, scan, scan_bytes, scan2, scan2_bytes, total;
    int shared_pieces;  // state pieces per (b, h) that the dk and dv scans share (0: none)
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// share_states (the unnormalised backward): the dk and dv reverse scans
// compute the same state, transposed (sum q dy^T and sum dy q^T, with the
// same decay); when their plans cut T alike, the dv scan takes the dk scan's
// state pieces, transposed into a second scan workspace, instead of running
// its own state pass.
BwdLayout bwd_layout(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int kind, bool share_states = false) {
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
        long long key_k = 0, key_v = 0;
        const int nk = la::fwd_tc_state_pieces(B, H, T, Dv, Dk, false, &key_k);
        const int nv = la::fwd_tc_state_pieces(B, H, T, Dk, Dv, false, &key_v);
        if (share_states && nk > 0 && nk == nv && key_k == key_v) {
            L.shared_pieces = nk;
            L.scan2_bytes = round256(b);
        }
    }
    L.scan2 = L.scan + L.scan_bytes;
    L.total = L.scan2 + L.scan2_bytes;
    return L;
}

// Scratch of the normalised backward: the unnormalised backward's regions,
// then the key-sum panels (fp32: z_0 as a [Dk][16] and a [16][Dk] panel,
// d_final_z as [16][Dk], the recomputed z_T as [Dk][16], dz_1 as [16][Dk])
// and the per-token arrays (`dtype`): the ones panel, the denominator panel,
// the numerator n, dn, the dden panel and the key-sum part of dq.
struct NormLayout {
    BwdLayout base;
    size_t z0p, z0t, dzft, ztp, dz1p, ones, denp, y, dn, ddp, scan, scan_bytes, total;
};

NormLayout norm_layout(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int kind) {
    NormLayout L{};
    L.base = bwd_layout(B, H, T, Dk, Dv, dtype, kind);
    const size_t BH = static_cast<size_t>(B) * H, es = dtype == LA_BF16 ? 2 : 4;
    const size_t panel = round256(sizeof(float) * BH * Dk * 16);
    const size_t tok16 = round256(es * BH * T * 16);
    L.z0p = L.base.scan;  // after the unnormalised regions (whose own scan area moves to the end)
    L.z0t = L.z0p + panel;
    L.dzft = L.z0t + panel;
    L.ztp = L.dzft + panel;
    L.dz1p = L.ztp + panel;
    L.ones = L.dz1p + panel;
    L.denp = L.ones + tok16;
    L.y = L.denp + tok16;
    L.dn = L.y + round256(es * BH * T * Dv);
    L.ddp = L.dn + round256(es * BH * T * Dv);
    L.scan = L.ddp + tok16;
    L.scan_bytes = 0;
    if (dtype == LA_BF16) {
        const int dims[5][3] = {{Dk, Dv, 1}, {Dk, 16, 0}, {Dv, Dk, 0}, {16, Dk, 0}, {Dk, Dv, 0}};
        for (const auto& d : dims) {
            const size_t b = la::fwd_tc_workspace_bytes(B, H, T, d[0], d[1], d[2] != 0);
            if (b > L.scan_bytes) L.scan_bytes = b;
        }
        L.scan_bytes = round256(L.scan_bytes);
    }
    L.total = L.scan + L.scan_bytes;
    return L;
}

// The normalised backward with the value panel [v | 1 | 0] (W = Dv + 16 for
// bf16, Dv + 1 for fp32): one scan gives [n | den], and dq, dk each come from one scan
// of [dn | dden | 0] against it, so that the cancellation between the
// numerator's and the denominator's terms happens inside the scores (fp32)
// instead of between two rounded outputs.  Regions (256-aligned): the
// unnormalised layout's shifted decay and decay-gradient scratch, then fp32
// state panels [S_0 | z_0], its transpose, [dSf | dzf], its transpose, the
// final state of the first scan and of the dk scan, then per-token arrays
// (`dtype`): the value panel, [n | den], [dn | dden], dn, and the scans'
// T-segment workspace.
int panel_width(int Dv, la_dtype dtype) {
    if (dtype == LA_F32) return Dv + 1 <= 128 ? Dv + 1 : 0;
    return Dv + 16 <= 128 ? Dv + 16 : 0;  // bf16 widths are multiples of 16
}

struct PanelLayout {
    BwdLayout base;
    int W;
    size_t ainit, binit, dpan, cinit, f1, f4, pk, nd, pq, dn, scan, scan_bytes, total;
};

PanelLayout panel_layout(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int kind) {
    PanelLayout L{};
    L.base = bwd_layout(B, H, T, Dk, Dv, dtype, kind);
    L.W = panel_width(Dv, dtype);
    const size_t BH = static_cast<size_t>(B) * H, es = dtype == LA_BF16 ? 2 : 4, W = L.W;
    const size_t sp = round256(sizeof(float) * BH * Dk * W);
    const size_t tw = round256(es * BH * T * W);
    L.ainit = L.base.scan;
    L.binit = L.ainit + sp;
    L.dpan = L.binit + sp;
    L.cinit = L.dpan + sp;
    L.f1 = L.cinit + sp;
    L.f4 = L.f1 + sp;
    L.pk = L.f4 + sp;
    L.nd = L.pk + tw;
    L.pq = L.nd + tw;
    L.dn = L.pq + tw;
    L.scan = L.dn + round256(es * BH * T * Dv);
    L.scan_bytes = 0;
    if (dtype == LA_BF16) {
        const int dims[4][2] = {{Dk, L.W}, {L.W, Dk}, {Dk, Dv}, {Dv, Dk}};
        for (const auto& d : dims) {
            const size_t b = la::fwd_tc_workspace_bytes(B, H, T, d[0], d[1], false);
            if (b > L.scan_bytes) L.scan_bytes = b;
        }
        L.scan_bytes = round256(L.scan_bytes);
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

size_t la_chunk_state_workspace_size(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int normalize) {
    if (dtype != LA_BF16 || B < 1 || H < 1 || T < 1) return 0;
    if (!fits_int(static_cast<long long>(B) * H * 8)) return 0;
    return la::fwd_state_workspace_bytes(B, H, T, Dk, Dv, normalize != 0);
}

la_status la_chunk_state_ws(const void* k, const void* v, const la_decay* decay, int normalize, float* state_out,
                            float* z_out, float* log_g_total, int B, int H, int T, int Dk, int Dv, la_dtype dtype,
                            void* workspace, size_t workspace_bytes, la_stream_t stream) {
    if (B < 0 || H < 0 || T < 0 || Dk < 1 || Dv < 1) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return LA_ERR_INVALID_ARG;
    int kind;
    const float* log_g;
    if (check_decay(decay, &kind, &log_g) != LA_OK) return LA_ERR_INVALID_ARG;
    normalize = normalize ? 1 : 0;
    const long long BH = static_cast<long long>(B) * H;
    if (!fits_int(BH * 8)) return LA_ERR_INVALID_ARG;
    if (!state_out || !aligned16(state_out)) return LA_ERR_INVALID_ARG;
    if (normalize && (!z_out || !aligned16(z_out))) return LA_ERR_INVALID_ARG;
    if (log_g_total && !aligned4(log_g_total)) return LA_ERR_INVALID_ARG;
    if (BH > 0 && T > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return LA_ERR_INVALID_ARG;
    if (dtype == LA_F32 && (Dk > 128 || Dv > 128)) return LA_ERR_UNSUPPORTED;
    if (dtype == LA_BF16 && !la::fwd_tc_supports(Dk, Dv)) return LA_ERR_UNSUPPORTED;
    if (BH == 0) return LA_OK;
    if (dtype == LA_BF16 && T > 0) {
        const size_t need = la::fwd_state_workspace_bytes(B, H, T, Dk, Dv, normalize != 0);
        if (!workspace || workspace_bytes < need) return LA_ERR_INVALID_ARG;
    }
    if (launch_fault_injected()) return LA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {  // an empty span: zero state, no decay
        cudaError_t e = cudaMemsetAsync(state_out, 0, sizeof(float) * static_cast<size_t>(BH) * Dk * Dv, s);
        if (e == cudaSuccess && normalize) e = cudaMemsetAsync(z_out, 0, sizeof(float) * static_cast<size_t>(BH) * Dk, s);
        if (e == cudaSuccess && log_g_total) e = cudaMemsetAsync(log_g_total, 0, sizeof(float) * BH, s);
        return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
    }
    la::FwdArgs a{};
    a.q = k;  // no read-out is kept: the keys stand in for the queries
    a.k = k;
    a.v = v;
    a.decay_kind = kind;
    a.log_g = log_g;
    a.normalize = normalize;
    a.B = B;
    a.H = H;
    a.T = T;
    a.Dk = Dk;
    a.Dv = Dv;
    a.stream = s;
    a.err_word = err_word_for_current_device();
    a.q_scale = 1.f;
    cudaError_t e;
    if (dtype == LA_F32) {
        a.out = nullptr;  // the recurrent kernel keeps the state alone
        a.final_state = state_out;
        a.final_z = normalize ? z_out : nullptr;
        e = la::launch_fwd_f32(a);
        if (e == cudaSuccess && log_g_total)
            e = la::launch_log_total(log_g, kind, static_cast<int>(BH), H, T, log_g_total, s);
    } else {
        a.workspace = workspace;
        a.workspace_bytes = workspace_bytes;
        int pieces = 0;
        e = la::launch_fwd_state(a, &pieces);
        if (e == cudaErrorNotSupported) return LA_ERR_UNSUPPORTED;
        if (e == cudaSuccess) {
            // fold the pieces, in order, into the span's state
            const long long DkDv = static_cast<long long>(Dk) * Dv;
            const float* base = static_cast<const float*>(workspace);
            la::CombineArgs c{};
            c.S = base;
            c.S_span = DkDv;
            c.S_bh = pieces * DkDv;
            c.z = base + BH * pieces * DkDv;
            c.z_span = Dk;
            c.z_bh = static_cast<long long>(pieces) * Dk;
            c.L = c.z + BH * pieces * Dk;
            c.L_span = 1;
            c.L_bh = pieces;
            c.n = pieces;
            c.log2_units = 1;
            c.out_S = state_out;
            c.out_z = normalize ? z_out : nullptr;
            c.out_L = log_g_total;
            c.BH = static_cast<int>(BH);
            c.Dk = Dk;
            c.Dv = Dv;
            c.stream = s;
            e = la::launch_fold(c);
        }
    }
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_state_combine(const float* seg_state, const float* seg_z, const float* seg_log_g, long long state_stride,
                           long long z_stride, long long log_stride, int n, const float* init_state,
                           const float* init_z, float* state_out, float* z_out, float* log_g_out, int B, int H,
                           int Dk, int Dv, la_stream_t stream) {
    if (B < 0 || H < 0 || Dk < 1 || Dv < 1 || n < 0) return LA_ERR_INVALID_ARG;
    if (state_stride < 0 || z_stride < 0 || log_stride < 0) return LA_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(B) * H;
    if (!fits_int(BH * 8)) return LA_ERR_INVALID_ARG;
    if (!state_out || !aligned4(state_out)) return LA_ERR_INVALID_ARG;
    for (const void* p : {static_cast<const void*>(seg_state), static_cast<const void*>(seg_z),
                          static_cast<const void*>(seg_log_g), static_cast<const void*>(init_state),
                          static_cast<const void*>(init_z), static_cast<const void*>(z_out),
                          static_cast<const void*>(log_g_out)})
        if (p && !aligned4(p)) return LA_ERR_INVALID_ARG;
    if (n > 0 && (!seg_state || !seg_log_g)) return LA_ERR_INVALID_ARG;
    if (n > 0 && z_out && !seg_z) return LA_ERR_INVALID_ARG;
    if (BH == 0) return LA_OK;
    if (launch_fault_injected()) return LA_ERR_CUDA;
    la::CombineArgs c{};
    c.S = seg_state;
    c.S_span = state_stride;
    c.S_bh = static_cast<long long>(Dk) * Dv;
    c.z = seg_z;
    c.z_span = z_stride;
    c.z_bh = Dk;
    c.L = seg_log_g;
    c.L_span = log_stride;
    c.L_bh = 1;
    c.n = n;
    c.log2_units = 0;
    c.init_S = init_state;
    c.init_z = z_out ? init_z : nullptr;
    c.out_S = state_out;
    c.out_z = z_out;
    c.out_L = log_g_out;
    c.BH = static_cast<int>(BH);
    c.Dk = Dk;
    c.Dv = Dv;
    c.stream = reinterpret_cast<cudaStream_t>(stream);
    return la::launch_fold(c) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
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
    return bwd_layout(B, H, T, Dk, Dv, dtype, decay_kind, true).total;
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
    const BwdLayout L = work ? bwd_layout(B, H, T, Dk, Dv, dtype, kind, true) : BwdLayout{};
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
    if (L.shared_pieces > 0) {
        // its state pieces are the dk scan's ([B H][pieces][Dv][Dk], then the
        // key sums, then the log decays), transposed, with the same log decays
        const int np = L.shared_pieces;
        const size_t n_s = static_cast<size_t>(BH) * np * Dk * Dv;
        const float* from = static_cast<const float*>(scan_ws);
        float* to = reinterpret_cast<float*>(ws + L.scan2);
        if (!cuda_ok(la::launch_transpose(from, to, bh * np, Dv, Dk, s)) ||
            !cuda_ok(cudaMemcpyAsync(to + n_s + static_cast<size_t>(BH) * np * Dk,
                                     from + n_s + static_cast<size_t>(BH) * np * Dv,
                                     sizeof(float) * static_cast<size_t>(BH) * np, cudaMemcpyDeviceToDevice, s)))
            return LA_ERR_CUDA;
        r = scan(k, q, dy, rdecay, 0, d_final_state, nullptr, dv, d_init_state, nullptr, B, H, T, Dk, Dv, dtype,
                 ws + L.scan2, L.scan2_bytes, stream, 1, 0, nullptr, 1);
    } else {
        r = scan(k, q, dy, rdecay, 0, d_final_state, nullptr, dv, d_init_state, nullptr, B, H, T, Dk, Dv, dtype,
                 scan_ws, L.scan_bytes, stream, 1, 0);
    }
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
        a.st = st;  // S_T^T [Dv][Dk]
        a.st_bh = static_cast<long long>(Dk) * Dv;
        a.st_i = 1;
        a.st_j = Dk;
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

size_t la_chunk_backward_norm_workspace_size(int B, int H, int T, int Dk, int Dv, la_dtype dtype, int decay_kind) {
    if ((dtype != LA_F32 && dtype != LA_BF16) || B < 1 || H < 1 || T < 1 || Dk < 1 || Dv < 1) return 0;
    if (decay_kind < LA_DECAY_NONE || decay_kind > LA_DECAY_PER_STEP) return 0;
    if (!fits_int(static_cast<long long>(B) * H * 8)) return 0;
    if (panel_width(Dv, dtype)) return panel_layout(B, H, T, Dk, Dv, dtype, decay_kind).total;
    return norm_layout(B, H, T, Dk, Dv, dtype, decay_kind).total;
}

// The normalised forward's gradients by scans: n and the denominator are
// recomputed (the denominator as the scan of a ones value panel), then
// dn = dy / den and dden = -(dy . n) / den^2 feed the scans of the
// unnormalised backward plus two 16-wide panel scans for the key-sum path.
la_status la_chunk_backward_norm_ws(const void* q, const void* k, const void* v, const la_decay* decay,
                                    const float* init_state, const float* init_z, const void* dy,
                                    const float* d_final_state, const float* d_final_z, void* dq, void* dk, void* dv,
                                    float* d_log_g, float* d_init_state, float* d_init_z, int B, int H, int T, int Dk,
                                    int Dv, la_dtype dtype, void* workspace, size_t workspace_bytes,
                                    la_stream_t stream) {
    if (B < 0 || H < 0 || T < 0 || Dk < 1 || Dv < 1) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    int kind;
    const float* log_g;
    if (check_decay(decay, &kind, &log_g) != LA_OK) return LA_ERR_INVALID_ARG;
    if (d_log_g && (kind == LA_DECAY_NONE || !aligned4(d_log_g))) return LA_ERR_INVALID_ARG;
    if (init_state && !init_z) return LA_ERR_INVALID_ARG;  // a carried state needs its key sum
    const long long BH = static_cast<long long>(B) * H;
    if (!fits_int(BH * 8) || BH > 65535) return BH > 65535 ? LA_ERR_UNSUPPORTED : LA_ERR_INVALID_ARG;
    for (const void* p : {static_cast<const void*>(init_state), static_cast<const void*>(init_z),
                          static_cast<const void*>(d_final_state), static_cast<const void*>(d_final_z),
                          static_cast<const void*>(d_init_state), static_cast<const void*>(d_init_z)})
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
    const int W = panel_width(Dv, dtype);
    const NormLayout L = work && !W ? norm_layout(B, H, T, Dk, Dv, dtype, kind) : NormLayout{};
    const PanelLayout LP = work && W ? panel_layout(B, H, T, Dk, Dv, dtype, kind) : PanelLayout{};
    if (work && workspace_bytes < (W ? LP.total : L.total)) return LA_ERR_INVALID_ARG;
    if (BH == 0) return LA_OK;
    if (launch_fault_injected()) return LA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t sbytes = sizeof(float) * static_cast<size_t>(BH) * Dk * Dv;
    const size_t zbytes = sizeof(float) * static_cast<size_t>(BH) * Dk;

    if (T == 0) {  // the state and key-sum gradients pass through
        cudaError_t e = cudaSuccess;
        if (d_init_state)
            e = d_final_state ? cudaMemcpyAsync(d_init_state, d_final_state, sbytes, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(d_init_state, 0, sbytes, s);
        if (e == cudaSuccess && d_init_z)
            e = d_final_z ? cudaMemcpyAsync(d_init_z, d_final_z, zbytes, cudaMemcpyDeviceToDevice, s)
                          : cudaMemsetAsync(d_init_z, 0, zbytes, s);
        if (e == cudaSuccess && d_log_g && kind == LA_DECAY_PER_HEAD)
            e = cudaMemsetAsync(d_log_g, 0, sizeof(float) * H, s);
        return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
    }

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto at = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    const int bh = static_cast<int>(BH);
    const long long ntok = BH * T;
    la_status r;
#define LA_SCAN(...)                      \
    do {                                  \
        r = scan(__VA_ARGS__);            \
        if (r != LA_OK) return r;         \
    } while (0)
    if (W) {
        float* lsh = kind != LA_DECAY_NONE ? at(LP.base.lsh) : nullptr;
        const bool has_init = init_state || init_z, has_final = d_final_state || d_final_z;
        float* ainit = has_init ? at(LP.ainit) : nullptr;
        float* binit = has_init ? at(LP.binit) : nullptr;
        float* cinit = has_final ? at(LP.cinit) : nullptr;
        float* f1 = (d_log_g && has_final) ? at(LP.f1) : nullptr;
        float* f4 = d_init_z ? at(LP.f4) : nullptr;
        void* pk = ws + LP.pk;
        void* nd = ws + LP.nd;
        void* pq = ws + LP.pq;
        void* dn = ws + LP.dn;
        void* scan_ws = LP.scan_bytes ? ws + LP.scan : nullptr;
        const size_t sw = LP.scan_bytes;
        if (lsh && !ok(la::launch_shift_decay(log_g, kind, lsh, B, H, T, s))) return LA_ERR_CUDA;
        if (ainit && (!ok(la::launch_pack_state_panel(init_state, init_z, ainit, bh, Dk, Dv, W, s)) ||
                      !ok(la::launch_transpose(ainit, binit, bh, Dk, W, s))))
            return LA_ERR_CUDA;
        if (cinit && (!ok(la::launch_pack_state_panel(d_final_state, d_final_z, at(LP.dpan), bh, Dk, Dv, W, s)) ||
                      !ok(la::launch_transpose(at(LP.dpan), cinit, bh, Dk, W, s))))
            return LA_ERR_CUDA;
        if (!ok(la::launch_pack_value_panel(v, pk, Dv, W, ntok, dtype, s))) return LA_ERR_CUDA;
        const la_decay shifted{LA_DECAY_PER_STEP, lsh};
        const la_decay* rdecay = lsh ? &shifted : nullptr;
        // [n | den] = q^T [S | z] by one scan of the value panel [v | 1]
        LA_SCAN(q, k, pk, decay, 0, ainit, nullptr, nd, f1, nullptr, B, H, T, Dk, W, dtype, scan_ws, sw, stream, 0,
                0);
        if (!ok(la::launch_norm_grad_panel(dy, nd, pq, dn, Dv, W, ntok, dtype, s))) return LA_ERR_CUDA;
        // dq_t = [S_t | z_t] [dn_t; dden_t]: scores [dn | dden] . [v | 1]
        LA_SCAN(pq, pk, k, decay, 0, binit, nullptr, dq, nullptr, nullptr, B, H, T, W, Dk, dtype, scan_ws, sw,
                stream, 0, 0);
        // dk_t = [dS_t^T; dz_t^T]^T [v_t; 1]: the reverse scan of ([v | 1], [dn | dden], q)
        LA_SCAN(pk, pq, q, rdecay, 0, cinit, nullptr, dk, f4, nullptr, B, H, T, W, Dk, dtype, scan_ws, sw, stream,
                1, 0);
        LA_SCAN(k, q, dn, rdecay, 0, d_final_state, nullptr, dv, d_init_state, nullptr, B, H, T, Dk, Dv, dtype,
                scan_ws, sw, stream, 1, 0);
        if (d_init_state && kind != LA_DECAY_NONE &&
            !ok(la::launch_scale_by_first_decay(d_init_state, log_g, kind, B, H, T, Dk * Dv, s)))
            return LA_ERR_CUDA;
        if (f4 && !ok(la::launch_panel_row_scaled(f4, d_init_z, log_g, kind, B, H, T, Dk, W, Dv, s)))
            return LA_ERR_CUDA;
        if (d_log_g) {
            la::DlogArgs a{};
            a.q = q;
            a.k = k;
            a.dq = dq;
            a.dk = dk;
            a.d_final_state = d_final_state;
            a.st = f1;  // [S_T | z_T | 0] as [Dk][W]
            a.st_bh = static_cast<long long>(Dk) * W;
            a.st_i = W;
            a.st_j = 1;
            a.d_final_z = d_final_z;
            a.zt = f1 ? f1 + Dv : nullptr;
            a.zt_bh = static_cast<long long>(Dk) * W;
            a.zt_i = W;
            a.d_log_g = d_log_g;
            a.kind = kind;
            a.B = B;
            a.H = H;
            a.T = T;
            a.Dk = Dk;
            a.Dv = Dv;
            a.dtype = dtype;
            a.scratch = reinterpret_cast<double*>(ws + LP.base.dlog);
            a.stream = s;
            if (!ok(la::launch_dlog(a))) return LA_ERR_CUDA;
        }
        return LA_OK;
    }
    // Dv + 1 above the widest panel: the numerator's and the denominator's
    // terms of dq and dk come from separate scans, the second adding into the
    // first's output (fp32 add, one rounding)
    float* s0t = init_state ? at(L.base.s0t) : nullptr;
    float* dsft = d_final_state ? at(L.base.dsft) : nullptr;
    const bool need_st = d_log_g && d_final_state;
    float* st = need_st ? at(L.base.st) : nullptr;
    float* lsh = kind != LA_DECAY_NONE ? at(L.base.lsh) : nullptr;
    float* z0p = init_z ? at(L.z0p) : nullptr;
    float* z0t = init_z ? at(L.z0t) : nullptr;
    float* dzft = d_final_z ? at(L.dzft) : nullptr;
    float* ztp = (d_log_g && d_final_z) ? at(L.ztp) : nullptr;
    float* dz1p = d_init_z ? at(L.dz1p) : nullptr;
    void* ones = ws + L.ones;
    void* denp = ws + L.denp;
    void* y = ws + L.y;
    void* dn = ws + L.dn;
    void* ddp = ws + L.ddp;
    void* scan_ws = L.scan_bytes ? ws + L.scan : nullptr;
    const size_t sw = L.scan_bytes;

    if (s0t && !ok(la::launch_transpose(init_state, s0t, bh, Dk, Dv, s))) return LA_ERR_CUDA;
    if (dsft && !ok(la::launch_transpose(d_final_state, dsft, bh, Dk, Dv, s))) return LA_ERR_CUDA;
    if (lsh && !ok(la::launch_shift_decay(log_g, kind, lsh, B, H, T, s))) return LA_ERR_CUDA;
    if (z0p && !ok(la::launch_vec_panel(init_z, z0p, bh, Dk, true, s))) return LA_ERR_CUDA;
    if (z0t && !ok(la::launch_vec_panel(init_z, z0t, bh, Dk, false, s))) return LA_ERR_CUDA;
    if (dzft && !ok(la::launch_vec_panel(d_final_z, dzft, bh, Dk, false, s))) return LA_ERR_CUDA;
    if (!ok(la::launch_ones_panel(ones, ntok, dtype, s))) return LA_ERR_CUDA;
    const la_decay shifted{LA_DECAY_PER_STEP, lsh};
    const la_decay* rdecay = lsh ? &shifted : nullptr;
    // the normalised output y_t = n_t / den_t (one rounding of the ratio, whose
    // numerator and denominator share the kernel's scores) and the
    // denominator q_t . z_t (ones value panel, column 0)
    LA_SCAN(q, k, v, decay, 1, init_state, init_z, y, nullptr, nullptr, B, H, T, Dk, Dv, dtype, scan_ws, sw, stream,
            0, 0);
    LA_SCAN(q, k, ones, decay, 0, z0p, nullptr, denp, ztp, nullptr, B, H, T, Dk, 16, dtype, scan_ws, sw, stream, 0,
            0);
    if (!ok(la::launch_norm_grad(dy, y, denp, dn, ddp, Dv, ntok, dtype, s))) return LA_ERR_CUDA;
    // dq = S_t dn_t + dden_t z_t (the second scan adds into dq)
    LA_SCAN(dn, v, k, decay, 0, s0t, nullptr, dq, st, nullptr, B, H, T, Dv, Dk, dtype, scan_ws, sw, stream, 0, 0);
    LA_SCAN(ddp, ones, k, decay, 0, z0t, nullptr, dq, nullptr, nullptr, B, H, T, 16, Dk, dtype, scan_ws, sw, stream,
            0, 1);
    // dk = dS_t v_t + dz_t (the second scan adds into dk), dv = dS_t^T k_t
    LA_SCAN(v, dn, q, rdecay, 0, dsft, nullptr, dk, nullptr, nullptr, B, H, T, Dv, Dk, dtype, scan_ws, sw, stream,
            1, 0);
    LA_SCAN(ones, ddp, q, rdecay, 0, dzft, nullptr, dk, dz1p, nullptr, B, H, T, 16, Dk, dtype, scan_ws, sw, stream,
            1, 1);
    LA_SCAN(k, q, dn, rdecay, 0, d_final_state, nullptr, dv, d_init_state, nullptr, B, H, T, Dk, Dv, dtype, scan_ws,
            sw, stream, 1, 0);
#undef LA_SCAN
    if (d_init_state && kind != LA_DECAY_NONE &&
        !ok(la::launch_scale_by_first_decay(d_init_state, log_g, kind, B, H, T, Dk * Dv, s)))
        return LA_ERR_CUDA;
    if (dz1p && !ok(la::launch_panel_row_scaled(dz1p, d_init_z, log_g, kind, B, H, T, Dk, 16, 0, s)))
        return LA_ERR_CUDA;
    if (d_log_g) {
        la::DlogArgs a{};
        a.q = q;
        a.k = k;
        a.dq = dq;
        a.dk = dk;
        a.d_final_state = d_final_state;
        a.st = st;  // S_T^T [Dv][Dk]
        a.st_bh = static_cast<long long>(Dk) * Dv;
        a.st_i = 1;
        a.st_j = Dk;
        a.d_final_z = d_final_z;
        a.zt = ztp;  // column 0 of [Dk][16]
        a.zt_bh = 16LL * Dk;
        a.zt_i = 16;
        a.d_log_g = d_log_g;
        a.kind = kind;
        a.B = B;
        a.H = H;
        a.T = T;
        a.Dk = Dk;
        a.Dv = Dv;
        a.dtype = dtype;
        a.scratch = reinterpret_cast<double*>(ws + L.base.dlog);
        a.stream = s;
        if (!ok(la::launch_dlog(a))) return LA_ERR_CUDA;
    }
    return LA_OK;
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

la_status la_ema_scan(const void* x, const void* f, const float* init_state, void* out, float* final_state, int B,
                      int T, int C, la_dtype dtype, int reverse, la_stream_t stream) {
    if (B < 0 || T < 0 || C < 1) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if ((init_state && !aligned4(init_state)) || (final_state && !aligned4(final_state))) return LA_ERR_INVALID_ARG;
    if (B > 0 && T > 0) {
        if (!x || !f || !out) return LA_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(f) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    }
    // rows of x and f are TMA tiles: their byte stride must be a multiple of 16
    if (C % (dtype == LA_BF16 ? 8 : 4) != 0) return LA_ERR_UNSUPPORTED;
    if (B > 65535 || !fits_int(static_cast<long long>(T) * C) || !fits_int(static_cast<long long>(B) * C))
        return LA_ERR_UNSUPPORTED;
    if (B == 0) return LA_OK;
    if (launch_fault_injected()) return LA_ERR_CUDA;
    la::EmaArgs a{};
    a.x = x;
    a.f = f;
    a.init_state = init_state;
    a.out = out;
    a.final_state = final_state;
    a.B = B;
    a.T = T;
    a.C = C;
    a.dtype = dtype;
    a.reverse = reverse ? 1 : 0;
    a.err_word = err_word_for_current_device();
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    return la::launch_ema(a) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
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
