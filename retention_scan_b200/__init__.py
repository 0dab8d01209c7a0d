"""retention_scan_b200: causal linear attention with an optional decay on B200.

Python binding of the C ABI in include/la.h (libla.so, built in-tree by
``python -m retention_scan_b200.build``).  This module only marshals
arguments: it checks shapes and dtypes, allocates outputs with torch when the
caller does not pass them, and hands raw device pointers and the current CUDA
stream to the library.  Every step of the computation runs in the library's
CUDA kernels; there is no fallback.  Importing works without a GPU; calling
a compute function without the built library or without a CUDA device raises.
"""
import ctypes
import os

import torch

__all__ = ["chunk_forward", "bidirectional", "chunk_backward", "chunk_backward_normalized", "wkv4_forward", "ema_scan",
           "chunk_state", "state_combine", "state_workspace_size", "workspace_size",
           "backward_workspace_size",
           "decode_step", "device_error", "LAError", "lib", "library_path",
           "DECAY_NONE", "DECAY_PER_HEAD", "DECAY_PER_STEP", "FEATURE_NONE", "FEATURE_ELU1", "EXPORTED_SYMBOLS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libla.so")

DECAY_NONE, DECAY_PER_HEAD, DECAY_PER_STEP = 0, 1, 2
FEATURE_NONE, FEATURE_ELU1 = 0, 1
LA_F32, LA_BF16 = 0, 1
EXPORTED_SYMBOLS = ("la_chunk_forward", "la_chunk_forward_ws", "la_chunk_forward_workspace_size",
                    "la_chunk_reverse_ws", "la_chunk_bidirectional_ws",
                    "la_chunk_backward_ws", "la_chunk_backward_workspace_size", "la_wkv4_forward",
                    "la_wkv4_forward_ws", "la_wkv4_workspace_size", "la_chunk_forward_pro_ws",
                    "la_decode_step_pro", "la_chunk_backward_norm_ws", "la_chunk_backward_norm_workspace_size",
                    "la_ema_scan", "la_chunk_state_ws", "la_chunk_state_workspace_size", "la_state_combine",
                    "la_decode_step", "la_status_string", "la_device_error", "la_version")


class LAError(RuntimeError):
    """A nonzero la_status from the library."""

    def __init__(self, status, message):
        super().__init__(message)
        self.status = status


class _Decay(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("log_g", ctypes.c_void_p)]


class _Prologue(ctypes.Structure):
    _fields_ = [("feature_map", ctypes.c_int), ("q_scale", ctypes.c_float)]


_lib = None


def lib():
    """The loaded libla.so (ctypes).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise ImportError(f"retention_scan_b200: {library_path} is missing; build it with "
                              "`python -m retention_scan_b200.build`")
        L = ctypes.CDLL(library_path)
        vp, i = ctypes.c_void_p, ctypes.c_int
        L.la_chunk_forward.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), i, vp, vp, vp, vp, vp,
                                       i, i, i, i, i, i, vp]
        L.la_chunk_forward.restype = i
        L.la_chunk_forward_ws.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), i, vp, vp, vp, vp, vp,
                                          i, i, i, i, i, i, vp, ctypes.c_size_t, vp]
        L.la_chunk_forward_ws.restype = i
        L.la_chunk_forward_pro_ws.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), i, ctypes.POINTER(_Prologue),
                                              vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, ctypes.c_size_t, vp]
        L.la_chunk_forward_pro_ws.restype = i
        L.la_decode_step_pro.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), i, ctypes.POINTER(_Prologue), vp, vp,
                                         vp, i, i, i, i, i, vp]
        L.la_decode_step_pro.restype = i
        L.la_chunk_reverse_ws.argtypes = L.la_chunk_forward_ws.argtypes
        L.la_chunk_reverse_ws.restype = i
        L.la_chunk_bidirectional_ws.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), i, vp,
                                                i, i, i, i, i, i, vp, ctypes.c_size_t, vp]
        L.la_chunk_bidirectional_ws.restype = i
        L.la_chunk_backward_ws.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), vp, vp, vp, vp, vp, vp, vp, vp,
                                           i, i, i, i, i, i, vp, ctypes.c_size_t, vp]
        L.la_chunk_backward_ws.restype = i
        L.la_chunk_backward_norm_ws.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), vp, vp, vp, vp, vp, vp, vp, vp,
                                                vp, vp, vp, i, i, i, i, i, i, vp, ctypes.c_size_t, vp]
        L.la_chunk_backward_norm_ws.restype = i
        L.la_chunk_backward_norm_workspace_size.argtypes = [i, i, i, i, i, i, i]
        L.la_chunk_backward_norm_workspace_size.restype = ctypes.c_size_t
        L.la_chunk_backward_workspace_size.argtypes = [i, i, i, i, i, i, i]
        L.la_chunk_backward_workspace_size.restype = ctypes.c_size_t
        L.la_ema_scan.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, vp]
        L.la_ema_scan.restype = i
        L.la_chunk_state_ws.argtypes = [vp, vp, ctypes.POINTER(_Decay), i, vp, vp, vp, i, i, i, i, i, i, vp,
                                        ctypes.c_size_t, vp]
        L.la_chunk_state_ws.restype = i
        L.la_chunk_state_workspace_size.argtypes = [i, i, i, i, i, i, i]
        L.la_chunk_state_workspace_size.restype = ctypes.c_size_t
        ll = ctypes.c_longlong
        L.la_state_combine.argtypes = [vp, vp, vp, ll, ll, ll, i, vp, vp, vp, vp, vp, i, i, i, i, vp]
        L.la_state_combine.restype = i
        L.la_wkv4_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp]
        L.la_wkv4_forward.restype = i
        L.la_wkv4_forward_ws.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp, ctypes.c_size_t, vp]
        L.la_wkv4_forward_ws.restype = i
        L.la_wkv4_workspace_size.argtypes = [i, i, i, i]
        L.la_wkv4_workspace_size.restype = ctypes.c_size_t
        L.la_chunk_forward_workspace_size.argtypes = [i, i, i, i, i, i, i]
        L.la_chunk_forward_workspace_size.restype = ctypes.c_size_t
        L.la_decode_step.argtypes = [vp, vp, vp, ctypes.POINTER(_Decay), i, vp, vp, vp,
                                     i, i, i, i, i, vp]
        L.la_decode_step.restype = i
        L.la_status_string.argtypes = [i]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), vp]
        L.la_device_error.restype = i
        L.la_version.argtypes = []
        L.la_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status):
    if status != 0:
        raise LAError(status, lib().la_status_string(status).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt):
    if dt == torch.float32:
        return LA_F32
    if dt == torch.bfloat16:
        return LA_BF16
    raise TypeError(f"q, k, v must be float32 or bfloat16, got {dt}")


def _need(t, name, shape, dtype, device):
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _decay(kind, log_g):
    if kind == DECAY_NONE:
        return None
    if log_g is None:
        raise ValueError("log_g is required for a per-head or per-step decay")
    return _Decay(kind, log_g.data_ptr())


def _stream(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(B, H, T, Dk, Dv, dtype=torch.bfloat16, normalize=False):
    """Scratch bytes chunk_forward can use for these sizes (la_chunk_forward_workspace_size)."""
    return int(lib().la_chunk_forward_workspace_size(B, H, T, Dk, Dv, _dtype_code(dtype), int(bool(normalize))))


def _workspace(workspace, B, H, T, Dk, Dv, dtype, normalize, stream, dev):
    if workspace is True:
        nbytes = workspace_size(B, H, T, Dk, Dv, dtype, normalize)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
        if workspace is not None and stream is not None:
            workspace.record_stream(stream)
    elif workspace is False:
        workspace = None
    if workspace is not None:
        if workspace.device != dev or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
            raise ValueError("workspace: expected a contiguous uint8 tensor on the inputs' device")
    return workspace


def chunk_forward(q, k, v, decay_kind=DECAY_NONE, log_g=None, normalize=False,
                  init_state=None, init_z=None, out=None, final_state=None, final_z=None,
                  return_final=True, stream=None, workspace=True, reverse=False,
                  feature_map=FEATURE_NONE, q_scale=1.0):
    """Whole-sequence forward (la_chunk_forward_ws), or with reverse=True the
    anti-causal scan from the last token back (la_chunk_reverse_ws; the
    carried state then enters after token T and final_* hold the state at
    token 1).

    q, k: [B,H,T,Dk]; v: [B,H,T,Dv]; float32 or bfloat16 CUDA tensors.
    decay_kind: DECAY_NONE, DECAY_PER_HEAD (log_g [H]) or DECAY_PER_STEP
    (log_g [B,H,T]); log_g is fp32 natural log of the decay factor, <= 0.
    init_state [B,H,Dk,Dv] / init_z [B,H,Dk]: fp32 carried state and key sum.
    Returns (out, final_state, final_z); final_* are None unless requested
    (return_final, or passed in), final_z only when normalize.
    workspace: True allocates the scratch that lets short-on-heads inputs run
    as T-segments (a torch allocation on the call's stream), None/False runs
    without, or a CUDA uint8 tensor to use.
    feature_map / q_scale: the input prologue (la_chunk_forward_pro_ws): the
    kernels read phi(q) * q_scale and phi(k), phi = FEATURE_ELU1 (elu + 1)
    or FEATURE_NONE.  Forward scans only.
    """
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    code = _dtype_code(q.dtype)
    _need(k, "k", (B, H, T, Dk), q.dtype, dev)
    _need(v, "v", (B, H, T, Dv), q.dtype, dev)
    _need(q, "q", (B, H, T, Dk), q.dtype, dev)
    if decay_kind == DECAY_PER_HEAD:
        _need(log_g, "log_g", (H,), torch.float32, dev)
    elif decay_kind == DECAY_PER_STEP:
        _need(log_g, "log_g", (B, H, T), torch.float32, dev)
    _need(init_state, "init_state", (B, H, Dk, Dv), torch.float32, dev)
    _need(init_z, "init_z", (B, H, Dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, T, Dv), dtype=q.dtype, device=dev)
    _need(out, "out", (B, H, T, Dv), q.dtype, dev)
    if final_state is None and return_final:
        final_state = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev)
    if final_z is None and return_final and normalize:
        final_z = torch.empty((B, H, Dk), dtype=torch.float32, device=dev)
    _need(final_state, "final_state", (B, H, Dk, Dv), torch.float32, dev)
    _need(final_z, "final_z", (B, H, Dk), torch.float32, dev)
    d = _decay(decay_kind, log_g)
    with torch.cuda.device(dev):
        workspace = _workspace(workspace, B, H, T, Dk, Dv, q.dtype, normalize, stream, dev)
        nbytes = 0 if workspace is None else workspace.numel()
        if feature_map != FEATURE_NONE or q_scale != 1.0:
            if reverse:
                raise ValueError("the input prologue applies to the forward scan")
            pro = _Prologue(int(feature_map), float(q_scale))
            _check(lib().la_chunk_forward_pro_ws(
                _ptr(q), _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, int(bool(normalize)),
                ctypes.byref(pro), _ptr(init_state), _ptr(init_z), _ptr(out), _ptr(final_state), _ptr(final_z),
                B, H, T, Dk, Dv, code, _ptr(workspace), nbytes, _stream(stream, dev)))
            return out, final_state, (final_z if normalize else None)
        entry = lib().la_chunk_reverse_ws if reverse else lib().la_chunk_forward_ws
        _check(entry(
            _ptr(q), _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, int(bool(normalize)),
            _ptr(init_state), _ptr(init_z), _ptr(out), _ptr(final_state), _ptr(final_z),
            B, H, T, Dk, Dv, code, _ptr(workspace), nbytes, _stream(stream, dev)))
    return out, final_state, (final_z if normalize else None)


def bidirectional(q, k, v, decay_kind=DECAY_NONE, log_g=None, normalize=False, out=None, stream=None,
                  workspace=True):
    """Bidirectional encoder output (la_chunk_bidirectional_ws): the forward
    scan plus the reverse scan, both from zero states.  Arguments as
    chunk_forward.  Returns out [B,H,T,Dv]."""
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    code = _dtype_code(q.dtype)
    _need(k, "k", (B, H, T, Dk), q.dtype, dev)
    _need(v, "v", (B, H, T, Dv), q.dtype, dev)
    _need(q, "q", (B, H, T, Dk), q.dtype, dev)
    if decay_kind == DECAY_PER_HEAD:
        _need(log_g, "log_g", (H,), torch.float32, dev)
    elif decay_kind == DECAY_PER_STEP:
        _need(log_g, "log_g", (B, H, T), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, T, Dv), dtype=q.dtype, device=dev)
    _need(out, "out", (B, H, T, Dv), q.dtype, dev)
    d = _decay(decay_kind, log_g)
    with torch.cuda.device(dev):
        workspace = _workspace(workspace, B, H, T, Dk, Dv, q.dtype, normalize, stream, dev)
        _check(lib().la_chunk_bidirectional_ws(
            _ptr(q), _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, int(bool(normalize)),
            _ptr(out), B, H, T, Dk, Dv, code, _ptr(workspace), 0 if workspace is None else workspace.numel(),
            _stream(stream, dev)))
    return out


def backward_workspace_size(B, H, T, Dk, Dv, dtype=torch.bfloat16, decay_kind=DECAY_NONE):
    """Scratch bytes chunk_backward needs (la_chunk_backward_workspace_size)."""
    return int(lib().la_chunk_backward_workspace_size(B, H, T, Dk, Dv, _dtype_code(dtype), int(decay_kind)))


def chunk_backward(q, k, v, dy, decay_kind=DECAY_NONE, log_g=None, init_state=None, d_final_state=None,
                   need_log_g=True, need_init_state=True, stream=None, workspace=None, out=None):
    """Gradients of the unnormalised forward (la_chunk_backward_ws) for the
    loss sum(dy * y) + sum(d_final_state * final_state).

    q, k: [B,H,T,Dk]; v, dy: [B,H,T,Dv] (float32 or bfloat16, all one dtype);
    decay_kind / log_g as chunk_forward; init_state [B,H,Dk,Dv] fp32 or None;
    d_final_state [B,H,Dk,Dv] fp32 or None.  Returns (dq, dk, dv, d_log_g,
    d_init_state): dq, dk, dv in the input dtype; d_log_g fp32 with log_g's
    shape (None without a decay or need_log_g=False); d_init_state fp32 (None
    with need_init_state=False).  workspace: None allocates it with torch on
    the call's stream, or a CUDA uint8 tensor of at least
    backward_workspace_size(...) bytes.  out: None, or a tuple (dq, dk, dv,
    d_log_g, d_init_state) of preallocated outputs (entries may be None to
    skip d_log_g / d_init_state).
    """
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    code = _dtype_code(q.dtype)
    _need(k, "k", (B, H, T, Dk), q.dtype, dev)
    _need(v, "v", (B, H, T, Dv), q.dtype, dev)
    _need(dy, "dy", (B, H, T, Dv), q.dtype, dev)
    _need(q, "q", (B, H, T, Dk), q.dtype, dev)
    if decay_kind == DECAY_PER_HEAD:
        _need(log_g, "log_g", (H,), torch.float32, dev)
    elif decay_kind == DECAY_PER_STEP:
        _need(log_g, "log_g", (B, H, T), torch.float32, dev)
    _need(init_state, "init_state", (B, H, Dk, Dv), torch.float32, dev)
    _need(d_final_state, "d_final_state", (B, H, Dk, Dv), torch.float32, dev)
    if out is None:
        dq, dk = torch.empty_like(q), torch.empty_like(k)
        dv = torch.empty_like(v)
        d_log_g = torch.empty_like(log_g) if (decay_kind != DECAY_NONE and need_log_g) else None
        d_init = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev) if need_init_state else None
    else:
        dq, dk, dv, d_log_g, d_init = out
        _need(dq, "dq", (B, H, T, Dk), q.dtype, dev)
        _need(dk, "dk", (B, H, T, Dk), q.dtype, dev)
        _need(dv, "dv", (B, H, T, Dv), q.dtype, dev)
        if d_log_g is not None:
            _need(d_log_g, "d_log_g", tuple(log_g.shape), torch.float32, dev)
        _need(d_init, "d_init_state", (B, H, Dk, Dv), torch.float32, dev)
    d = _decay(decay_kind, log_g)
    with torch.cuda.device(dev):
        nbytes = backward_workspace_size(B, H, T, Dk, Dv, q.dtype, decay_kind)
        if workspace is None:
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
            if stream is not None:
                workspace.record_stream(stream)
        elif workspace.device != dev or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
            raise ValueError("workspace: expected a contiguous uint8 tensor on the inputs' device")
        _check(lib().la_chunk_backward_ws(
            _ptr(q), _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, _ptr(init_state), _ptr(dy),
            _ptr(d_final_state), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(d_log_g), _ptr(d_init),
            B, H, T, Dk, Dv, code, _ptr(workspace), workspace.numel(), _stream(stream, dev)))
    return dq, dk, dv, d_log_g, d_init


def state_workspace_size(B, H, T, Dk, Dv, dtype=torch.bfloat16, normalize=False):
    """Scratch bytes chunk_state needs for these sizes (la_chunk_state_workspace_size)."""
    return int(lib().la_chunk_state_workspace_size(B, H, T, Dk, Dv, _dtype_code(dtype), int(bool(normalize))))


def chunk_state(k, v, decay_kind=DECAY_NONE, log_g=None, normalize=False, state_out=None, z_out=None,
                log_g_total=None, stream=None, workspace=True):
    """A span's own state from zero and its total log decay (la_chunk_state_ws):
    S_T and z_T of the recurrence started from zero, and sum_t log g_t per
    (b, h).  k [B,H,T,Dk], v [B,H,T,Dv] float32 or bfloat16; decay as
    chunk_forward.  Returns (state [B,H,Dk,Dv], z [B,H,Dk] or None,
    log_g_total [B,H]), fp32.  workspace: True allocates the bf16 scratch, or
    a CUDA uint8 tensor of at least state_workspace_size bytes."""
    B, H, T, Dk = k.shape
    Dv = v.shape[-1]
    dev = k.device
    code = _dtype_code(k.dtype)
    _need(v, "v", (B, H, T, Dv), k.dtype, dev)
    if decay_kind == DECAY_PER_HEAD:
        _need(log_g, "log_g", (H,), torch.float32, dev)
    elif decay_kind == DECAY_PER_STEP:
        _need(log_g, "log_g", (B, H, T), torch.float32, dev)
    if state_out is None:
        state_out = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev)
    if z_out is None and normalize:
        z_out = torch.empty((B, H, Dk), dtype=torch.float32, device=dev)
    if log_g_total is None:
        log_g_total = torch.empty((B, H), dtype=torch.float32, device=dev)
    _need(state_out, "state_out", (B, H, Dk, Dv), torch.float32, dev)
    _need(z_out, "z_out", (B, H, Dk), torch.float32, dev)
    _need(log_g_total, "log_g_total", (B, H), torch.float32, dev)
    d = _decay(decay_kind, log_g)
    with torch.cuda.device(dev):
        if workspace is True:
            nbytes = state_workspace_size(B, H, T, Dk, Dv, k.dtype, normalize)
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
            if workspace is not None and stream is not None:
                workspace.record_stream(stream)
        elif workspace is False:
            workspace = None
        _check(lib().la_chunk_state_ws(
            _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, int(bool(normalize)), _ptr(state_out),
            _ptr(z_out if normalize else None), _ptr(log_g_total), B, H, T, Dk, Dv, code, _ptr(workspace),
            0 if workspace is None else workspace.numel(), _stream(stream, dev)))
    return state_out, (z_out if normalize else None), log_g_total


def _span_rows(t, name, inner):
    """t: [n, *inner] fp32 whose spans (dim 0) are each contiguous; its
    stride along dim 0 in floats."""
    if tuple(t.shape[1:]) != tuple(inner):
        raise ValueError(f"{name}: expected shape [n, {', '.join(map(str, inner))}], got {tuple(t.shape)}")
    if t.dtype != torch.float32:
        raise TypeError(f"{name}: expected float32, got {t.dtype}")
    if t.shape[0] > 0 and not t[0].is_contiguous():
        raise ValueError(f"{name}: each span must be contiguous")
    return t.stride(0)


def state_combine(seg_state, seg_log_g, seg_z=None, init_state=None, init_z=None, state_out=None, z_out=None,
                  log_g_out=None, stream=None):
    """The left fold of n consecutive spans' states (la_state_combine):
    S <- init_state (or 0); for each span j: S <- exp(L_j) S + S_j (z
    likewise); returns (state, z or None, total log decay).  seg_state
    [n,B,H,Dk,Dv], seg_log_g [n,B,H], seg_z [n,B,H,Dk] (needed for z) -
    fp32 CUDA tensors whose spans may be strided views of one buffer."""
    n, B, H, Dk, Dv = seg_state.shape
    dev = seg_state.device
    ss = _span_rows(seg_state, "seg_state", (B, H, Dk, Dv))
    ls = _span_rows(seg_log_g, "seg_log_g", (B, H))
    zs = _span_rows(seg_z, "seg_z", (B, H, Dk)) if seg_z is not None else 0
    if state_out is None:
        state_out = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev)
    if z_out is None and seg_z is not None:
        z_out = torch.empty((B, H, Dk), dtype=torch.float32, device=dev)
    if log_g_out is None:
        log_g_out = torch.empty((B, H), dtype=torch.float32, device=dev)
    for t, name, shape in ((init_state, "init_state", (B, H, Dk, Dv)), (init_z, "init_z", (B, H, Dk)),
                           (state_out, "state_out", (B, H, Dk, Dv)), (z_out, "z_out", (B, H, Dk)),
                           (log_g_out, "log_g_out", (B, H))):
        _need(t, name, shape, torch.float32, dev)
    with torch.cuda.device(dev):
        _check(lib().la_state_combine(
            _ptr(seg_state) if n else None, _ptr(seg_z) if n and seg_z is not None else None,
            _ptr(seg_log_g) if n else None, ss, zs, ls, n, _ptr(init_state), _ptr(init_z), _ptr(state_out),
            _ptr(z_out), _ptr(log_g_out), B, H, Dk, Dv, _stream(stream, dev)))
    return state_out, z_out, log_g_out


def ema_scan(x, f, init_state=None, reverse=False, out=None, final_state=None, return_final=True, stream=None):
    """Cumulative EMA along T (la_ema_scan): s <- f_t s + x_t per channel,
    out_t = s, forward or reverse.  x, f: [B,T,C] float32 or bfloat16 CUDA
    tensors (C a multiple of 8 for bf16, 4 for fp32); init_state [B,C] fp32
    or None.  Returns (out [B,T,C], final_state [B,C] or None)."""
    B, T, C = x.shape
    dev = x.device
    code = _dtype_code(x.dtype)
    _need(f, "f", (B, T, C), x.dtype, dev)
    _need(x, "x", (B, T, C), x.dtype, dev)
    _need(init_state, "init_state", (B, C), torch.float32, dev)
    if out is None:
        out = torch.empty((B, T, C), dtype=x.dtype, device=dev)
    _need(out, "out", (B, T, C), x.dtype, dev)
    if final_state is None and return_final:
        final_state = torch.empty((B, C), dtype=torch.float32, device=dev)
    _need(final_state, "final_state", (B, C), torch.float32, dev)
    with torch.cuda.device(dev):
        _check(lib().la_ema_scan(_ptr(x), _ptr(f), _ptr(init_state), _ptr(out), _ptr(final_state), B, T, C, code,
                                 int(bool(reverse)), _stream(stream, dev)))
    return out, final_state


WKV4_EMPTY_SCALE = -1e38  # pp of an empty RWKV-4 state (aa = bb = 0)


def wkv4_workspace_size(B, T, C, dtype=torch.bfloat16):
    """Scratch bytes wkv4_forward can use (la_wkv4_workspace_size)."""
    return int(lib().la_wkv4_workspace_size(B, T, C, _dtype_code(dtype)))


def wkv4_forward(k, v, w, u, init_state=None, out=None, final_state=None, return_final=True, stream=None,
                 workspace=True):
    """RWKV-4 WKV recurrence (la_wkv4_forward_ws).  k, v: [B,T,C] float32 or
    bfloat16 CUDA tensors (C a multiple of 8 for bf16, 4 for fp32); w (log
    of the per-step decay) and u (bonus): [C] fp32; init_state: [B,3,C] fp32
    (planes aa, bb, pp) or None for the empty state.  Returns (out [B,T,C],
    final_state [B,3,C] or None).  final_state may be init_state itself.
    workspace: True allocates the T-segment scratch with torch on the call's
    stream, None/False runs one segment, or a CUDA uint8 tensor to use."""
    B, T, C = k.shape
    dev = k.device
    code = _dtype_code(k.dtype)
    _need(v, "v", (B, T, C), k.dtype, dev)
    _need(k, "k", (B, T, C), k.dtype, dev)
    _need(w, "w", (C,), torch.float32, dev)
    _need(u, "u", (C,), torch.float32, dev)
    _need(init_state, "init_state", (B, 3, C), torch.float32, dev)
    if out is None:
        out = torch.empty((B, T, C), dtype=k.dtype, device=dev)
    _need(out, "out", (B, T, C), k.dtype, dev)
    if final_state is None and return_final:
        final_state = torch.empty((B, 3, C), dtype=torch.float32, device=dev)
    _need(final_state, "final_state", (B, 3, C), torch.float32, dev)
    with torch.cuda.device(dev):
        if workspace is True:
            nbytes = wkv4_workspace_size(B, T, C, k.dtype)
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
            if workspace is not None and stream is not None:
                workspace.record_stream(stream)
        elif workspace is False:
            workspace = None
        _check(lib().la_wkv4_forward_ws(_ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(init_state), _ptr(out),
                                        _ptr(final_state), B, T, C, code, _ptr(workspace),
                                        0 if workspace is None else workspace.numel(), _stream(stream, dev)))
    return out, final_state


def chunk_backward_normalized(q, k, v, dy, decay_kind=DECAY_NONE, log_g=None, init_state=None, init_z=None,
                              d_final_state=None, d_final_z=None, need_log_g=True, need_init_state=True,
                              stream=None, workspace=None):
    """Gradients of the normalised forward (la_chunk_backward_norm_ws) for the
    loss sum(dy * y) + sum(d_final_state * final_state) + sum(d_final_z *
    final_z).  Arguments as chunk_backward, plus init_z / d_final_z [B,H,Dk]
    fp32 (init_z is required with init_state).  Returns (dq, dk, dv,
    d_log_g, d_init_state, d_init_z)."""
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    code = _dtype_code(q.dtype)
    _need(k, "k", (B, H, T, Dk), q.dtype, dev)
    _need(v, "v", (B, H, T, Dv), q.dtype, dev)
    _need(dy, "dy", (B, H, T, Dv), q.dtype, dev)
    _need(q, "q", (B, H, T, Dk), q.dtype, dev)
    if decay_kind == DECAY_PER_HEAD:
        _need(log_g, "log_g", (H,), torch.float32, dev)
    elif decay_kind == DECAY_PER_STEP:
        _need(log_g, "log_g", (B, H, T), torch.float32, dev)
    _need(init_state, "init_state", (B, H, Dk, Dv), torch.float32, dev)
    _need(init_z, "init_z", (B, H, Dk), torch.float32, dev)
    _need(d_final_state, "d_final_state", (B, H, Dk, Dv), torch.float32, dev)
    _need(d_final_z, "d_final_z", (B, H, Dk), torch.float32, dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    d_log_g = torch.empty_like(log_g) if (decay_kind != DECAY_NONE and need_log_g) else None
    d_init = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev) if need_init_state else None
    d_init_z = torch.empty((B, H, Dk), dtype=torch.float32, device=dev) if need_init_state else None
    d = _decay(decay_kind, log_g)
    with torch.cuda.device(dev):
        nbytes = int(lib().la_chunk_backward_norm_workspace_size(B, H, T, Dk, Dv, code, int(decay_kind)))
        if workspace is None:
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
            if stream is not None:
                workspace.record_stream(stream)
        elif workspace.device != dev or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
            raise ValueError("workspace: expected a contiguous uint8 tensor on the inputs' device")
        _check(lib().la_chunk_backward_norm_ws(
            _ptr(q), _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, _ptr(init_state), _ptr(init_z),
            _ptr(dy), _ptr(d_final_state), _ptr(d_final_z), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(d_log_g),
            _ptr(d_init), _ptr(d_init_z), B, H, T, Dk, Dv, code, _ptr(workspace), workspace.numel(),
            _stream(stream, dev)))
    return dq, dk, dv, d_log_g, d_init, d_init_z


def decode_step(q, k, v, state, z=None, decay_kind=DECAY_NONE, log_g=None, normalize=False,
                out=None, stream=None, feature_map=FEATURE_NONE, q_scale=1.0):
    """One token (la_decode_step); state [B,H,Dk,Dv] and z [B,H,Dk] (fp32) are
    updated in place.  q, k: [B,H,Dk]; v: [B,H,Dv].  Returns out [B,H,Dv].
    feature_map / q_scale: the input prologue (la_decode_step_pro): the kernel
    reads phi(q) * q_scale and phi(k)."""
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    code = _dtype_code(q.dtype)
    _need(k, "k", (B, H, Dk), q.dtype, dev)
    _need(v, "v", (B, H, Dv), q.dtype, dev)
    _need(state, "state", (B, H, Dk, Dv), torch.float32, dev)
    if normalize:
        if z is None:
            raise ValueError("z is required when normalize")
        _need(z, "z", (B, H, Dk), torch.float32, dev)
    if decay_kind == DECAY_PER_HEAD:
        _need(log_g, "log_g", (H,), torch.float32, dev)
    elif decay_kind == DECAY_PER_STEP:
        _need(log_g, "log_g", (B, H), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, Dv), dtype=q.dtype, device=dev)
    _need(out, "out", (B, H, Dv), q.dtype, dev)
    d = _decay(decay_kind, log_g)
    with torch.cuda.device(dev):
        if feature_map != FEATURE_NONE or q_scale != 1.0:
            pro = _Prologue(int(feature_map), float(q_scale))
            _check(lib().la_decode_step_pro(
                _ptr(q), _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, int(bool(normalize)),
                ctypes.byref(pro), _ptr(state), _ptr(z if normalize else None), _ptr(out), B, H, Dk, Dv, code,
                _stream(stream, dev)))
        else:
            _check(lib().la_decode_step(
                _ptr(q), _ptr(k), _ptr(v), ctypes.byref(d) if d is not None else None, int(bool(normalize)),
                _ptr(state), _ptr(z if normalize else None), _ptr(out), B, H, Dk, Dv, code,
                _stream(stream, dev)))
    return out


def device_error(device=None, stream=None):
    """Read and clear the library's device error word (0 = no kernel gave up
    waiting).  Synchronises with the stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    code = ctypes.c_int(0)
    with torch.cuda.device(dev):
        _check(lib().la_device_error(ctypes.byref(code), _stream(stream, dev)))
    return code.value
