"""The oracle: float64 CPU implementations of causal linear attention.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs may import this package.  The CUDA library
(retention_scan_b200) never imports it and shares no code with it.

  forward(...)           recurrent definition, plain C (la_ref.c), token by token
  reverse(...)           the reverse scan, by its definition: forward of the
                         time-reversed arguments, output reversed back
  bidirectional(...)     forward + reverse
  decode_step(...)       one token of the same recurrence, in place
  backward(...)          gradients of a loss through the forward recurrence,
                         by the chain rule token by token (la_ref.c)
  wkv4(...)              the RWKV-4 WKV recurrence of BlinkDL/RWKV-LM issue
                         167 (formula 14) as an online weighted mean (wkv4_ref.c)
  wkv4_direct(...)       the same output from its definition, O(T^2), numpy
  ema(...)               the cumulative EMA of RetNet issue 21 (values,
                         factors, reverse), per channel (ema_ref.c)
  parallel_forward(...)  brute-force O(T^2) parallel form, numpy (parallel.py)
  parallel_reverse(...)  brute-force O(T^2) anti-causal form, numpy (parallel.py)

Every array argument is converted to contiguous float64; bf16 and fp32
inputs up-cast exactly, so the oracle reads the same input bits as the GPU.
"""
import ctypes
import os
import subprocess

import numpy as np

from .parallel import parallel_forward, parallel_reverse  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_ref.c")
_SRCS = (_SRC, os.path.join(_HERE, "wkv4_ref.c"), os.path.join(_HERE, "ema_ref.c"))
_LIB_PATH = os.path.join(_HERE, "liblaref.so")
_libs = {}

DECAY_KINDS = {None: 0, "none": 0, "per_head": 1, "per_step": 2}


def build(force=False):
    """Compile la_ref.c and wkv4_ref.c into liblaref.so beside them (gcc -O2,
    pthreads)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(p) for p in _SRCS):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
                        "-o", tmp, *_SRCS, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path=None):
    """ctypes handle of the compiled oracle (default: liblaref.so, built on
    demand).  Tests pass another path to load a deliberately broken copy."""
    path = build() if path is None else path
    if path not in _libs:
        lib = ctypes.CDLL(path)
        d = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.la_ref_forward.argtypes = [d, d, d, i, d, i, d, d, d, d, d, i, i, i, i, i, i]
        lib.la_ref_forward.restype = i
        lib.la_ref_decode_step.argtypes = [d, d, d, i, d, i, d, d, d, i, i, i, i]
        lib.la_ref_decode_step.restype = i
        lib.la_ref_backward.argtypes = [d, d, d, i, d, i, d, d, d, d, d, d, d, d, d, d, d,
                                        i, i, i, i, i, i]
        lib.la_ref_backward.restype = i
        if hasattr(lib, "la_ref_wkv4"):
            lib.la_ref_wkv4.argtypes = [d, d, d, d, d, d, d, i, i, i]
            lib.la_ref_wkv4.restype = i
        if hasattr(lib, "la_ref_ema"):
            lib.la_ref_ema.argtypes = [d, d, d, d, d, i, i, i, i]
            lib.la_ref_ema.restype = i
        _libs[path] = lib
    return _libs[path]


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor: exact up-cast on the CPU
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _kind(decay_kind):
    return DECAY_KINDS[decay_kind] if not isinstance(decay_kind, int) else decay_kind


def forward(q, k, v, decay_kind=0, log_g=None, normalize=False,
            init_state=None, init_z=None, nthreads=None, lib=None):
    """Recurrent float64 forward.  Shapes as in include/la.h.

    Returns (y [B,H,T,Dv], final_state [B,H,Dk,Dv], final_z [B,H,Dk]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    log_g, init_state, init_z = _f64(log_g), _f64(init_state), _f64(init_z)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    y = np.zeros((B, H, T, Dv))
    S = np.zeros((B, H, Dk, Dv))
    z = np.zeros((B, H, Dk))
    nt = nthreads if nthreads else (os.cpu_count() or 1)
    rc = (lib or load_library()).la_ref_forward(_ptr(q), _ptr(k), _ptr(v), _kind(decay_kind), _ptr(log_g),
                                int(bool(normalize)), _ptr(init_state), _ptr(init_z),
                                _ptr(y), _ptr(S), _ptr(z), B, H, T, Dk, Dv, nt)
    if rc != 0:
        raise ValueError("la_ref_forward rejected its arguments")
    if not normalize:
        z = None
    return y, S, z


def backward(q, k, v, dy, decay_kind=0, log_g=None, normalize=False, init_state=None, init_z=None,
             d_final_state=None, d_final_z=None, nthreads=None, lib=None):
    """Gradients of L = sum_t dy_t . y_t + <d_final_state, S_T> + <d_final_z, z_T>
    through forward(q, k, v, decay_kind, log_g, normalize, init_state, init_z),
    float64, by reverse-mode differentiation of the recurrence (la_ref.c).

    Returns (dq, dk, dv, dlog_g, d_init_state, d_init_z): dlog_g has the shape
    of log_g ([H]: the per-step gradients summed over b and t, since every step
    of head h shares log g_h; [B,H,T]; None without decay); d_init_z is None
    unless normalize.
    """
    q, k, v, dy = _f64(q), _f64(k), _f64(v), _f64(dy)
    log_g, init_state, init_z = _f64(log_g), _f64(init_state), _f64(init_z)
    d_final_state, d_final_z = _f64(d_final_state), _f64(d_final_z)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    kind = _kind(decay_kind)
    dq, dk, dv = np.zeros((B, H, T, Dk)), np.zeros((B, H, T, Dk)), np.zeros((B, H, T, Dv))
    dlog = np.zeros((B, H, T))
    dS0, dz0 = np.zeros((B, H, Dk, Dv)), np.zeros((B, H, Dk))
    nt = nthreads if nthreads else (os.cpu_count() or 1)
    rc = (lib or load_library()).la_ref_backward(
        _ptr(q), _ptr(k), _ptr(v), kind, _ptr(log_g), int(bool(normalize)), _ptr(init_state), _ptr(init_z),
        _ptr(dy), _ptr(d_final_state), _ptr(d_final_z), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlog),
        _ptr(dS0), _ptr(dz0), B, H, T, Dk, Dv, nt)
    if rc != 0:
        raise ValueError("la_ref_backward rejected its arguments")
    dlog_g = None
    if kind == 1:
        dlog_g = dlog.sum(axis=(0, 2))
    elif kind == 2:
        dlog_g = dlog
    return dq, dk, dv, dlog_g, dS0, (dz0 if normalize else None)


def ema(x, f, init_state=None, reverse=False, lib=None):
    """Cumulative EMA along T, float64 (ema_ref.c: RetNet issue 21's
    cumulative_ema): s <- f_t s + x_t per channel, out_t = s.  x, f
    [B,T,C]; init_state [B,C] or None (0).  Returns (out [B,T,C], final
    state [B,C])."""
    x, f, init_state = _f64(x), _f64(f), _f64(init_state)
    B, T, C = x.shape
    out = np.zeros((B, T, C))
    fin = np.zeros((B, C))
    rc = (lib or load_library()).la_ref_ema(_ptr(x), _ptr(f), _ptr(init_state), _ptr(out), _ptr(fin), B, T, C,
                                            int(bool(reverse)))
    if rc != 0:
        raise ValueError("la_ref_ema rejected its arguments")
    return out, fin


WKV4_EMPTY_SCALE = -1e38  # pp of an empty RWKV-4 state (aa = bb = 0)


def wkv4(k, v, w, u, init_state=None, lib=None):
    """RWKV-4 WKV recurrence, float64 (wkv4_ref.c: formula 14 of
    BlinkDL/RWKV-LM issue 167 evaluated as an online weighted mean).  k, v
    [B,T,C]; w (log decay, <= 0), u (bonus) [C]; init_state [B,3,C] (planes
    aa, bb, pp: the sums e^pp aa and e^pp bb) or None for an empty state.
    Returns (out [B,T,C], final_state [B,3,C]) with the final state written
    as (weighted mean, 1, log of the total weight)."""
    k, v, w, u, init_state = _f64(k), _f64(v), _f64(w), _f64(u), _f64(init_state)
    B, T, C = k.shape
    out = np.zeros((B, T, C))
    fin = np.zeros((B, 3, C))
    rc = (lib or load_library()).la_ref_wkv4(_ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(init_state), _ptr(out),
                                             _ptr(fin), B, T, C)
    if rc != 0:
        raise ValueError("la_ref_wkv4 rejected its arguments")
    return out, fin


def wkv4_direct(k, v, w, u, init_state=None):
    """The RWKV-4 WKV output written out as its definition, float64 numpy,
    O(T^2 C): wkv_t = (e^{t w + pp0} aa0 + sum_{i<t} e^{(t-1-i) w + k_i} v_i
    + e^{u + k_t} v_t) / (e^{t w + pp0} bb0 + sum_{i<t} e^{(t-1-i) w + k_i}
    + e^{u + k_t}) with 0-based t (BlinkDL/RWKV-LM issue 167's formula 14 as
    the loop computes it).  Forms the exponentials directly: callers keep the
    exponents moderate (or shift k, which the ratio ignores)."""
    k, v, w, u = _f64(k), _f64(v), _f64(w), _f64(u)
    B, T, C = k.shape
    out = np.zeros((B, T, C))
    for t in range(T):
        lag = (t - 1 - np.arange(t))[None, :, None] * w[None, None, :]   # [1, t, C]
        wt = np.exp(lag + k[:, :t])                                      # [B, t, C]
        cur = np.exp(u[None, :] + k[:, t])                               # [B, C]
        num = (wt * v[:, :t]).sum(axis=1) + cur * v[:, t]
        den = wt.sum(axis=1) + cur
        if init_state is not None:
            s = _f64(init_state)
            g = np.exp(t * w[None, :] + s[:, 2])
            num = num + g * s[:, 0]
            den = den + g * s[:, 1]
        out[:, t] = num / den
    return out


def decode_step(q, k, v, state, z=None, decay_kind=0, log_g=None, normalize=False, lib=None):
    """One token; q, k [B,H,Dk], v [B,H,Dv].  Returns (y, new_state, new_z)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    log_g = _f64(log_g)
    state = _f64(state).copy()
    z = _f64(z).copy() if z is not None else None
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    y = np.zeros((B, H, Dv))
    rc = (lib or load_library()).la_ref_decode_step(_ptr(q), _ptr(k), _ptr(v), _kind(decay_kind), _ptr(log_g),
                                    int(bool(normalize)), _ptr(state), _ptr(z), _ptr(y),
                                    B, H, Dk, Dv)
    if rc != 0:
        raise ValueError("la_ref_decode_step rejected its arguments")
    return y, state, z


def _flip_time(a, axis):
    return None if a is None else np.ascontiguousarray(np.flip(a, axis=axis))


def reverse(q, k, v, decay_kind=0, log_g=None, normalize=False,
            init_state=None, init_z=None, nthreads=None, lib=None):
    """Reverse scan, float64.  Jamie-Stirling/RetNet issue 21 (the
    cumulative_ema docstring): with reverse=True the result is the reverse of
    the non-reversed call on arguments reversed along time.  So, per sequence,
    S_t = g_t S_{t+1} + k_t v_t^T and z_t = g_t z_{t+1} + k_t for t = T..1,
    y_t = q_t^T S_t (or / q_t^T z_t).  init_state / init_z enter from beyond
    token T (decayed by g_T); the returned state is the one at token 1.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    log_g = _f64(log_g)
    kind = _kind(decay_kind)
    lg = _flip_time(log_g, 2) if kind == 2 else log_g
    y, S, z = forward(_flip_time(q, 2), _flip_time(k, 2), _flip_time(v, 2), kind, lg, normalize,
                      init_state, init_z, nthreads=nthreads, lib=lib)
    return np.ascontiguousarray(y[:, :, ::-1]), S, z


def bidirectional(q, k, v, decay_kind=0, log_g=None, normalize=False, nthreads=None, lib=None):
    """Bidirectional encoder, float64: the forward scan plus the reverse scan
    (RetNet issue 21, Details, closing remark: an encoder built from one
    reverse=False and one reverse=True retention; read as their sum, so the
    diagonal term appears in both).  No carried state."""
    yf, _, _ = forward(q, k, v, decay_kind, log_g, normalize, nthreads=nthreads, lib=lib)
    yr, _, _ = reverse(q, k, v, decay_kind, log_g, normalize, nthreads=nthreads, lib=lib)
    return yf + yr
