"""The C-ABI library without a GPU: it loads, exports every symbol that
include/la.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

import retention_scan_b200 as la

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from retention_scan_b200 import build
    build.build()
    return la.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "la.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(la_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("la_chunk_forward", "la_decode_step", "la_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", la.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (la_[a-z0-9_]+)\b", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared in la.h but not exported: {missing}"
    assert set(la.EXPORTED_SYMBOLS) <= exported
    for n in declared_functions():
        assert hasattr(L, n)


def test_status_strings_and_version(L):
    for code in range(4):
        assert L.la_status_string(code)
    assert L.la_status_string(0) == b"LA_OK"
    assert re.fullmatch(rb"\d+\.\d+\.\d+", L.la_version())


def _fwd(L, **over):
    a = dict(q=16, k=16, v=16, decay=None, normalize=0, init_state=None, init_z=None, out=16,
             final_state=None, final_z=None, B=1, H=1, T=4, Dk=16, Dv=16, dtype=1, stream=None)
    a.update(over)
    vp = ctypes.c_void_p
    dec = a["decay"]
    return L.la_chunk_forward(vp(a["q"]), vp(a["k"]), vp(a["v"]),
                              ctypes.byref(dec) if dec is not None else None, a["normalize"],
                              vp(a["init_state"]), vp(a["init_z"]), vp(a["out"]), vp(a["final_state"]),
                              vp(a["final_z"]), a["B"], a["H"], a["T"], a["Dk"], a["Dv"], a["dtype"],
                              vp(a["stream"]))


# None of these reach CUDA: the library validates before it launches.
@pytest.mark.parametrize("over,status", [
    (dict(q=None), 1),
    (dict(out=None), 1),
    (dict(q=8), 1),                       # not 16-byte aligned
    (dict(B=-1), 1),
    (dict(T=-3), 1),
    (dict(Dk=0), 1),
    (dict(dtype=7), 1),
    (dict(normalize=1, init_state=32, init_z=None), 1),   # carried state without its key sum
    (dict(Dk=40), 2),                     # bf16 tensor-core path: multiples of 16 up to 128
    (dict(Dk=144), 2),
    (dict(Dv=256), 2),
    (dict(dtype=0, Dk=129), 2),
], ids=str)
def test_forward_validation(L, over, status):
    assert _fwd(L, **over) == status


def test_decay_descriptor_validation(L):
    assert _fwd(L, decay=la._Decay(5, 64)) == 1
    assert _fwd(L, decay=la._Decay(1, None)) == 1
    assert _fwd(L, decay=la._Decay(2, 2)) == 1       # log_g misaligned


def test_empty_batch_is_a_noop(L):
    assert _fwd(L, B=0) == 0
    assert _fwd(L, H=0, q=None, k=None, v=None, out=None) == 0


def test_decode_validation(L):
    vp = ctypes.c_void_p

    def dec(**over):
        a = dict(q=16, k=16, v=16, normalize=0, state=16, z=None, out=16, B=1, H=1, Dk=16, Dv=16)
        a.update(over)
        return L.la_decode_step(vp(a["q"]), vp(a["k"]), vp(a["v"]), None, a["normalize"],
                                vp(a["state"]), vp(a["z"]), vp(a["out"]), a["B"], a["H"], a["Dk"],
                                a["Dv"], 1, None)
    assert dec(state=None) == 1
    assert dec(normalize=1, z=None) == 1
    assert dec(normalize=1, z=24) == 1
    assert dec(Dk=200) == 2
    assert dec(B=0) == 0


def test_injected_launch_failure(L, monkeypatch):
    # LA_FAULT_INJECT=launch: the library reports a failed launch and enqueues nothing
    code = r'''
import ctypes, sys
sys.path.insert(0, %r)
import retention_scan_b200 as la
L = la.lib()
vp = ctypes.c_void_p
r = L.la_chunk_forward(vp(16), vp(16), vp(16), None, 0, None, None, vp(16), None, None,
                       1, 1, 4, 16, 16, 1, None)
r2 = L.la_decode_step(vp(16), vp(16), vp(16), None, 0, vp(16), None, vp(16), 1, 1, 16, 16, 1, None)
print(r, r2)
''' % ROOT
    env = dict(os.environ, LA_FAULT_INJECT="launch")
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, env=env, check=True)
    assert out.stdout.split() == ["3", "3"]


def _ws_bytes(BH, Dk, Dv, nS):
    b = 4 * BH * nS * (Dk * Dv + Dk + 1)
    return (b + 255) // 256 * 256


def test_workspace_size_follows_the_segment_plan(L, monkeypatch):
    # 148 SMs (the B200 count, also the host default without a device).
    # 32 heads of 16 chunks: too short to cut (segments of at least 16 chunks)
    monkeypatch.delenv("LA_SEGMENTS", raising=False)
    monkeypatch.delenv("LA_DV_SPLIT", raising=False)
    assert L.la_chunk_forward_workspace_size(4, 8, 2048, 64, 64, 1, 0) == 0
    # 8 heads of 64 chunks, Dk = Dv = 64: four segments of 16 chunks, then
    # four value slices (8 x 4 x 4 = 128 CTAs); the state pass runs one
    # 64-column slice, each of the first three segments cut into four state
    # segments (8 x 1 x 3 x 4 = 96 CTAs)
    assert L.la_chunk_forward_workspace_size(1, 8, 8192, 64, 64, 1, 0) == _ws_bytes(8, 64, 64, 12)
    # 32 heads of 512 chunks, Dk = Dv = 128: two value slices, two segments;
    # the state pass runs one 128-column slice, the first segment cut into
    # four state segments (32 x 4 = 128 CTAs)
    assert L.la_chunk_forward_workspace_size(1, 32, 65536, 128, 128, 1, 0) == _ws_bytes(32, 128, 128, 4)
    # 128 heads fill the GPU: no segments
    assert L.la_chunk_forward_workspace_size(8, 16, 4096, 128, 128, 1, 1) == 0
    # fp32, empty or too short inputs: none
    assert L.la_chunk_forward_workspace_size(4, 8, 2048, 64, 64, 0, 0) == 0
    assert L.la_chunk_forward_workspace_size(0, 8, 2048, 64, 64, 1, 0) == 0
    assert L.la_chunk_forward_workspace_size(4, 8, 0, 64, 64, 1, 0) == 0
    assert L.la_chunk_forward_workspace_size(4, 8, 128, 64, 64, 1, 0) == 0
    # an explicit segment count (test override)
    monkeypatch.setenv("LA_SEGMENTS", "5")
    assert L.la_chunk_forward_workspace_size(1, 2, 1100, 64, 64, 1, 0) > 0


def test_segmented_entry_rejects_misaligned_workspace(L):
    buf = ctypes.create_string_buffer(64)
    addr = ctypes.addressof(buf) + 4
    st = L.la_chunk_forward_ws(None, None, None, None, 0, None, None, None, None, None,
                               1, 1, 0, 16, 16, 1, ctypes.c_void_p(addr), 60, None)
    assert st == 1  # LA_ERR_INVALID_ARG


def test_reverse_and_bidirectional_validate_like_the_forward(L):
    vp = ctypes.c_void_p

    def rev(**over):
        a = dict(q=16, k=16, v=16, out=16, B=1, H=1, T=4, Dk=16, Dv=16, dtype=1, normalize=0,
                 init_state=None, init_z=None)
        a.update(over)
        return L.la_chunk_reverse_ws(vp(a["q"]), vp(a["k"]), vp(a["v"]), None, a["normalize"],
                                     vp(a["init_state"]), vp(a["init_z"]), vp(a["out"]), None, None,
                                     a["B"], a["H"], a["T"], a["Dk"], a["Dv"], a["dtype"], None, 0, None)

    def bi(**over):
        a = dict(q=16, k=16, v=16, out=16, B=1, H=1, T=4, Dk=16, Dv=16, dtype=1, normalize=0, ws=None)
        a.update(over)
        return L.la_chunk_bidirectional_ws(vp(a["q"]), vp(a["k"]), vp(a["v"]), None, a["normalize"],
                                           vp(a["out"]), a["B"], a["H"], a["T"], a["Dk"], a["Dv"], a["dtype"],
                                           vp(a["ws"]), 64, None)
    for f in (rev, bi):
        assert f(q=None) == 1
        assert f(out=8) == 1
        assert f(T=-1) == 1
        assert f(dtype=9) == 1
        assert f(Dk=40) == 2
        assert f(dtype=0, Dv=200) == 2
        assert f(B=0) == 0
    assert rev(normalize=1, init_state=32, init_z=None) == 1
    assert bi(ws=4) == 1  # misaligned workspace


def test_injected_launch_failure_reverse_and_bidirectional():
    code = r'''
import ctypes, sys
sys.path.insert(0, %r)
import retention_scan_b200 as la
L = la.lib()
vp = ctypes.c_void_p
r = L.la_chunk_reverse_ws(vp(16), vp(16), vp(16), None, 0, None, None, vp(16), None, None,
                          1, 1, 4, 16, 16, 1, None, 0, None)
r2 = L.la_chunk_bidirectional_ws(vp(16), vp(16), vp(16), None, 0, vp(16), 1, 1, 4, 16, 16, 1, None, 0, None)
print(r, r2)
''' % ROOT
    env = dict(os.environ, LA_FAULT_INJECT="launch")
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, env=env, check=True)
    assert out.stdout.split() == ["3", "3"]


def _bwd(L, **over):
    """la_chunk_backward_ws with fake (never dereferenced) aligned addresses."""
    vp = ctypes.c_void_p
    a = dict(q=16, k=16, v=16, decay=None, init_state=None, dy=16, dSf=None, dq=16, dk=16, dv=16,
             dlog=None, dS0=None, B=1, H=1, T=4, Dk=16, Dv=16, dtype=1, ws=256, ws_bytes=None)
    a.update(over)
    if a["ws_bytes"] is None:
        a["ws_bytes"] = L.la_chunk_backward_workspace_size(a["B"], a["H"], max(a["T"], 1), a["Dk"], a["Dv"],
                                                           a["dtype"] if a["dtype"] in (0, 1) else 1,
                                                           a["decay"].kind if a["decay"] is not None else 0)
    dec = a["decay"]
    return L.la_chunk_backward_ws(vp(a["q"]), vp(a["k"]), vp(a["v"]), ctypes.byref(dec) if dec is not None else None,
                                  vp(a["init_state"]), vp(a["dy"]), vp(a["dSf"]), vp(a["dq"]), vp(a["dk"]),
                                  vp(a["dv"]), vp(a["dlog"]), vp(a["dS0"]), a["B"], a["H"], a["T"], a["Dk"],
                                  a["Dv"], a["dtype"], vp(a["ws"]), a["ws_bytes"], None)


# None of these reach CUDA: the backward validates before it launches.
@pytest.mark.parametrize("over,status", [
    (dict(dy=None), 1),
    (dict(dq=None), 1),
    (dict(dv=8), 1),                          # not 16-byte aligned
    (dict(ws=None), 1),                       # the backward needs its workspace
    (dict(ws=264), 1),                        # misaligned workspace
    (dict(ws_bytes=64), 1),                   # workspace too small
    (dict(dlog=64), 1),                       # a decay gradient without a decay
    (dict(decay=la._Decay(1, 64), dlog=2), 1),  # d_log_g misaligned
    (dict(dS0=8), 1),
    (dict(T=-1), 1),
    (dict(dtype=5), 1),
    (dict(Dk=40), 2),
    (dict(dtype=0, Dv=130), 2),
    (dict(B=0), 0),                           # empty batch: a no-op
], ids=str)
def test_backward_validation(L, over, status):
    assert _bwd(L, **over) == status


def test_backward_workspace_size(L):
    # S_0^T, d_final_state^T, S_T^T, the shifted decay, the decay-gradient
    # scratch and the scans' T-segment workspace, each rounded to 256 bytes,
    # then a second scan workspace: the dk and dv scans share their state
    # pieces (same plan), which the dv scan takes transposed
    def r(x):
        return (x + 255) // 256 * 256
    B, H, T, D = 1, 8, 8192, 64
    state = r(4 * B * H * D * D)
    nblk = (T + 255) // 256
    scan = L.la_chunk_forward_workspace_size(B, H, T, D, D, 1, 0)
    want = 3 * state + r(4 * B * H * T) + r(8 * (B * H + 3 * B * H * nblk)) + 2 * r(scan)
    assert L.la_chunk_backward_workspace_size(B, H, T, D, D, 1, 2) == want
    assert L.la_chunk_backward_workspace_size(B, H, T, D, D, 1, 0) == want - r(4 * B * H * T)
    assert L.la_chunk_backward_workspace_size(B, H, T, D, D, 0, 2) == want - 2 * r(scan)  # fp32: no segments
    assert L.la_chunk_backward_workspace_size(0, H, T, D, D, 1, 0) == 0
    assert L.la_chunk_backward_workspace_size(B, H, T, D, D, 1, 3) == 0


def test_injected_launch_failure_backward():
    code = r'''
import ctypes, sys
sys.path.insert(0, %r)
import retention_scan_b200 as la
L = la.lib()
vp = ctypes.c_void_p
n = L.la_chunk_backward_workspace_size(1, 1, 4, 16, 16, 1, 0)
print(L.la_chunk_backward_ws(vp(16), vp(16), vp(16), None, None, vp(16), None, vp(16), vp(16), vp(16),
                             None, None, 1, 1, 4, 16, 16, 1, vp(256), n, None))
''' % ROOT
    env = dict(os.environ, LA_FAULT_INJECT="launch")
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, env=env, check=True)
    assert out.stdout.split() == ["3"]


def _wkv(L, **over):
    vp = ctypes.c_void_p
    a = dict(k=16, v=16, w=4, u=4, S0=None, out=16, Sf=None, B=1, T=4, C=8, dtype=1)
    a.update(over)
    return L.la_wkv4_forward(vp(a["k"]), vp(a["v"]), vp(a["w"]), vp(a["u"]), vp(a["S0"]), vp(a["out"]),
                             vp(a["Sf"]), a["B"], a["T"], a["C"], a["dtype"], None)


# None of these reach CUDA.
@pytest.mark.parametrize("over,status", [
    (dict(k=None), 1),
    (dict(out=None), 1),
    (dict(w=None), 1),
    (dict(u=2), 1),                      # not 4-byte aligned
    (dict(v=8), 1),                      # not 16-byte aligned
    (dict(S0=6), 1),
    (dict(B=-1), 1),
    (dict(C=0), 1),
    (dict(dtype=3), 1),
    (dict(C=12), 2),                     # bf16 rows: C a multiple of 8
    (dict(C=6, dtype=0), 2),             # fp32 rows: C a multiple of 4
    (dict(B=70000), 2),
    (dict(B=0), 0),
], ids=str)
def test_wkv4_validation(L, over, status):
    assert _wkv(L, **over) == status


def test_wkv4_workspace_size(L):
    # 148 SMs (the host default without a device), eight CTAs per SM, CTAs of
    # 64 channels: B8 C2048 (256 CTAs) doubles twice to four segments of 1024
    # tokens; one CTA and T = 4173 reaches eight segments of at least 512
    assert L.la_wkv4_workspace_size(8, 4096, 2048, 1) == 8 * 4 * 3 * 2048 * 4
    assert L.la_wkv4_workspace_size(1, 4173, 64, 1) == 1 * 8 * 3 * 64 * 4
    assert L.la_wkv4_workspace_size(2, 1000, 192, 1) == 0   # segments would be shorter than 512 tokens
    assert L.la_wkv4_workspace_size(0, 4096, 64, 1) == 0
    assert L.la_wkv4_workspace_size(1, 4096, 64, 9) == 0
    vp = ctypes.c_void_p
    assert L.la_wkv4_forward_ws(vp(16), vp(16), vp(4), vp(4), None, vp(16), None, 1, 4, 8, 1, vp(24), 64,
                                None) == 1  # misaligned workspace


def test_prologue_validation(L):
    vp = ctypes.c_void_p

    def fwd(pro, dtype=1):
        return L.la_chunk_forward_pro_ws(vp(16), vp(16), vp(16), None, 0, ctypes.byref(pro) if pro else None,
                                         None, None, vp(16), None, None, 1, 1, 4, 16, 16, dtype, None, 0, None)

    def dec(pro):
        return L.la_decode_step_pro(vp(16), vp(16), vp(16), None, 0, ctypes.byref(pro), vp(16), None, vp(16),
                                    1, 1, 16, 16, 1, None)
    P = la._Prologue
    assert fwd(P(2, 1.0)) == 1                   # feature map out of range
    assert fwd(P(0, float("inf"))) == 1          # q scale not finite
    assert fwd(P(0, float("nan"))) == 1
    # the bf16 tensor-core path takes the feature map too: its argument
    # checks pass, and an unsupported width still gives LA_ERR_UNSUPPORTED
    assert L.la_chunk_forward_pro_ws(vp(16), vp(16), vp(16), None, 0, ctypes.byref(P(1, 1.0)), None, None, vp(16),
                                     None, None, 1, 1, 4, 40, 16, 1, None, 0, None) == 2
    assert L.la_chunk_forward_pro_ws(None, None, None, None, 0, ctypes.byref(P(1, 1.0)), None, None, None, None,
                                     None, 0, 1, 4, 16, 16, 1, None, 0, None) == 0
    assert dec(P(-1, 1.0)) == 1
    assert dec(P(0, float("inf"))) == 1
    # B = 0 with valid prologues: no-ops (the fp32 path takes the feature map)
    assert L.la_chunk_forward_pro_ws(None, None, None, None, 0, ctypes.byref(P(1, 0.5)), None, None, None, None,
                                     None, 0, 1, 4, 16, 16, 0, None, 0, None) == 0


def test_backward_norm_validation(L):
    vp = ctypes.c_void_p

    def bn(**over):
        a = dict(q=16, k=16, v=16, init_state=None, init_z=None, dy=16, dq=16, dk=16, dv=16, ws=256, B=1, T=4)
        a.update(over)
        n = L.la_chunk_backward_norm_workspace_size(1, 1, max(a["T"], 1), 16, 16, 1, 0)
        return L.la_chunk_backward_norm_ws(vp(a["q"]), vp(a["k"]), vp(a["v"]), None, vp(a["init_state"]),
                                           vp(a["init_z"]), vp(a["dy"]), None, None, vp(a["dq"]), vp(a["dk"]),
                                           vp(a["dv"]), None, None, None, a["B"], 1, a["T"], 16, 16, 1,
                                           vp(a["ws"]), n, None)
    assert bn(init_state=32, init_z=None) == 1   # a carried state without its key sum
    assert bn(dy=None) == 1
    assert bn(ws=None) == 1
    assert bn(dk=8) == 1
    assert bn(B=0) == 0
    assert L.la_chunk_backward_norm_workspace_size(1, 8, 8192, 64, 64, 1, 2) > \
        L.la_chunk_backward_workspace_size(1, 8, 8192, 64, 64, 1, 2)


def test_ema_validation(L):
    vp = ctypes.c_void_p

    def ema(**over):
        a = dict(x=16, f=16, s0=None, out=16, sf=None, B=1, T=4, C=8, dtype=1, rev=0)
        a.update(over)
        return L.la_ema_scan(vp(a["x"]), vp(a["f"]), vp(a["s0"]), vp(a["out"]), vp(a["sf"]), a["B"], a["T"], a["C"],
                             a["dtype"], a["rev"], None)
    assert ema(x=None) == 1
    assert ema(f=8) == 1          # not 16-byte aligned
    assert ema(s0=2) == 1         # not 4-byte aligned
    assert ema(C=0) == 1
    assert ema(dtype=4) == 1
    assert ema(C=12) == 2         # bf16 rows: C a multiple of 8
    assert ema(C=6, dtype=0) == 2
    assert ema(B=0) == 0


def _state(L, **over):
    a = dict(k=16, v=16, decay=None, norm=0, S=16, z=None, lg=None, B=1, H=1, T=4, Dk=16, Dv=16, dtype=0,
             ws=None, nbytes=0)
    a.update(over)
    vp = ctypes.c_void_p
    dec = a["decay"]
    return L.la_chunk_state_ws(vp(a["k"]), vp(a["v"]), ctypes.byref(dec) if dec is not None else None, a["norm"],
                               vp(a["S"]), vp(a["z"]), vp(a["lg"]), a["B"], a["H"], a["T"], a["Dk"], a["Dv"],
                               a["dtype"], vp(a["ws"]), a["nbytes"], None)


def test_chunk_state_validation(L):
    assert _state(L, k=None) == 1
    assert _state(L, v=8) == 1                   # not 16-byte aligned
    assert _state(L, S=None) == 1                # the state output is required
    assert _state(L, norm=1) == 1                # normalize needs z_out
    assert _state(L, lg=2) == 1                  # not 4-byte aligned
    assert _state(L, Dk=0) == 1
    assert _state(L, dtype=3) == 1
    assert _state(L, decay=la._Decay(7, 16)) == 1
    assert _state(L, decay=la._Decay(2, 0)) == 1  # a decay without its array
    assert _state(L, Dk=200) == 2                # fp32: D above 128
    assert _state(L, Dk=24, dtype=1) == 2        # bf16: D a multiple of 16
    assert _state(L, dtype=1) == 1               # bf16 needs its workspace
    need = L.la_chunk_state_workspace_size(1, 1, 4, 16, 16, 1, 0)
    assert need > 0
    assert _state(L, dtype=1, ws=256, nbytes=need - 16) == 1
    assert _state(L, dtype=1, ws=264, nbytes=need) == 1   # misaligned workspace
    assert _state(L, B=0) == 0


def test_chunk_state_workspace_size(L):
    # 148 SMs (the host default without a device).  32 heads, Dk = Dv = 128:
    # one 128-column slice (the state-pass instance); pieces doubled while
    # 32 x 1 x pieces fits: four
    assert L.la_chunk_state_workspace_size(1, 32, 65536, 128, 128, 1, 0) == _ws_bytes(32, 128, 128, 4)
    # one chunk: one piece
    assert L.la_chunk_state_workspace_size(1, 1, 100, 64, 32, 1, 0) == _ws_bytes(1, 64, 32, 1)
    # fp32 and empty inputs: none
    assert L.la_chunk_state_workspace_size(1, 32, 65536, 128, 128, 0, 0) == 0
    assert L.la_chunk_state_workspace_size(0, 32, 65536, 128, 128, 1, 0) == 0
    assert L.la_chunk_state_workspace_size(1, 32, 0, 128, 128, 1, 0) == 0


def _combine(L, **over):
    a = dict(S=16, z=None, lg=16, ss=256, zs=0, ls=1, n=2, S0=None, z0=None, out=16, zo=None, lo=None,
             B=1, H=1, Dk=4, Dv=4)
    a.update(over)
    vp = ctypes.c_void_p
    return L.la_state_combine(vp(a["S"]), vp(a["z"]), vp(a["lg"]), a["ss"], a["zs"], a["ls"], a["n"], vp(a["S0"]),
                              vp(a["z0"]), vp(a["out"]), vp(a["zo"]), vp(a["lo"]), a["B"], a["H"], a["Dk"],
                              a["Dv"], None)


def test_state_combine_validation(L):
    assert _combine(L, n=-1) == 1
    assert _combine(L, ss=-4) == 1
    assert _combine(L, out=None) == 1            # the state output is required
    assert _combine(L, S=None) == 1              # spans without states
    assert _combine(L, lg=None) == 1             # spans without log decays
    assert _combine(L, zo=32) == 1               # a key-sum output needs the spans' key sums
    assert _combine(L, S0=2) == 1                # not 4-byte aligned
    assert _combine(L, Dv=0) == 1
    assert _combine(L, B=0) == 0


def test_injected_launch_failure_state_entry_points():
    code = r'''
import ctypes, sys
sys.path.insert(0, %r)
import retention_scan_b200 as la
L = la.lib()
vp = ctypes.c_void_p
r = L.la_chunk_state_ws(vp(16), vp(16), None, 0, vp(16), None, None, 1, 1, 4, 16, 16, 0, None, 0, None)
r2 = L.la_state_combine(vp(16), None, vp(16), 256, 0, 1, 2, None, None, vp(16), None, None, 1, 1, 4, 4, None)
print(r, r2)
''' % ROOT
    env = dict(os.environ, LA_FAULT_INJECT="launch")
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, env=env, check=True)
    assert out.stdout.split() == ["3", "3"]
