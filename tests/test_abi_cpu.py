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
    return sorted(set(re.findall(r"\b(la_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("la_chunk_forward", "la_decode_step", "la_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", la.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (la_[a-z_]+)\b", out))
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
    (dict(Dk=48), 2),                     # bf16 tensor-core path: widths 16/32/64/128
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
