"""la_chunk_forward_noalloc: the forward whose T-segment workspace is a fixed
device array inside the library, so that a call allocates no device memory.
(Named to be collected last: its first GPU call reserves the array.)"""
import ctypes
import math

import pytest
import torch

import retention_scan_b200 as la
from parity import TOL, oracle_forward, rel_err, to_dev

LA_ERR_UNSUPPORTED = 2


@pytest.fixture(scope="module")
def L():
    from retention_scan_b200 import build
    build.build()
    L = la.lib()
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.la_chunk_forward_noalloc.argtypes = [vp, vp, vp, ctypes.POINTER(la._Decay), i, vp, vp, vp, vp, vp,
                                           i, i, i, i, i, i, vp]
    L.la_chunk_forward_noalloc.restype = i
    L.la_chunk_forward_noalloc_capacity.argtypes = []
    L.la_chunk_forward_noalloc_capacity.restype = ctypes.c_size_t
    return L


def test_capacity_and_size_limit(L, monkeypatch):
    cap = L.la_chunk_forward_noalloc_capacity()
    assert cap == 16 << 20
    # 128 heads of 128 x 128 state cut into 64 segments need more than the array:
    # refused before anything is read or enqueued (null pointers are never touched)
    monkeypatch.setenv("LA_SEGMENTS", "64")
    monkeypatch.setenv("LA_DV_SPLIT", "2")
    assert L.la_chunk_forward_workspace_size(8, 16, 65536, 128, 128, 1, 0) > cap
    st = L.la_chunk_forward_noalloc(None, None, None, None, 0, None, None, None, None, None,
                                    8, 16, 65536, 128, 128, 1, None)
    assert st == LA_ERR_UNSUPPORTED


def _case(seed=950):
    g = torch.Generator().manual_seed(seed)
    B, H, T, D = 1, 8, 8192, 128
    q = (torch.randn(B, H, T, D, generator=g) * D ** -0.5).bfloat16()
    k = torch.randn(B, H, T, D, generator=g).bfloat16()
    v = torch.randn(B, H, T, D, generator=g).bfloat16()
    log_g = torch.nn.functional.logsigmoid(torch.randn(B, H, T, generator=g) + 3.0)
    S0 = torch.randn(B, H, D, D, generator=g)
    return dict(q=q, k=k, v=v, log_g=log_g, decay_kind=2), S0


def _call(L, d, S0, out, fs):
    B, H, T, D = d["q"].shape
    dec = la._Decay(2, d["log_g"].data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.la_chunk_forward_noalloc(
        d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), ctypes.byref(dec), 0,
        S0.data_ptr(), None, out.data_ptr(), fs.data_ptr(), None, B, H, T, D, D, 1, stream)


@pytest.mark.gpu
def test_noalloc_parity_and_no_allocation(L):
    inp, S0 = _case()
    B, H, T, D = inp["q"].shape
    need = L.la_chunk_forward_workspace_size(B, H, T, D, D, 1, 0)
    assert 0 < need <= L.la_chunk_forward_noalloc_capacity()  # this shape runs as T-segments
    d = to_dev(inp)
    S0d = S0.cuda()
    out = torch.empty(B, H, T, D, dtype=torch.bfloat16, device="cuda")
    fs = torch.empty(B, H, D, D, dtype=torch.float32, device="cuda")
    assert _call(L, d, S0d, out, fs) == 0  # the first call may load the library's device code
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert _call(L, d, S0d, out, fs) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, "the call allocated device memory"
    assert la.device_error() == 0
    yr, Sr, _ = oracle_forward(inp, False, S0, None)
    tol = TOL[torch.bfloat16]
    assert rel_err(out, yr) <= tol and rel_err(fs, Sr) <= tol
    # same plan and kernels as the caller-workspace entry point: identical bits
    y2, S2, _ = la.chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"], False, S0d)
    torch.cuda.synchronize()
    assert torch.equal(out, y2) and torch.equal(fs, S2)
    assert not math.isnan(float(out.float().abs().max()))
