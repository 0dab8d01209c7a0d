"""Out-of-bounds write checks on the GPU path (in place of a memory checker):
every output, in-place state and workspace is a view in the middle of a
larger buffer whose bands before and after it hold a NaN bit pattern; after
the call the bands must be unchanged and the outputs must match the float64
oracle.  The cases are the ragged ones, where tail chunks, tail tiles and
partial value slices end inside a tile: T in {1, 2, 127, 129, 255, 257},
widths that run on padded kernel instances, decode with widths 5 and 7, and
the per-channel scans with C not a multiple of their 64-channel tiles."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, gen_case, oracle_forward, rel_err, to_dev

pytestmark = pytest.mark.gpu

BAND = 4096 + 16  # bytes on each side; the odd 16 also moves the view off 32-byte alignment
CANARY = {2: 0x7FA5, 4: 0x7FA5A5A5, 1: 0xA5}  # quiet-NaN payloads (bf16, fp32), a byte pattern (uint8)
INT_OF = {2: torch.int16, 4: torch.int32, 1: torch.uint8}


@pytest.fixture(scope="module", autouse=True)
def built():
    from retention_scan_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    import retention_scan_b200 as la
    assert la.device_error() == 0, "a kernel gave up waiting on a barrier"


def la():
    import retention_scan_b200
    return retention_scan_b200


class Guarded:
    """A tensor of `shape` inside a buffer with canary bands before and after."""

    def __init__(self, shape, dtype, shift=0, init=None):
        es = torch.tensor([], dtype=dtype).element_size()
        self.n = int(np.prod(shape)) if len(shape) else 1
        self.band = (BAND + shift) // es
        self.buf = torch.empty(self.band * 2 + self.n, dtype=dtype, device="cuda")
        pat = CANARY[es]
        raw = self.buf.view(INT_OF[es])
        raw.fill_(pat - (1 << (8 * es)) if pat >= 1 << (8 * es - 1) and es > 1 else pat)
        self.pattern = raw[:1].clone()
        self.t = self.buf[self.band:self.band + self.n].view(shape)
        if init is not None:
            self.t.copy_(init)

    def intact(self):
        es = self.buf.element_size()
        raw = self.buf.view(INT_OF[es])
        lo, hi = raw[:self.band], raw[self.band + self.n:]
        return bool((lo == self.pattern).all()) and bool((hi == self.pattern).all())


def _ws_bytes(B, H, T, Dk, Dv, dtype, normalize):
    return la().workspace_size(B, H, T, Dk, Dv, dtype, normalize)


@pytest.mark.parametrize("T", [1, 2, 127, 129, 255, 257])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("reverse", [False, True])
def test_forward_bands(T, dtype, reverse):
    B, H, Dk, Dv = 1, 3, 64, 48 if dtype == torch.bfloat16 else 40
    inp, S0, z0 = gen_case(B, H, T, Dk, Dv, dtype=dtype, kind=2, normalize=True, init=True, seed=8000 + T)
    d = to_dev(inp)
    out = Guarded((B, H, T, Dv), dtype, shift=16 * (T % 2))
    fs = Guarded((B, H, Dk, Dv), torch.float32)
    fz = Guarded((B, H, Dk), torch.float32)
    la().chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"], True, S0.cuda(), z0.cuda(), out=out.t,
                       final_state=fs.t, final_z=fz.t, reverse=reverse)
    torch.cuda.synchronize()
    assert out.intact() and fs.intact() and fz.intact()
    ref = (oracle.reverse if reverse else oracle.forward)(inp["q"], inp["k"], inp["v"], 2, inp["log_g"], True, S0, z0)
    tol = TOL[dtype]
    assert rel_err(out.t, ref[0]) <= tol and rel_err(fs.t, ref[1]) <= tol and rel_err(fz.t, ref[2]) <= tol


@pytest.mark.parametrize("Dk,Dv", [(48, 80), (112, 96), (16, 112)])
@pytest.mark.parametrize("segments", [1, 3])
def test_forward_bands_padded_widths_and_workspace(monkeypatch, Dk, Dv, segments):
    """Key tiles wider than Dk, a last value slice past Dv, and (with
    segments) the workspace of the state pass, all inside guard bands."""
    monkeypatch.setenv("LA_SEGMENTS", str(segments))
    B, H, T = 1, 2, 128 * 7 + 3
    inp, S0, _ = gen_case(B, H, T, Dk, Dv, kind=2, init=True, seed=8100 + Dk + Dv + segments, decay_mean=4.0)
    d = to_dev(inp)
    out = Guarded((B, H, T, Dv), torch.bfloat16)
    fs = Guarded((B, H, Dk, Dv), torch.float32)
    nb = _ws_bytes(B, H, T, Dk, Dv, torch.bfloat16, False)
    ws = Guarded((max(nb, 16),), torch.uint8)
    la().chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"], False, S0.cuda(), out=out.t, final_state=fs.t,
                       workspace=ws.t if nb else None)
    torch.cuda.synchronize()
    assert out.intact() and fs.intact() and ws.intact()
    yr, Sr, _ = oracle_forward(inp, False, S0)
    assert rel_err(out.t, yr) <= 2e-2 and rel_err(fs.t, Sr) <= 2e-2


@pytest.mark.parametrize("Dk,Dv", [(5, 7), (7, 5), (128, 128)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_bands(Dk, Dv, dtype):
    B, H = 3, 2
    inp, S0, z0 = gen_case(B, H, 1, Dk, Dv, dtype=dtype, kind=1, normalize=True, init=True, seed=8200 + Dk)
    d = to_dev(inp)
    S = Guarded((B, H, Dk, Dv), torch.float32, init=S0.cuda())
    z = Guarded((B, H, Dk), torch.float32, init=z0.cuda())
    out = Guarded((B, H, Dv), dtype)
    la().decode_step(d["q"][:, :, 0].contiguous(), d["k"][:, :, 0].contiguous(), d["v"][:, :, 0].contiguous(),
                     S.t, z.t, 1, d["log_g"], True, out=out.t)
    torch.cuda.synchronize()
    assert out.intact() and S.intact() and z.intact()
    yr, Sr, zr = oracle_forward(inp, True, S0, z0)
    assert rel_err(out.t, yr[:, :, 0]) <= TOL[dtype] and rel_err(S.t, Sr) <= 1e-5 and rel_err(z.t, zr) <= 1e-5


@pytest.mark.parametrize("T", [1, 33, 257])
@pytest.mark.parametrize("C,dtype", [(72, torch.bfloat16), (100, torch.float32), (136, torch.bfloat16)])
def test_wkv4_bands(T, C, dtype):
    B = 2
    g = torch.Generator().manual_seed(8300 + T + C)
    k, v = (torch.randn(B, T, C, generator=g).to(dtype) for _ in range(2))
    w, u = -torch.exp(torch.randn(C, generator=g)), torch.randn(C, generator=g)
    out = Guarded((B, T, C), dtype)
    fin = Guarded((B, 3, C), torch.float32)
    nb = la().wkv4_workspace_size(B, T, C, dtype)
    ws = Guarded((max(nb, 16),), torch.uint8)
    la().wkv4_forward(k.cuda(), v.cuda(), w.cuda(), u.cuda(), out=out.t, final_state=fin.t,
                      workspace=ws.t if nb else False)
    torch.cuda.synchronize()
    assert out.intact() and fin.intact() and ws.intact()
    ro, _ = oracle.wkv4(k, v, w, u)
    assert float(np.max(np.abs(out.t.cpu().double().numpy() - ro)) / np.max(np.abs(ro))) <= TOL[dtype]


@pytest.mark.parametrize("T", [1, 65, 257])
@pytest.mark.parametrize("C,dtype", [(72, torch.bfloat16), (100, torch.float32)])
@pytest.mark.parametrize("reverse", [False, True])
def test_ema_bands(T, C, dtype, reverse):
    B = 2
    g = torch.Generator().manual_seed(8400 + T + C)
    x = torch.randn(B, T, C, generator=g).to(dtype)
    f = torch.sigmoid(torch.randn(B, T, C, generator=g) + 3).to(dtype)
    out = Guarded((B, T, C), dtype)
    fin = Guarded((B, C), torch.float32)
    la().ema_scan(x.cuda(), f.cuda(), reverse=reverse, out=out.t, final_state=fin.t)
    torch.cuda.synchronize()
    assert out.intact() and fin.intact()
    ro, _ = oracle.ema(x, f, reverse=reverse)
    assert float(np.max(np.abs(out.t.cpu().double().numpy() - ro)) / np.max(np.abs(ro))) <= TOL[dtype]


@pytest.mark.parametrize("Dk,Dv", [(64, 48), (48, 112)])
def test_backward_bands(Dk, Dv):
    B, H, T = 1, 2, 129
    inp, S0, _ = gen_case(B, H, T, Dk, Dv, kind=2, init=True, seed=8500 + Dk)
    d = to_dev(inp)
    dy = torch.randn(B, H, T, Dv, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    gq = Guarded((B, H, T, Dk), torch.bfloat16)
    gk = Guarded((B, H, T, Dk), torch.bfloat16)
    gv = Guarded((B, H, T, Dv), torch.bfloat16)
    glg = Guarded((B, H, T), torch.float32)
    gS = Guarded((B, H, Dk, Dv), torch.float32)
    nb = la().backward_workspace_size(B, H, T, Dk, Dv, torch.bfloat16, 2)
    ws = Guarded((nb,), torch.uint8)
    la().chunk_backward(d["q"], d["k"], d["v"], dy.cuda(), 2, d["log_g"], S0.cuda(), workspace=ws.t,
                        out=(gq.t, gk.t, gv.t, glg.t, gS.t))
    torch.cuda.synchronize()
    assert all(g.intact() for g in (gq, gk, gv, glg, gS, ws))
    rq, rk, rv, _, rS0, _ = oracle.backward(inp["q"], inp["k"], inp["v"], dy, 2, inp["log_g"], False, S0)
    for x, r in ((gq.t, rq), (gk.t, rk), (gv.t, rv), (gS.t, rS0)):
        assert rel_err(x, r) <= 2e-2
