"""GPU parity of the cumulative EMA (la_ema_scan; RetNet issue 21's
cumulative_ema, values and factors scanned along T per channel, forward and
reverse) against the float64 oracle, through the C ABI.  Bar: per batch
row, max|x - ref| / max|ref| at most 1e-4 for fp32 inputs and 2e-2 for bf16
inputs (the kernel computes in fp32; bf16 rounds the stored output)."""
import pytest
import torch

import oracle
import workloads as W
from parity import TOL
from test_wkv4_gpu import row_err

pytestmark = pytest.mark.gpu


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


def case(B, T, C, dtype, init, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, C, generator=g).to(dtype)
    f = torch.sigmoid(torch.randn(B, T, C, generator=g) + 3.0).to(dtype)
    s0 = torch.randn(B, C, generator=g) if init else None
    return x, f, s0


def check(x, f, s0, reverse, tol=None):
    tol = tol or TOL[x.dtype]
    out, fin = la().ema_scan(x.cuda(), f.cuda(), None if s0 is None else s0.cuda(), reverse=reverse)
    torch.cuda.synchronize()
    ro, rf = oracle.ema(x, f, s0, reverse=reverse)
    errs = (row_err(out, ro), row_err(fin, rf))
    assert max(errs) <= tol, errs


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("T", [1, 31, 32, 33, 500])
@pytest.mark.parametrize("C", [4, 36])
def test_ema_fp32(T, C, init, reverse):
    check(*case(2, T, C, torch.float32, init, seed=7000 + T + C), reverse)


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 1000, 4096 + 7])
@pytest.mark.parametrize("C", [8, 72, 192])
def test_ema_bf16(T, C, init, reverse):
    check(*case(2, T, C, torch.bfloat16, init, seed=7100 + T + C), reverse)


def test_ema_factor_one_is_a_cumulative_sum():
    x = torch.randn(2, 300, 64).to(torch.float32)
    out, fin = la().ema_scan(x.cuda(), torch.ones_like(x).cuda())
    torch.cuda.synchronize()
    ref = torch.cumsum(x.double(), dim=1).numpy()
    assert row_err(out, ref) <= 1e-5


def test_ema_split_and_carry_in_place():
    x, f, s0 = case(3, 777, 128, torch.bfloat16, True, seed=7200)
    xd, fd = x.cuda(), f.cuda()
    full, ffin = la().ema_scan(xd, fd, s0.cuda())
    state = s0.cuda().clone()
    a, _ = la().ema_scan(xd[:, :300].contiguous(), fd[:, :300].contiguous(), state, final_state=state)
    b, _ = la().ema_scan(xd[:, 300:].contiguous(), fd[:, 300:].contiguous(), state, final_state=state)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([a, b], 1), full)
    assert torch.equal(state, ffin)


def test_ema_empty_sequence():
    x = torch.zeros(2, 0, 16, dtype=torch.bfloat16, device="cuda")
    _, fin = la().ema_scan(x, x)
    torch.cuda.synchronize()
    assert torch.all(fin == 0)
    s0 = torch.randn(2, 16, device="cuda")
    _, fin = la().ema_scan(x, x, s0)
    torch.cuda.synchronize()
    assert torch.equal(fin, s0)


def test_ema_workload_sampled_rows():
    """The bench workload (B8 T4096 C2048 bf16) at full size; two batch rows
    against the oracle."""
    wl = W.EMA
    inp = W.ema_inputs(wl)
    out, fin = la().ema_scan(inp["x"].cuda(), inp["f"].cuda())
    torch.cuda.synchronize()
    for b in (0, 6):
        ro, rf = oracle.ema(inp["x"][b:b + 1], inp["f"][b:b + 1])
        assert max(row_err(out[b:b + 1], ro), row_err(fin[b:b + 1], rf)) <= 2e-2
