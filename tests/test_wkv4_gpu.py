"""GPU parity of the RWKV-4 WKV recurrence (la_wkv4_forward; BlinkDL/RWKV-LM
issue 167, formula 14 and its recurrent form) against the float64 oracle,
through the C ABI.

Bar (the library's stated one): per batch row, max|x - ref| / max|ref| at most
1e-4 for fp32 inputs and 2e-2 for bf16 inputs, for the output and for the
final state.  A state (aa, bb, pp) stands for the two sums e^pp aa and
e^pp bb, and the kernel and the oracle write different but equivalent
representatives, so the state is compared as those sums (aa and bb brought
to the oracle's scale) and as the log of the total weight, pp + log bb.  The
kernel computes in fp32 whatever the input type; bf16 only rounds the stored
output."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import TOL

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


def row_err(x, ref):
    """Worst batch row of max|x - ref| / max|ref| (x, ref shaped [B, ...])."""
    x = x.detach().cpu().double().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape
    worst = 0.0
    for a, r in zip(x.reshape(x.shape[0], -1), ref.reshape(ref.shape[0], -1)):
        scale = float(np.max(np.abs(r))) if r.size else 0.0
        err = float(np.max(np.abs(a - r))) if r.size else 0.0
        if not np.isfinite(err):
            return float("inf")
        worst = max(worst, err / scale if scale > 0 else err)
    return worst


def case(B, T, C, dtype=torch.bfloat16, init=False, seed=0, kshift=0.0):
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(B, T, C, generator=g) + kshift).to(dtype)
    v = torch.randn(B, T, C, generator=g).to(dtype)
    w = -torch.exp(torch.randn(C, generator=g) * 1.5 - 1.0)
    u = torch.randn(C, generator=g) * 0.4 - 0.6
    S0 = None
    if init:
        S0 = torch.stack([torch.randn(B, C, generator=g), torch.rand(B, C, generator=g) + 0.1,
                          torch.randn(B, C, generator=g) + kshift], dim=1)
    return k, v, w, u, S0


def state_errs(fin, rf):
    """The state (the sums e^pp aa, e^pp bb) against the oracle's: aa and bb
    brought to the oracle's scale (x e^(pp - pp_ref)), which is what they
    represent, and the log of the total weight pp + log bb (its error is the
    relative error of the total weight).  fp32 rounding of the kernel's running
    scale moves pp by a few ulps of its size and aa, bb with it, without
    changing the sums."""
    f = fin.detach().cpu().double().numpy()
    r = np.asarray(rf, np.float64)
    rescale = np.exp(f[:, 2] - r[:, 2])
    with np.errstate(divide="ignore"):
        logw = np.where(f[:, 1] > 0, f[:, 2] + np.log(np.maximum(f[:, 1], 1e-300)), r[:, 2])
        logw_ref = np.where(r[:, 1] > 0, r[:, 2] + np.log(np.maximum(r[:, 1], 1e-300)), r[:, 2])
    return {"aa": row_err(f[:, 0] * rescale, r[:, 0]), "bb": row_err(f[:, 1] * rescale, r[:, 1]),
            "log_weight": float(np.max(np.abs(logw - logw_ref)))}


def check(k, v, w, u, S0=None, tol=None):
    tol = tol or TOL[k.dtype]
    out, fin = la().wkv4_forward(k.cuda(), v.cuda(), w.cuda(), u.cuda(), None if S0 is None else S0.cuda())
    torch.cuda.synchronize()
    ro, rf = oracle.wkv4(k, v, w, u, S0)
    errs = {"out": row_err(out, ro), **state_errs(fin, rf)}
    assert all(e <= tol for e in errs.values()), errs
    return errs


@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 77, 300])
def test_wkv4_fp32(T, init):
    check(*case(2, T, 40, torch.float32, init, seed=4000 + T))


@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 300, 1000])
@pytest.mark.parametrize("C", [8, 72, 192])
def test_wkv4_bf16(T, C, init):
    check(*case(2, T, C, torch.bfloat16, init, seed=4100 + T + C))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_wkv4_large_keys_stay_finite(dtype):
    """Keys near 100: e^100 overflows fp32, the max-shifted loop does not.
    The output meets the bar.  The state does to a bar derived from fp32:
    the running scale is near 100 (144 in the kernel's log2 units), so each
    step's w + pp rounds by about ulp(144) = 2^-16 relative to what aa and bb
    represent; aa and bb drift together (their ratio, hence the output, does
    not), by up to 8 ulp(144) sqrt(T) here."""
    T = 200
    k, v, w, u, S0 = case(2, T, 64, dtype, True, seed=4200, kshift=100.0)
    out, fin = la().wkv4_forward(k.cuda(), v.cuda(), w.cuda(), u.cuda(), S0.cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(fin).all()
    ro, rf = oracle.wkv4(k, v, w, u, S0)
    assert row_err(out, ro) <= TOL[dtype]
    bar = max(TOL[dtype], 8 * 2.0 ** -16 * T ** 0.5)
    errs = state_errs(fin, rf)
    assert max(errs.values()) <= bar, (errs, bar)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_wkv4_mixed_scales(dtype):
    """Inputs that take every branch of the kernel's per-token work: key
    spikes far above and below the running scale in some channels and some
    tokens (single batches of eight tokens redone token by token), channels
    with a large bonus or a growing factor (w > 0: their warps always step
    token by token), an empty start in one batch row and a carried state at
    a large scale in the other; T and C ragged."""
    B, T, C = 2, 333, 72
    g = torch.Generator().manual_seed(4250)
    k = torch.randn(B, T, C, generator=g)
    spikes = torch.rand(B, T, C, generator=g)
    k = torch.where(spikes < 0.01, k + 70.0, k)
    k = torch.where(spikes > 0.99, k - 120.0, k)
    v = torch.randn(B, T, C, generator=g)
    w = -torch.exp(torch.randn(C, generator=g) * 1.5 - 1.0)
    w[5] = 0.0
    w[40] = 0.05
    w[70] = -60.0
    u = torch.randn(C, generator=g) * 0.4 - 0.6
    u[33] = 30.0
    u[66] = -40.0
    S0 = torch.stack([torch.randn(B, C, generator=g), torch.rand(B, C, generator=g) + 0.1,
                      torch.randn(B, C, generator=g) + 50.0], dim=1)
    S0[0, 0] = 0.0
    S0[0, 1] = 0.0
    S0[0, 2] = oracle.WKV4_EMPTY_SCALE
    k, v = k.to(dtype), v.to(dtype)
    out, fin = la().wkv4_forward(k.cuda(), v.cuda(), w.cuda(), u.cuda(), S0.cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(fin).all()
    ro, rf = oracle.wkv4(k, v, w, u, S0)
    assert row_err(out, ro) <= TOL[dtype]
    # the running scale reaches about 70 (100 in log2 units): the state bar
    # of the large-key case
    bar = max(TOL[dtype], 8 * 2.0 ** -16 * T ** 0.5)
    errs = state_errs(fin, rf)
    assert max(errs.values()) <= bar, (errs, bar)


def test_wkv4_split_and_carry_in_place():
    """Two calls with the state carried in place equal one call."""
    k, v, w, u, S0 = case(3, 257, 128, torch.bfloat16, True, seed=4300)
    kd, vd, wd, ud = k.cuda(), v.cuda(), w.cuda(), u.cuda()
    full, ffin = la().wkv4_forward(kd, vd, wd, ud, S0.cuda())
    state = S0.cuda().clone()
    a, _ = la().wkv4_forward(kd[:, :100].contiguous(), vd[:, :100].contiguous(), wd, ud, state,
                             final_state=state)
    b, _ = la().wkv4_forward(kd[:, 100:].contiguous(), vd[:, 100:].contiguous(), wd, ud, state,
                             final_state=state)
    torch.cuda.synchronize()
    # the carried pp passes through natural-log units (x log2 e and back):
    # about one fp32 rounding, which may move a stored bf16 output by one ulp
    assert row_err(torch.cat([a, b], 1), full.cpu().double().numpy()) <= 1e-2
    assert max(state_errs(state, ffin.cpu().double().numpy()).values()) <= 1e-5


def test_wkv4_empty_sequence():
    B, C = 2, 16
    k = torch.zeros(B, 0, C, dtype=torch.bfloat16, device="cuda")
    w, u = torch.full((C,), -0.5, device="cuda"), torch.zeros(C, device="cuda")
    _, fin = la().wkv4_forward(k, k, w, u)
    torch.cuda.synchronize()
    assert torch.all(fin[:, :2] == 0) and torch.all(fin[:, 2] == oracle.WKV4_EMPTY_SCALE)
    S0 = torch.randn(B, 3, C, device="cuda")
    _, fin = la().wkv4_forward(k, k, w, u, S0)
    torch.cuda.synchronize()
    assert torch.equal(fin, S0)


def test_wkv4_workload_sampled_rows():
    """The bench workload (B8 T4096 C2048 bf16) at full size on the GPU; two
    batch rows against the oracle."""
    wl = W.WKV4
    inp = W.wkv4_inputs(wl)
    out, fin = la().wkv4_forward(inp["k"].cuda(), inp["v"].cuda(), inp["w"].cuda(), inp["u"].cuda())
    torch.cuda.synchronize()
    for b in (0, 5):
        ro, rf = oracle.wkv4(inp["k"][b:b + 1], inp["v"][b:b + 1], inp["w"], inp["u"])
        errs = [row_err(out[b:b + 1], ro)] + list(state_errs(fin[b:b + 1], rf).values())
        assert max(errs) <= 2e-2, (b, errs)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("init", [False, True])
def test_wkv4_t_segments(dtype, init):
    """One channel tile and a long sequence: the library cuts it into
    T-segments (a state pass, then the output pass starting each segment from
    the combined earlier states); ragged last segment."""
    B, T, C = 1, 4096 + 77, 64
    assert la().wkv4_workspace_size(B, T, C, dtype) > 0
    k, v, w, u, S0 = case(B, T, C, dtype, init, seed=4400 + init)
    check(k, v, w, u, S0)
    # the same call without a workspace (one segment) agrees to fp32 rounding
    kd, vd, wd, ud = k.cuda(), v.cuda(), w.cuda(), u.cuda()
    S0d = None if S0 is None else S0.cuda()
    a, fa = la().wkv4_forward(kd, vd, wd, ud, S0d)
    b, fb = la().wkv4_forward(kd, vd, wd, ud, S0d, workspace=False)
    torch.cuda.synchronize()
    assert row_err(a, b.cpu().double().numpy()) <= (1e-5 if dtype == torch.float32 else 1e-2)
    assert max(state_errs(fa, fb.cpu().double().numpy()).values()) <= 1e-5


def test_wkv4_t_segments_in_place():
    """The carried state read and written in place with T-segments."""
    B, T, C = 2, 3000, 128
    k, v, w, u, S0 = case(B, T, C, torch.bfloat16, True, seed=4500)
    assert la().wkv4_workspace_size(B, T, C) > 0
    ro, rf = oracle.wkv4(k, v, w, u, S0)
    state = S0.cuda().clone()
    out, _ = la().wkv4_forward(k.cuda(), v.cuda(), w.cuda(), u.cuda(), state, final_state=state)
    torch.cuda.synchronize()
    assert row_err(out, ro) <= 2e-2
    assert max(state_errs(state, rf).values()) <= 2e-2
