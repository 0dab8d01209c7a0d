"""GPU parity of the backward pass (la_chunk_backward_ws) against the float64
oracle's chain rule through the recurrence, through the C ABI.

dq, dk, dv and d_init_state: the forward's bar, max relative error per (b, h)
slice 1e-4 for fp32 inputs and 2e-2 for bf16 inputs.

d_log_g: the library forms it as a suffix sum over tokens of
q_s . dq_s - k_s . dk_s (RWKV-LM discussion 189: gradients by cumulative
sums), and each term carries the rounding of the dq, dk it is made from
(bf16: about 2^-9 relative per element, twice: the stored output and the
kernel's bf16 operands).  Those errors do not decay along the sum, so the bar
derived from the arithmetic is, per token t,
    |d - ref| <= tol * max|ref| + 4 u sqrt(sum_{s>=t} sigma_s^2),
    sigma_s^2 = sum_e (q_se dq_se)^2 + (k_se dk_se)^2   (oracle values),
u = 2^-8 for bf16, 2^-20 for fp32; for a per-head decay the sum over b and t
weights token s by the s + 1 suffix sums it enters.  A simulation with
bf16-rounded dq, dk stays near 0.2 of this bar; a dropped <d_final_state,
S_T> term or a sign error in k . dk exceeds it 27 to 240 times.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import TOL, gen_case, rel_err, to_dev

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


def _np(x):
    return x.detach().to("cpu").double().numpy()


def dlog_excess(d, ref, q, k, dq, dk, kind, tol, dtype):
    """max over tokens (per step) or heads (per head) of |d - ref| / bar."""
    u = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -20
    qd, kd = _np(q), _np(k)
    sig2 = ((qd * dq) ** 2).sum(-1) + ((kd * dk) ** 2).sum(-1)  # [B,H,T]
    d = _np(d)
    if kind == 2:
        suf = np.cumsum(sig2[..., ::-1], axis=-1)[..., ::-1]
        bar = tol * np.abs(ref).max(axis=-1, keepdims=True) + 4 * u * np.sqrt(suf)
    else:
        T = sig2.shape[-1]
        w = np.arange(1, T + 1, dtype=np.float64)[None, None, :] ** 2
        bar = tol * np.abs(ref).max() + 4 * u * np.sqrt((sig2 * w).sum(axis=(0, 2)))
    return float(np.max(np.abs(d - ref) / bar))


def check_backward(inp, S0=None, dSf=None, seed=0, tol=None, dy=None):
    dtype = inp["q"].dtype
    tol = tol or TOL[dtype]
    B, H, T, Dk = inp["q"].shape
    Dv = inp["v"].shape[-1]
    if dy is None:
        g = torch.Generator().manual_seed(seed)
        dy = torch.randn(B, H, T, Dv, generator=g).to(dtype)
    d = to_dev(inp)
    dq, dk, dv, dlg, dS0 = la().chunk_backward(d["q"], d["k"], d["v"], dy.cuda(), d["decay_kind"], d["log_g"],
                                               None if S0 is None else S0.cuda(),
                                               None if dSf is None else dSf.cuda())
    torch.cuda.synchronize()
    rq, rk, rv, rlg, rS0, _ = oracle.backward(inp["q"], inp["k"], inp["v"], dy, inp["decay_kind"], inp["log_g"],
                                              False, S0, None, dSf, None)
    errs = {"dq": rel_err(dq, rq), "dk": rel_err(dk, rk), "dv": rel_err(dv, rv), "dS0": rel_err(dS0, rS0)}
    bad = {n: e for n, e in errs.items() if not e <= tol}
    if inp["decay_kind"] != 0:
        errs["dlog/bar"] = dlog_excess(dlg, rlg, inp["q"], inp["k"], rq, rk, inp["decay_kind"], tol, dtype)
        if not errs["dlog/bar"] <= 1.0:
            bad["dlog/bar"] = errs["dlog/bar"]
    else:
        assert dlg is None
    assert not bad, errs
    return errs


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("final", [False, True])
def test_backward_fp32(kind, init, final):
    inp, S0, _ = gen_case(2, 3, 77, 24, 40, dtype=torch.float32, kind=kind, init=init,
                          seed=3000 + kind * 4 + init * 2 + final)
    dSf = torch.randn(2, 3, 24, 40, generator=torch.Generator().manual_seed(31)) if final else None
    check_backward(inp, S0, dSf, seed=kind)


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("final", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_backward_tc(kind, init, final, D):
    inp, S0, _ = gen_case(2, 2, 600, D, D, kind=kind, init=init,
                          seed=3100 + kind * 8 + init * 4 + final * 2 + (D == 128))
    dSf = torch.randn(2, 2, D, D, generator=torch.Generator().manual_seed(37)) if final else None
    check_backward(inp, S0, dSf, seed=7 + kind)


@pytest.mark.parametrize("Dk,Dv", [(16, 128), (128, 32), (64, 16), (32, 64), (48, 80), (112, 96), (96, 48)])
def test_backward_widths(Dk, Dv):
    inp, S0, _ = gen_case(1, 3, 333, Dk, Dv, kind=2, init=True, seed=3200 + Dk + Dv)
    dSf = torch.randn(1, 3, Dk, Dv, generator=torch.Generator().manual_seed(41))
    check_backward(inp, S0, dSf, seed=11)


@pytest.mark.parametrize("kind", [0, 1, 2])
def test_backward_t_segments(kind):
    """Few heads and a long sequence: the three scans run as T-segments
    (a state pass, then the output pass)."""
    inp, S0, _ = gen_case(1, 2, 4096 + 77, 64, 64, kind=kind, init=True, seed=3300 + kind, decay_mean=4.0)
    dSf = torch.randn(1, 2, 64, 64, generator=torch.Generator().manual_seed(43))
    assert la().workspace_size(1, 2, 4096 + 77, 64, 64) > 0  # the plan does segment these sizes
    check_backward(inp, S0, dSf, seed=13)


@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 128), (128, 64), (32, 96)])
def test_backward_t_segments_widths(Dk, Dv):
    """T-segments with square and mixed widths: the dv scan reuses the dk
    scan's state pieces (transposed) when the two plans cut T alike, and
    runs its own state pass otherwise."""
    inp, S0, _ = gen_case(1, 2, 4096 + 77, Dk, Dv, kind=2, init=True, seed=3310 + Dk + Dv, decay_mean=4.0)
    dSf = torch.randn(1, 2, Dk, Dv, generator=torch.Generator().manual_seed(47))
    assert la().workspace_size(1, 2, 4096 + 77, Dk, Dv) > 0
    check_backward(inp, S0, dSf, seed=17)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 2, 129])
def test_backward_short(dtype, T):
    inp, S0, _ = gen_case(1, 2, T, 16, 16, dtype=dtype, kind=2, init=True, seed=3400 + T)
    dSf = torch.randn(1, 2, 16, 16, generator=torch.Generator().manual_seed(47))
    check_backward(inp, S0, dSf, seed=17)


def test_backward_empty_sequence_passes_the_state_gradient():
    B, H, D = 2, 3, 16
    q = torch.zeros(B, H, 0, D, dtype=torch.bfloat16, device="cuda")
    dSf = torch.randn(B, H, D, D, device="cuda")
    lg = torch.full((H,), -0.1, device="cuda")
    dq, dk, dv, dlg, dS0 = la().chunk_backward(q, q, q, q, la().DECAY_PER_HEAD, lg, None, dSf)
    torch.cuda.synchronize()
    assert torch.equal(dS0, dSf)
    assert torch.equal(dlg, torch.zeros_like(lg))


def test_backward_is_deterministic():
    inp, S0, _ = gen_case(1, 2, 700, 64, 64, kind=1, init=True, seed=3500)
    d = to_dev(inp)
    dy = torch.randn(1, 2, 700, 64, device="cuda").to(torch.bfloat16)
    a = la().chunk_backward(d["q"], d["k"], d["v"], dy, 1, d["log_g"], S0.cuda())
    b = la().chunk_backward(d["q"], d["k"], d["v"], dy, 1, d["log_g"], S0.cuda())
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_retention_workload_full():
    """The retention workload (B4 H8 T2048 D64, per-head decay), every head."""
    wl = W.WORKLOADS[2]
    inp = W.forward_inputs(wl)
    g = torch.Generator().manual_seed(wl.seed + 500)
    dy = torch.randn(wl.B, wl.H, wl.T, wl.Dv, generator=g).to(torch.bfloat16)
    check_backward(inp, dy=dy)


def test_backward_gated_workload_sampled_heads():
    """The gated workload (B1 H32 T65536 D128, per-step decay) at full size on
    the GPU; two sampled heads against the oracle."""
    wl = W.WORKLOADS[4]
    inp = W.forward_inputs(wl)
    g = torch.Generator().manual_seed(wl.seed + 500)
    dy = torch.randn(wl.B, wl.H, wl.T, wl.Dv, generator=g).to(torch.bfloat16)
    d = to_dev(inp)
    dq, dk, dv, dlg, dS0 = la().chunk_backward(d["q"], d["k"], d["v"], dy.cuda(), d["decay_kind"], d["log_g"])
    torch.cuda.synchronize()
    for h in (0, 29):
        sl = lambda x: x[:, h:h + 1].contiguous()  # noqa: E731
        rq, rk, rv, rlg, rS0, _ = oracle.backward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(dy), 2,
                                                  sl(inp["log_g"]), False)
        errs = {"dq": rel_err(sl(dq), rq), "dk": rel_err(sl(dk), rk), "dv": rel_err(sl(dv), rv),
                "dS0": rel_err(sl(dS0), rS0),
                "dlog/bar": dlog_excess(sl(dlg), rlg, sl(inp["q"]), sl(inp["k"]), rq, rk, 2, 2e-2, torch.bfloat16)}
        assert max(errs["dq"], errs["dk"], errs["dv"], errs["dS0"]) <= 2e-2 and errs["dlog/bar"] <= 1.0, (h, errs)
