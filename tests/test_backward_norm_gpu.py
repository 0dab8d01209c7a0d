"""GPU parity of the normalised forward's backward (la_chunk_backward_norm_ws)
against the float64 oracle's chain rule, through the C ABI.  Bars as in
test_backward_gpu.py: the forward's relative bar for dq, dk, dv, d_init_state
and d_init_z; for d log g the relative bar plus the rounding that the bf16 dq
and dk carry along the undecayed suffix sum.

dq_t = S_t dn_t + dden_t z_t and dk_t = dS_t v_t + dz_t are differences of
comparable terms.  For Dv + 1 <= 128 the library forms each with one scan
whose scores hold both terms (fp32), and the bar above holds.  For Dv = 128
the two terms come from two scans: the second adds its fp32 result into the
first's rounded output, and each scan rounds its own scores and state copy
to bf16 before the terms meet.  Those roundings are relative to each term,
not to their difference, so the bar adds 4 u (|first| + |second|)
elementwise (u = 2^-8 for bf16, 2^-20 for fp32), the terms' sizes taken
from the float64 oracle's scans."""
import pytest
import torch

import oracle
from norm_bar import split_err, term_sizes
from parity import TOL, gen_case, rel_err, to_dev
from test_backward_gpu import dlog_excess

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


def check(inp, S0, z0, dSf, dzf, seed):
    dtype = inp["q"].dtype
    tol = TOL[dtype]
    B, H, T, Dk = inp["q"].shape
    Dv = inp["v"].shape[-1]
    dy = torch.randn(B, H, T, Dv, generator=torch.Generator().manual_seed(seed)).to(dtype)
    d = to_dev(inp)
    c = lambda x: None if x is None else x.cuda()  # noqa: E731
    dq, dk, dv, dlg, dS0, dz0 = la().chunk_backward_normalized(d["q"], d["k"], d["v"], dy.cuda(), d["decay_kind"],
                                                               d["log_g"], c(S0), c(z0), c(dSf), c(dzf))
    torch.cuda.synchronize()
    rq, rk, rv, rlg, rS0, rz0 = oracle.backward(inp["q"], inp["k"], inp["v"], dy, inp["decay_kind"], inp["log_g"],
                                                True, S0, z0, dSf, dzf)
    errs = {"dq": rel_err(dq, rq), "dk": rel_err(dk, rk), "dv": rel_err(dv, rv), "dS0": rel_err(dS0, rS0),
            "dz0": rel_err(dz0, rz0)}
    bad = {n: e for n, e in errs.items() if not e <= tol}
    if Dv + 1 > 128:  # two scans per gradient: the derived bar for dq and dk
        u = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -20
        tq, tk = term_sizes(inp, S0, z0, dSf, dzf, dy)
        errs["dq/bar"], errs["dk/bar"] = split_err(dq, rq, tq, tol, u), split_err(dk, rk, tk, tol, u)
        bad.pop("dq", None)
        bad.pop("dk", None)
        bad.update({n: errs[n] for n in ("dq/bar", "dk/bar") if not errs[n] <= 1.0})
    if inp["decay_kind"] != 0:
        errs["dlog/bar"] = dlog_excess(dlg, rlg, inp["q"], inp["k"], rq, rk, inp["decay_kind"], tol, dtype)
        if not errs["dlog/bar"] <= 1.0:
            bad["dlog/bar"] = errs["dlog/bar"]
    assert not bad, errs
    return errs


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("final", [False, True])
def test_backward_norm_fp32(kind, init, final):
    inp, S0, z0 = gen_case(2, 3, 77, 24, 40, dtype=torch.float32, kind=kind, normalize=True, init=init,
                           seed=6000 + kind * 4 + init * 2 + final)
    g = torch.Generator().manual_seed(61)
    dSf = torch.randn(2, 3, 24, 40, generator=g) * 0.1 if final else None
    dzf = torch.randn(2, 3, 24, generator=g) * 0.1 if final else None
    check(inp, S0, z0, dSf, dzf, seed=kind)


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("final", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_backward_norm_tc(kind, init, final, D):
    inp, S0, z0 = gen_case(2, 2, 600, D, D, kind=kind, normalize=True, init=init,
                           seed=6100 + kind * 8 + init * 4 + final * 2 + (D == 128))
    g = torch.Generator().manual_seed(67)
    dSf = torch.randn(2, 2, D, D, generator=g) * 0.1 if final else None
    dzf = torch.randn(2, 2, D, generator=g) * 0.1 if final else None
    check(inp, S0, z0, dSf, dzf, seed=9 + kind)


@pytest.mark.parametrize("Dk,Dv", [(16, 128), (128, 32), (64, 16), (80, 48), (48, 112)])
def test_backward_norm_widths(Dk, Dv):
    inp, S0, z0 = gen_case(1, 3, 333, Dk, Dv, kind=2, normalize=True, init=True, seed=6200 + Dk + Dv)
    check(inp, S0, z0, None, torch.randn(1, 3, Dk) * 0.1, seed=19)


@pytest.mark.parametrize("kind", [0, 2])
def test_backward_norm_t_segments(kind):
    inp, S0, z0 = gen_case(1, 2, 4096 + 77, 64, 64, kind=kind, normalize=True, init=True, seed=6300 + kind,
                           decay_mean=4.0)
    check(inp, S0, z0, torch.randn(1, 2, 64, 64) * 0.1, torch.randn(1, 2, 64) * 0.1, seed=23)
