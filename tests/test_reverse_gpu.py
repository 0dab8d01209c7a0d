"""GPU parity of the reverse scan and the bidirectional encoder (RetNet issue
21, Details: the cumulative EMA's reverse flag and the encoder built from one
forward and one reverse retention) against the float64 oracle, through the C
ABI.  Same bar as the forward: max relative error per (b, h) slice 1e-4 for
fp32 inputs, 2e-2 for bf16 inputs."""
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


def check_reverse(inp, normalize=False, S0=None, z0=None, tol=None, workspace=True):
    tol = tol or TOL[inp["q"].dtype]
    d = to_dev(inp)
    y, S, z = la().chunk_forward(d["q"], d["k"], d["v"], d["decay_kind"], d["log_g"], normalize,
                                 None if S0 is None else S0.cuda(), None if z0 is None else z0.cuda(),
                                 reverse=True, workspace=workspace)
    torch.cuda.synchronize()
    yr, Sr, zr = oracle.reverse(inp["q"], inp["k"], inp["v"], inp["decay_kind"], inp["log_g"], normalize,
                                S0, z0)
    errs = {"y": rel_err(y, yr), "S": rel_err(S, Sr)}
    if normalize:
        errs["z"] = rel_err(z, zr)
    assert all(e <= tol for e in errs.values()), errs
    return errs


def check_bidirectional(inp, normalize=False, out=None, tol=None):
    tol = tol or TOL[inp["q"].dtype]
    d = to_dev(inp)
    y = la().bidirectional(d["q"], d["k"], d["v"], d["decay_kind"], d["log_g"], normalize, out=out)
    torch.cuda.synchronize()
    yr = oracle.bidirectional(inp["q"], inp["k"], inp["v"], inp["decay_kind"], inp["log_g"], normalize)
    err = rel_err(y, yr)
    assert err <= tol, err
    return err


# ---------------------------------------------------------------- reverse scan

@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
@pytest.mark.parametrize("init", [False, True])
def test_reverse_fp32(kind, normalize, init):
    inp, S0, z0 = gen_case(2, 3, 77, 24, 40, dtype=torch.float32, kind=kind, normalize=normalize,
                           init=init, seed=2000 + kind * 4 + normalize * 2 + init)
    check_reverse(inp, normalize, S0, z0)


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_reverse_tc_flags(kind, normalize, init, D):
    inp, S0, z0 = gen_case(2, 2, 600, D, D, kind=kind, normalize=normalize, init=init,
                           seed=2100 + kind * 8 + normalize * 4 + init * 2 + (D == 128))
    check_reverse(inp, normalize, S0, z0)


@pytest.mark.parametrize("Dk", [16, 32, 48, 64, 112, 128])
@pytest.mark.parametrize("Dv", [16, 32, 80, 64, 96, 128])
def test_reverse_tc_widths(Dk, Dv):
    inp, S0, _ = gen_case(1, 2, 300, Dk, Dv, kind=2, init=True, seed=2200 + Dk + Dv)
    check_reverse(inp, False, S0)


@pytest.mark.parametrize("T", [1, 2, 5, 127, 128, 129, 255, 257, 1000])
@pytest.mark.parametrize("normalize", [False, True])
def test_reverse_ragged_lengths(T, normalize):
    # the ragged chunk is the first one the reverse scan visits
    inp, S0, z0 = gen_case(1, 2, T, 64, 64, kind=2, normalize=normalize, init=True, seed=2300 + T)
    check_reverse(inp, normalize, S0, z0)


@pytest.mark.parametrize("split", [1, 2, 4, 8])
def test_reverse_value_split(monkeypatch, split):
    monkeypatch.setenv("LA_DV_SPLIT", str(split))
    inp, S0, z0 = gen_case(1, 2, 700, 128, 128, kind=2, normalize=split % 2 == 0, init=True, seed=2400 + split)
    check_reverse(inp, split % 2 == 0, S0, z0)


@pytest.mark.parametrize("nseg", [2, 3, 5])
@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
def test_reverse_segments(monkeypatch, nseg, kind, normalize):
    monkeypatch.setenv("LA_SEGMENTS", str(nseg))
    inp, S0, z0 = gen_case(1, 2, 1100, 64, 64, kind=kind, normalize=normalize, init=True,
                           seed=2500 + nseg * 8 + kind * 2 + normalize)
    check_reverse(inp, normalize, S0, z0)


@pytest.mark.parametrize("decay_mean", [1.0, -30.0])
@pytest.mark.parametrize("nseg", [1, 4])
@pytest.mark.parametrize("D", [64, 128])
def test_reverse_direct_form(monkeypatch, decay_mean, nseg, D):
    # chunks whose total decay passes the fold limit take the direct form (at
    # D = 128 with segments, in the state pass's one 128-column slice too)
    monkeypatch.setenv("LA_SEGMENTS", str(nseg))
    inp, S0, z0 = gen_case(1, 2, 1000, D, D, kind=2, normalize=True, init=True, seed=2600 + nseg + D,
                           decay_mean=decay_mean)
    if decay_mean < 0:
        inp["log_g"] = torch.full_like(inp["log_g"], decay_mean)
    check_reverse(inp, True, S0, z0)


@pytest.mark.parametrize("nseg", [2, 4])
@pytest.mark.parametrize("normalize", [False, True])
def test_reverse_segments_d128(monkeypatch, nseg, normalize):
    # the reverse scan's state pass as one 128-column slice (the output pass
    # in two 64-column slices)
    monkeypatch.setenv("LA_SEGMENTS", str(nseg))
    inp, S0, z0 = gen_case(1, 2, 1100, 128, 128, kind=2, normalize=normalize, init=True,
                           seed=2700 + nseg * 2 + normalize)
    check_reverse(inp, normalize, S0, z0)


def test_reverse_is_forward_of_flipped_inputs():
    # a property of the definition, checked on the GPU alone: the reverse scan
    # equals the forward scan of the time-reversed sequence, reversed back
    inp, S0, _ = gen_case(2, 2, 384, 64, 64, dtype=torch.float32, kind=2, init=True, seed=2700)
    d = to_dev(inp)
    flip = lambda x: x.flip(2).contiguous()  # noqa: E731
    y1, S1, _ = la().chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"], False, S0.cuda(), None, reverse=True)
    y2, S2, _ = la().chunk_forward(flip(d["q"]), flip(d["k"]), flip(d["v"]), 2, flip(d["log_g"]), False,
                                   S0.cuda(), None)
    torch.cuda.synchronize()
    assert rel_err(y1, flip(y2).cpu().double()) < 1e-5
    assert rel_err(S1, S2.cpu().double()) < 1e-5


def test_reverse_full_length_sampled_heads():
    # the long gated sequence (T = 65536) in the segmented launch configuration,
    # two heads compared with the oracle
    wl = W.GATED
    heads = [0, 31]
    full = W.forward_inputs(wl)
    d = to_dev(full)
    y, S, _ = la().chunk_forward(d["q"], d["k"], d["v"], d["decay_kind"], d["log_g"], reverse=True)
    torch.cuda.synchronize()
    sub = W.forward_inputs(wl, heads=heads)
    yr, Sr, _ = oracle.reverse(sub["q"], sub["k"], sub["v"], sub["decay_kind"], sub["log_g"])
    yy = y.view(-1, wl.T, wl.Dv)[heads][None]
    SS = S.view(-1, wl.Dk, wl.Dv)[heads][None]
    assert rel_err(yy, yr) <= 2e-2 and rel_err(SS, Sr) <= 2e-2


# ---------------------------------------------------------------- bidirectional

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
def test_bidirectional(dtype, kind, normalize):
    inp, _, _ = gen_case(2, 2, 450, 64, 64, dtype=dtype, kind=kind, normalize=normalize,
                         seed=2800 + kind * 2 + normalize + (dtype == torch.bfloat16) * 10)
    check_bidirectional(inp, normalize)


@pytest.mark.parametrize("nseg", [2, 5])
def test_bidirectional_segments(monkeypatch, nseg):
    monkeypatch.setenv("LA_SEGMENTS", str(nseg))
    inp, _, _ = gen_case(1, 2, 1300, 128, 128, kind=2, normalize=True, seed=2900 + nseg)
    check_bidirectional(inp, True)


def test_bidirectional_output_only_16_byte_aligned():
    # the accumulating pass reads and writes through the 16-byte path
    inp, _, _ = gen_case(1, 2, 300, 64, 64, kind=1, seed=2950)
    buf = torch.empty(1 * 2 * 300 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    out = buf[8:].view(1, 2, 300, 64)
    assert out.data_ptr() % 32 == 16
    check_bidirectional(inp, False, out=out)


def test_bidirectional_sums_both_directions():
    # the encoder's output is the sum of the two scans it is made of (fp32:
    # the same kernels, the second adding to what the first wrote)
    inp, _, _ = gen_case(1, 3, 200, 32, 32, dtype=torch.float32, kind=2, seed=2960)
    d = to_dev(inp)
    yb = la().bidirectional(d["q"], d["k"], d["v"], 2, d["log_g"])
    yf, _, _ = la().chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"])
    yr, _, _ = la().chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"], reverse=True)
    torch.cuda.synchronize()
    assert torch.equal(yb, yf + yr)


def test_bidirectional_empty_and_invalid():
    q = torch.zeros(1, 1, 0, 16, dtype=torch.bfloat16, device="cuda")
    assert la().bidirectional(q, q, q).shape == (1, 1, 0, 16)
    x = torch.zeros(1, 1, 8, 24, dtype=torch.bfloat16, device="cuda")  # no kernel for Dk = 24 in bf16
    with pytest.raises(la().LAError) as ei:
        la().bidirectional(x, x, x)
    assert ei.value.status == 2


def test_bidirectional_full_size_sampled_heads():
    # the retention workload's sizes (4 x 8 heads, T = 2048, D = 64, per-head
    # decay), every head on the GPU, three compared with the oracle
    wl = W.RETENTION
    heads = [0, 13, wl.B * wl.H - 1]
    full = W.forward_inputs(wl)
    d = to_dev(full)
    y = la().bidirectional(d["q"], d["k"], d["v"], d["decay_kind"], d["log_g"])
    torch.cuda.synchronize()
    sub = W.forward_inputs(wl, heads=heads)  # each slice keeps its own head's decay
    yr = oracle.bidirectional(sub["q"], sub["k"], sub["v"], sub["decay_kind"], sub["log_g"])
    yy = y.view(-1, wl.T, wl.Dv)[heads][None]
    assert rel_err(yy, yr) <= 2e-2
