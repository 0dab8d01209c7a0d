"""GPU parity of the span states and their fold (la_chunk_state_ws,
la_state_combine) and of the sequence-parallel forward built on them,
through the C ABI.

A span's state is the recurrence's final state from zero (the oracle's
forward started from zero); its log total is the float64 sum of its log
decays.  The fold of consecutive spans' states onto an initial state must be
the final state of the oracle's forward over the concatenated sequence (RetNet
issue 21, the associative EMA operator), and each span's forward from the
folded state must be that sequence's outputs on the span.  Bar as the
forward: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs; the log totals to fp32
rounding of their sums (1e-5 of the largest)."""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle
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


def log_total(inp, B, H, T):
    kind, lg = inp["decay_kind"], inp["log_g"]
    if kind == 0:
        return np.zeros((B, H))
    lg = lg.double().numpy()
    if kind == 1:
        return np.broadcast_to(lg * T, (B, H)).copy()
    return lg.sum(-1)


def log_err(x, ref):
    ref = np.asarray(ref, np.float64)
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    return float(np.max(np.abs(x.detach().cpu().double().numpy() - ref))) / scale


def slice_t(inp, t0, t1):
    out = dict(inp)
    for key in ("q", "k", "v"):
        out[key] = inp[key][:, :, t0:t1].contiguous()
    if inp["decay_kind"] == 2:
        out["log_g"] = inp["log_g"][:, :, t0:t1].contiguous()
    return out


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
@pytest.mark.parametrize("T", [1, 100, 128, 777])
def test_span_state_from_zero(dtype, kind, normalize, T):
    B, H, Dk, Dv = 2, 3, 64, 32
    inp, _, _ = gen_case(B, H, T, Dk, Dv, dtype=dtype, kind=kind, normalize=normalize,
                         seed=7000 + T + 10 * kind + normalize)
    d = to_dev(inp)
    S, z, L = la().chunk_state(d["k"], d["v"], kind, d["log_g"], normalize)
    torch.cuda.synchronize()
    _, Sr, zr = oracle.forward(inp["k"], inp["k"], inp["v"], kind, inp["log_g"], normalize)
    errs = {"S": rel_err(S, Sr), "L": log_err(L, log_total(inp, B, H, T))}
    if normalize:
        errs["z"] = rel_err(z, zr)
    tol = TOL[dtype]
    assert errs["S"] <= tol and errs.get("z", 0.0) <= tol and errs["L"] <= 1e-5, errs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_span_state_bench_shape(dtype):
    """One head group of the gated long-sequence shape (Dk = Dv = 128), long
    enough that the state pass runs in several pieces."""
    B, H, T, D = 1, 4, 4096 + 50, 128
    inp, _, _ = gen_case(B, H, T, D, D, dtype=dtype, kind=2, seed=7100, decay_mean=4.0)
    d = to_dev(inp)
    S, _, L = la().chunk_state(d["k"], d["v"], 2, d["log_g"])
    torch.cuda.synchronize()
    _, Sr, _ = oracle.forward(inp["k"], inp["k"], inp["v"], 2, inp["log_g"])
    assert rel_err(S, Sr) <= TOL[dtype]
    assert log_err(L, log_total(inp, B, H, T)) <= 1e-5


def test_span_state_empty():
    B, H, Dk, Dv = 2, 2, 16, 16
    k = torch.zeros(B, H, 0, Dk, dtype=torch.bfloat16, device="cuda")
    S, z, L = la().chunk_state(k, k[..., :Dv], 0, None, True)
    torch.cuda.synchronize()
    assert not S.any() and not z.any() and not L.any()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("kind", [1, 2])
@pytest.mark.parametrize("normalize", [False, True])
def test_fold_of_spans_is_the_concatenated_forward(dtype, kind, normalize):
    """Ragged spans' states folded onto an initial state equal the final
    state of one forward over the whole sequence from that state."""
    B, H, Dk, Dv = 2, 2, 32, 48
    cuts = [0, 150, 151, 400, 640, 1001]
    T = cuts[-1]
    inp, S0, z0 = gen_case(B, H, T, Dk, Dv, dtype=dtype, kind=kind, normalize=normalize, init=True,
                           seed=7200 + kind + 2 * normalize)
    d = to_dev(inp)
    parts = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        s = slice_t(d, a, b)
        parts.append(la().chunk_state(s["k"], s["v"], kind, s["log_g"], normalize))
    segS = torch.stack([p[0] for p in parts])
    segL = torch.stack([p[2] for p in parts])
    segz = torch.stack([p[1] for p in parts]) if normalize else None
    S, z, L = la().state_combine(segS, segL, segz, S0.cuda(), z0.cuda() if normalize else None)
    torch.cuda.synchronize()
    _, Sr, zr = oracle.forward(inp["q"], inp["k"], inp["v"], kind, inp["log_g"], normalize, S0,
                               z0 if normalize else None)
    errs = {"S": rel_err(S, Sr), "L": log_err(L, log_total(inp, B, H, T))}
    if normalize:
        errs["z"] = rel_err(z, zr)
    tol = TOL[dtype]
    assert errs["S"] <= tol and errs.get("z", 0.0) <= tol and errs["L"] <= 1e-5, errs


def test_fold_of_nothing_copies_the_initial_state():
    B, H, Dk, Dv = 1, 3, 16, 32
    S0 = torch.randn(B, H, Dk, Dv, device="cuda")
    z0 = torch.rand(B, H, Dk, device="cuda")
    empty = torch.empty(0, B, H, Dk, Dv, device="cuda")
    S, z, L = la().state_combine(empty, torch.empty(0, B, H, device="cuda"), torch.empty(0, B, H, Dk, device="cuda"),
                                 S0, z0)
    S1, _, _ = la().state_combine(empty, torch.empty(0, B, H, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(S, S0) and torch.equal(z, z0) and not L.any() and not S1.any()


def test_fold_in_place_and_strided_records():
    """Spans as strided views of one record buffer (the exchange's layout)
    and the output written over the initial state."""
    from retention_scan_b200 import sequence_parallel as sp
    B, H, Dk, Dv, n = 2, 2, 16, 16, 3
    size = sp.record_layout(B, H, Dk, Dv)[3]
    g = torch.Generator().manual_seed(7300)
    buf = torch.randn(n, size, generator=g).cuda()
    S, z, lg = sp._views(buf, B, H, Dk, Dv)
    lg.copy_(-torch.rand(n, B, H, generator=g).cuda())
    S0 = torch.randn(B, H, Dk, Dv, generator=g).cuda()
    z0 = torch.rand(B, H, Dk, generator=g).cuda()
    ref_S, ref_z = S0.double().clone(), z0.double().clone()
    for j in range(n):  # the fold, in float64
        e = torch.exp(lg[j].double())
        ref_S = e[..., None, None] * ref_S + S[j].double()
        ref_z = e[..., None] * ref_z + z[j].double()
    out_S, out_z, _ = la().state_combine(S, lg, z, S0, z0, state_out=S0, z_out=z0)
    torch.cuda.synchronize()
    assert out_S.data_ptr() == S0.data_ptr()
    # fp32 exponentials and three fused multiply-adds per element
    assert rel_err(out_S, ref_S.cpu()) <= 2e-6 and rel_err(out_z, ref_z.cpu()) <= 2e-6


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("normalize", [False, True])
def test_span_forward_ranks_emulated_in_one_process(dtype, normalize):
    """The sequence-parallel forward's library path for four ranks, run one
    after another in one process: each rank's records come from the library,
    the exchange is a copy of all ranks' records (no rank waits on another)."""
    from retention_scan_b200 import sequence_parallel as sp
    B, H, Dk, Dv = 1, 4, 64, 64
    cuts = [0, 300, 640, 641, 1200]
    R, T = len(cuts) - 1, cuts[-1]
    inp, S0, z0 = gen_case(B, H, T, Dk, Dv, dtype=dtype, kind=2, normalize=normalize, init=True,
                           seed=7400 + normalize)
    d = to_dev(inp)
    spans = [slice_t(d, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    size = sp.record_layout(B, H, Dk, Dv)[3]
    records = torch.zeros(R, size, device="cuda")
    for r in range(R - 1):
        S, z, lg = sp._views(records[r:r + 1], B, H, Dk, Dv)
        sp.LibraryOps.state(spans[r]["k"], spans[r]["v"], 2, spans[r]["log_g"], normalize, S[0],
                            z[0] if normalize else None, lg[0])

    def gather(outs, x):
        for o, rec in zip(outs, records):
            o.copy_(rec)

    ys, fin = [], None
    for r in range(R):
        s = spans[r]
        y, Sf, zf = sp.span_forward_with(r, R, gather, sp.LibraryOps, s["q"], s["k"], s["v"], 2, s["log_g"],
                                         normalize, S0.cuda(), z0.cuda() if normalize else None)
        ys.append(y)
        fin = (Sf, zf)
    torch.cuda.synchronize()
    yr, Sr, zr = oracle.forward(inp["q"], inp["k"], inp["v"], 2, inp["log_g"], normalize, S0,
                                z0 if normalize else None)
    errs = {"y": rel_err(torch.cat(ys, 2), yr), "S": rel_err(fin[0], Sr)}
    if normalize:
        errs["z"] = rel_err(fin[1], zr)
    assert max(errs.values()) <= TOL[dtype], errs


def test_span_forward_one_rank_nccl_group():
    """The public call over a real one-rank NCCL group equals the plain
    forward."""
    import torch.distributed as dist
    from retention_scan_b200 import sequence_parallel as sp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0), timeout=datetime.timedelta(seconds=60))
    try:
        inp, S0, _ = gen_case(1, 2, 333, 32, 32, dtype=torch.bfloat16, kind=2, init=True, seed=7500)
        d = to_dev(inp)
        y, S, _ = sp.span_forward(d["q"], d["k"], d["v"], 2, d["log_g"], False, S0.cuda())
        y2, S2, _ = la().chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"], False, S0.cuda())
        torch.cuda.synchronize()
        assert torch.equal(y, y2) and torch.equal(S, S2)
    finally:
        dist.destroy_process_group()
