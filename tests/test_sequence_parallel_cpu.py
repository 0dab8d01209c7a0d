"""The host logic of the sequence-parallel forward on CPU: gloo ranks, each
holding one span of the sequence, with the three compute steps done by the
float64 oracle in place of the library's kernels (the kernels need a GPU).

What is checked is the part that is not a kernel: which spans a rank folds
(those before it, in order, onto the sequence's initial state), the record
layout of the exchange, that the last rank contributes nothing, and that
every rank's outputs and the last rank's final state are those of one
forward over the whole sequence (RetNet issue 21, the associative EMA
operator)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The compute steps in float64 on the host (test stand-ins)."""
    calls = None

    @staticmethod
    def state(k, v, kind, log_g, normalize, state_out, z_out, log_out):
        import oracle
        OracleOps.calls.append("state")
        _, S, z = oracle.forward(k, k, v, kind, log_g, normalize)
        state_out.copy_(torch.from_numpy(S))
        if normalize:
            z_out.copy_(torch.from_numpy(z))
        T, H = k.shape[2], k.shape[1]
        if kind == 0:
            log_out.zero_()
        elif kind == 1:
            log_out.copy_((log_g.double() * T).expand(log_out.shape))
        else:
            log_out.copy_(log_g.double().sum(-1))

    @staticmethod
    def combine(seg_state, seg_log_g, seg_z, init_state, init_z):
        OracleOps.calls.append(f"combine{seg_state.shape[0]}")
        S = init_state.double().clone() if init_state is not None else torch.zeros(seg_state.shape[1:],
                                                                                   dtype=torch.float64)
        z = None
        if seg_z is not None:
            z = init_z.double().clone() if init_z is not None else torch.zeros(seg_z.shape[1:], dtype=torch.float64)
        for j in range(seg_state.shape[0]):
            e = torch.exp(seg_log_g[j].double())
            S = e[..., None, None] * S + seg_state[j].double()
            if z is not None:
                z = e[..., None] * z + seg_z[j].double()
        return S.float(), (z.float() if z is not None else None)

    @staticmethod
    def forward(q, k, v, kind, log_g, normalize, init_state, init_z, out):
        import oracle
        OracleOps.calls.append("forward")
        y, S, z = oracle.forward(q, k, v, kind, log_g, normalize, init_state, init_z)
        return torch.from_numpy(y), torch.from_numpy(S), (torch.from_numpy(z) if normalize else None)


def _case(kind, normalize, T, seed):
    sys_path = os.path.join(ROOT, "tests")
    import sys
    if sys_path not in sys.path:
        sys.path.insert(0, sys_path)
    from parity import gen_case
    return gen_case(1, 2, T, 8, 12, dtype=torch.float32, kind=kind, normalize=normalize, init=True, seed=seed)


def _worker(rank, world, port, cuts, kind, normalize, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from retention_scan_b200 import sequence_parallel as sp
        inp, S0, z0 = _case(kind, normalize, cuts[-1], 900 + kind)
        a, b = cuts[rank], cuts[rank + 1]
        q, k, v = (inp[n][:, :, a:b].contiguous() for n in ("q", "k", "v"))
        lg = inp["log_g"]
        if kind == 2:
            lg = lg[:, :, a:b].contiguous()
        OracleOps.calls = []

        def gather(outs, x):
            dist.all_gather(outs, x)

        y, S, z = sp.span_forward_with(rank, world, gather, OracleOps, q, k, v, kind, lg, normalize, S0,
                                       z0 if normalize else None)
        out[rank] = (y.numpy(), S.numpy(), None if z is None else z.numpy(), list(OracleOps.calls))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("kind,normalize", [(2, False), (2, True), (1, True), (0, False)])
def test_three_gloo_ranks_match_one_forward(kind, normalize):
    import oracle
    oracle.build()
    cuts = [0, 37, 38, 90]
    world = len(cuts) - 1
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, cuts, kind, normalize, out), nprocs=world, join=True)
        res = dict(out)
    inp, S0, z0 = _case(kind, normalize, cuts[-1], 900 + kind)
    yr, Sr, zr = oracle.forward(inp["q"], inp["k"], inp["v"], kind, inp["log_g"], normalize, S0,
                                z0 if normalize else None)
    y = np.concatenate([res[r][0] for r in range(world)], axis=2)
    scale = np.abs(yr).max()
    assert np.abs(y - yr).max() <= 1e-5 * scale
    assert np.abs(res[world - 1][1] - Sr).max() <= 1e-5 * np.abs(Sr).max()
    if normalize:
        assert np.abs(res[world - 1][2] - zr).max() <= 1e-5 * np.abs(zr).max()
    # rank 0 folds nothing, rank r folds the r spans before it; the last
    # rank computes no state of its own
    assert res[0][3] == ["state", "forward"]
    assert res[1][3] == ["state", "combine1", "forward"]
    assert res[2][3] == ["combine2", "forward"]


def test_record_layout_is_16_byte_aligned():
    from retention_scan_b200 import sequence_parallel as sp
    for B, H, Dk, Dv in [(1, 1, 1, 1), (3, 5, 7, 9), (1, 32, 128, 128)]:
        s, z, lg, size = sp.record_layout(B, H, Dk, Dv)
        assert s == 0 and z % 4 == 0 and lg % 4 == 0 and size % 4 == 0
        assert z >= B * H * Dk * Dv and lg - z >= B * H * Dk and size - lg >= B * H


def test_binding_checks_shapes_before_any_call():
    """The binding rejects mismatched shapes and dtypes on the host, before
    it touches the library (CPU tensors: a call would need a device)."""
    import retention_scan_b200 as la
    from retention_scan_b200 import sequence_parallel as sp
    S = torch.zeros(2, 1, 2, 4, 4)
    with pytest.raises(ValueError):
        la.state_combine(S, torch.zeros(2, 1, 3))            # log totals of another shape
    with pytest.raises(TypeError):
        la.state_combine(S, torch.zeros(2, 1, 2, dtype=torch.float64))
    with pytest.raises(ValueError):
        la.state_combine(S, torch.zeros(2, 1, 2), torch.zeros(2, 1, 2, 5))   # key sums of another width
    with pytest.raises(ValueError):
        la.state_combine(S.transpose(3, 4), torch.zeros(2, 1, 2))           # spans not contiguous
    k = torch.zeros(1, 2, 8, 4)
    with pytest.raises(ValueError):
        la.chunk_state(k, torch.zeros(1, 2, 7, 4))          # v of another length
    with pytest.raises(ValueError):
        la.chunk_state(k, torch.zeros(1, 2, 8, 4), la.DECAY_PER_STEP, torch.zeros(1, 2, 9))
    with pytest.raises(ValueError):
        sp.span_forward_with(0, 1, None, None, k, k, k, normalize=True, init_state=torch.zeros(1, 2, 4, 4))
