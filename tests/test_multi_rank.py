"""The multi-GPU host path of bench.py on CPU: two gloo ranks.

Each rank times its own batch (weak scaling, no collective on the data
path); the job's time is the maximum over ranks, and the ranks' inputs are
independent batches of the same workload."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads as W
        wl = W.RETENTION.with_sizes(B=1, H=2, T=16)
        # per-rank "time": rank-dependent so the maximum is known
        t = bench.max_over_ranks(1.5 + rank, True, torch.device("cpu"))
        x = W.forward_inputs(wl, seed=bench.rank_seed(wl, rank))["q"].float()
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)  # test-only: compare the ranks' inputs
        out[rank] = (t, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_the_max_and_batches_differ():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == pytest.approx(2.5) and res[1][0] == pytest.approx(2.5)
    assert res[0][1] is False  # the two ranks hold different sequences


def test_single_process_needs_no_collective():
    import bench
    assert bench.max_over_ranks(3.25, False, torch.device("cpu")) == 3.25
    import workloads as W
    assert bench.rank_seed(W.RETENTION, 0) == W.RETENTION.seed


def test_bench_gpus_flag_starts_the_ranks_itself():
    """`bench.py --gpus 2` outside torchrun launches two ranks (gloo standing
    in for NCCL in the timing self-test); rank 0 reports n_gpus = 2 and the
    slowest rank's time."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--cpu-selftest"],
                       capture_output=True, text=True, timeout=240, env=dict(os.environ, OMP_NUM_THREADS="1"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and len(line["per_rank_ms"]) == 2
    assert line["ms_per_step"] == max(line["per_rank_ms"])
    assert line["per_rank_ms"][1] > line["per_rank_ms"][0]  # rank 1 works twice as long


def test_bench_refuses_a_rank_count_that_disagrees_with_gpus():
    import subprocess
    import sys
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--cpu-selftest"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0 and "ranks were launched" in r.stderr
