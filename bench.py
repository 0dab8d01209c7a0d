"""Benchmark of the causal-linear-attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..7] [--impl ours|reference]
                    [--direction forward|reverse|bidirectional|backward]

One step is one pass of the hot path over one batch of the workload:

  config 4 (the headline of the default run): gated per-step decay,
      B=1, H=32, T=65536, D=128 -> one la_chunk_forward call (the largest
      single-GPU workload)
  config 1: plain linear attention, fp32, B=1, H=1, T=64, D=16
  config 2: retention, per-head gamma_h = 1 - 2^(-5-h), bf16,
      B=4, H=8, T=2048, Dk=Dv=64
  config 3: normalised, elu+1 feature map, carried state, B=8, H=16, T=4096, D=128
  config 5: decode, B=256, H=32, D=128, normalised, 1024 la_decode_step calls
  config 6: the RWKV-4 WKV recurrence, B=8, T=4096, C=2048, bf16 -> one
      la_wkv4_forward call (tokens = B*T; a different recurrence)
  config 7: RetNet issue 21's cumulative EMA (values, factors), B=8, T=4096,
      C=2048, bf16 -> one la_ema_scan call (tokens = B*T)

--direction reverse times the anti-causal scan (la_chunk_reverse_ws) on the
same inputs; --direction bidirectional the encoder form (forward scan, then
the reverse scan adding to its output; no carried state); --direction
backward the gradients of the forward (la_chunk_backward_ws, or
la_chunk_backward_norm_ws for the normalised workload: dq, dk, dv, the
log-decay gradient and, with a carried state, the initial state's and key
sum's) for a seeded upstream gradient dy.  Configs 1-4; config 7 takes
forward or reverse (la_ema_scan's reverse flag).

Without --config the run times config 4 for the JSON line's headline
fields and adds a "configs" record with the same measurement of configs 3
(normalised, T=4096), 5 (decode, per token) and 2 (retention, T=2048), each
with its own roofline, clocks, e2e and cpu_baseline.

Timing: W untimed warm-up steps, then untimed steps until the GPU has run
the step for at least half a second (its clocks leave their idle state:
short runs otherwise time the ramp), then K steps, each bracketed by CUDA
events on the launching stream; the L2 cache (126 MB) is flushed by writing
a 512 MB buffer before every step whose inputs fit in L2, outside the events.
A barrier and a device synchronisation bracket the timed region; the time is
the maximum over ranks; ms_per_step is its mean, and the median, minimum and
maximum of the per-step times are reported beside it.  `--gpus N` without
torchrun's environment starts N local ranks itself (torch.distributed.run);
every rank runs the same per-GPU workload (weak scaling, no collective on
the data path).

Extra keys: roofline (dominant kernel, algorithmic bytes / event time against
the measured HBM copy bandwidth), e2e (the same metric through the public API
with pinned host buffers and the host<->device copies inside the timed
region), clocks (nvidia-smi sampled during the timed region), cpu_baseline
(the float64 oracle on the host cores, a bounded sample, rank 0 at N=1).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "linear-attn forward tokens/s (B·H·T/s) and % of roofline (tensor TFLOP/s or HBM GB/s)"


def metric_for(direction):
    return METRIC if direction == "forward" else METRIC.replace("forward", direction)
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 512 * 1024 * 1024


# ---------------------------------------------------------------- workload accounting

def algorithmic_bytes(wl, cfg, direction="forward"):
    """Bytes the hot path must move once: inputs read, outputs written, state
    in/out (fp32), decays; per launch of the dominant kernel.  The
    bidirectional form has no carried state; its minimum is one read of the
    inputs and one write of the output, although its two scans read the
    inputs twice (and the output once more)."""
    es = 4 if wl.dtype == "f32" else 2
    if cfg == 5:
        per_bh = 2 * 4 * wl.Dk * wl.Dv + 2 * 4 * wl.Dk + (2 * wl.Dk + wl.Dv) * es + wl.Dv * es
        return wl.B * wl.H * per_bh  # per decode call
    BH, T = wl.B * wl.H, wl.T
    b = BH * T * ((2 * wl.Dk + wl.Dv) * es + wl.Dv * es)
    if wl.decay == "per_step":
        b += BH * T * 4
    if direction == "bidirectional":
        return b
    if direction == "backward":
        # read q, k, v, dy; write dq, dk, dv; the log decay read and its gradient written
        b = BH * T * (2 * wl.Dk + 2 * wl.Dv) * es + BH * T * (2 * wl.Dk + wl.Dv) * es
        if wl.decay == "per_step":
            b += BH * T * 8
        return b
    b += BH * wl.Dk * wl.Dv * 4  # final state written
    if wl.prefix_T:
        b += BH * wl.Dk * wl.Dv * 4 + 2 * BH * wl.Dk * 4  # initial state, key sums in and out
    return b


def algorithmic_flops(wl, cfg, direction="forward"):
    n = wl.B * wl.H * (1 if cfg == 5 else wl.T)
    return 4 * wl.Dk * wl.Dv * n * {"bidirectional": 2, "backward": 3}.get(direction, 1)


def tokens_per_step(wl, cfg):
    return wl.B * wl.H * (wl.steps if cfg == 5 else wl.T)


def kernel_source_sha(files):
    """Hash of the kernel source files (names under csrc/, and include/la.h)
    that a measured kernel is built from."""
    h = hashlib.sha256()
    for f in sorted(files):
        path = os.path.join(ROOT, "include", f) if f == "la.h" else os.path.join(ROOT, "retention_scan_b200", "csrc", f)
        with open(path, "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload_name):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, if it was taken on the kernel's current sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(workload_name)
        if not rec or rec.get("kernel_sha") != kernel_source_sha(rec["sources"]):
            return None
    except (OSError, ValueError, KeyError):
        return None
    return rec.get("bytes_per_launch")


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 100 ms; keeps (wall time, row) pairs."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = bus_id.lower()
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        mine = [r for (t, r) in self.rows if r and r[0].lower().endswith(self.bus_id[-12:])]
        window = [r for (t, r) in self.rows if t0 - 0.15 <= t <= t1 + 0.15
                  and r and r[0].lower().endswith(self.bus_id[-12:])]
        use = window or mine[-5:]
        if not use:
            return None

        def num(x):
            try:
                return float(x.split()[0])
            except (ValueError, IndexError):
                return float("nan")
        sm = [num(r[1]) for r in use if len(r) > 1]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in use for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(num(r[2]) for r in use if len(r) > 2),
                "reasons": reasons, "samples": len(use), "in_window": bool(window)}


def bus_id_of(device):
    p = torch.cuda.get_device_properties(device)
    try:
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except AttributeError:
        return ""


# ---------------------------------------------------------------- our arm

class Job:
    """Device-resident inputs and the step function of one workload."""

    def __init__(self, cfg, device, wl=None, rank=0, direction="forward", prologue=False):
        import retention_scan_b200 as la
        self.la = la
        self.cfg = cfg
        self.direction = direction
        self.wl = wl = wl or W.WORKLOADS[cfg]
        self.dev = device
        # prologue: q, k handed over raw and the feature map applied inside
        # the forward kernel (la_chunk_forward_pro_ws) instead of by the caller
        self.prologue = prologue and wl.feature_map == "elu1"
        self.fmap = la.FEATURE_ELU1 if self.prologue else la.FEATURE_NONE
        if cfg == 5:
            S0, z0 = W.decode_initial_state(wl)
            self.S0, self.z0 = S0.to(device), z0.to(device)
            self.S, self.z = self.S0.clone(), self.z0.clone()
            self.q, self.k, self.v = W.decode_pool_device(wl, wl.steps, device)
            self.log_g = W.per_head_log_gamma(wl.H).to(device)
            self.out = torch.empty(wl.B, wl.H, wl.Dv, dtype=wl.torch_dtype, device=device)
            return
        inp = W.forward_inputs(wl.with_sizes(feature_map=None) if self.prologue else wl, seed=rank_seed(wl, rank))
        self.host = inp
        self.q, self.k, self.v = (inp[n].to(device) for n in ("q", "k", "v"))
        self.kind = inp["decay_kind"]
        self.log_g = inp["log_g"].to(device) if inp["log_g"] is not None else None
        self.out = torch.empty(wl.B, wl.H, wl.T, wl.Dv, dtype=wl.torch_dtype, device=device)
        self.S = torch.empty(wl.B, wl.H, wl.Dk, wl.Dv, dtype=torch.float32, device=device)
        self.z = torch.empty(wl.B, wl.H, wl.Dk, dtype=torch.float32, device=device) if wl.normalize else None
        self.S0 = self.z0 = None
        # launches per forward: a state pass precedes the output pass when the
        # library cuts the sequences into T-segments (it asks for a workspace)
        self.fwd_launches = 2 if (wl.dtype != "f32" and la.workspace_size(
            wl.B, wl.H, wl.T, wl.Dk, wl.Dv, wl.torch_dtype, wl.normalize) > 0) else 1
        if direction == "bidirectional":
            self.fwd_launches *= 2  # a forward and a reverse scan
        if direction == "backward":
            g = torch.Generator(device=device).manual_seed(wl.seed + 500 + 7919 * rank)
            self.dy = torch.randn(wl.B, wl.H, wl.T, wl.Dv, generator=g, device=device).to(wl.torch_dtype)
            self.grads = (torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v),
                          torch.empty_like(self.log_g) if self.log_g is not None else None,
                          torch.empty(wl.B, wl.H, wl.Dk, wl.Dv, dtype=torch.float32, device=device))
            if wl.normalize:
                nb = int(la.lib().la_chunk_backward_norm_workspace_size(wl.B, wl.H, wl.T, wl.Dk, wl.Dv, 1,
                                                                         self.kind))
            else:
                nb = la.backward_workspace_size(wl.B, wl.H, wl.T, wl.Dk, wl.Dv, wl.torch_dtype, self.kind)
            self.bws = torch.empty(nb, dtype=torch.uint8, device=device)
            self.fwd_launches = backward_launches(la, wl, self.kind, wl.prefix_T > 0)
        if wl.prefix_T and direction != "bidirectional":
            # carried state of the workload: the library's own forward over the seeded prefix
            pre = W.prefix_inputs(wl.with_sizes(feature_map=None) if self.prologue else wl)
            _, self.S0, self.z0 = la.chunk_forward(pre["q"].to(device), pre["k"].to(device),
                                                   pre["v"].to(device), pre["decay_kind"], None, True,
                                                   feature_map=self.fmap)

    def step(self):
        la, wl = self.la, self.wl
        if self.cfg == 5:
            for t in range(wl.steps):
                la.decode_step(self.q[t], self.k[t], self.v[t], self.S, self.z, 1, self.log_g, True,
                               out=self.out)
            return wl.steps
        if self.direction == "bidirectional":
            la.bidirectional(self.q, self.k, self.v, self.kind, self.log_g, wl.normalize, out=self.out)
        elif self.direction == "backward" and wl.normalize:
            la.chunk_backward_normalized(self.q, self.k, self.v, self.dy, self.kind, self.log_g, self.S0, self.z0,
                                         workspace=self.bws)
        elif self.direction == "backward":
            la.chunk_backward(self.q, self.k, self.v, self.dy, self.kind, self.log_g, self.S0, None,
                              workspace=self.bws, out=self.grads)
        else:
            la.chunk_forward(self.q, self.k, self.v, self.kind, self.log_g, wl.normalize, self.S0, self.z0,
                             out=self.out, final_state=self.S, final_z=self.z,
                             reverse=self.direction == "reverse", feature_map=self.fmap)
        return self.fwd_launches

    def caller_mapped_step(self):
        """The step as a caller without the prologue runs it: elu + 1 on q and
        k by a torch pass (fp32, stored as bf16), then the forward on them."""
        la, wl = self.la, self.wl
        phi = lambda x: (torch.nn.functional.elu(x.float()) + 1.0).to(x.dtype)  # noqa: E731
        la.chunk_forward(phi(self.q), phi(self.k), self.v, self.kind, self.log_g, wl.normalize, self.S0, self.z0,
                         out=self.out, final_state=self.S, final_z=self.z)

    E2E_DECODE_TOKENS = 64

    def e2e_step(self, pinned, stream):
        """Public API with host buffers: copy this step's inputs in, run, read
        the result back.  Returns the tokens processed."""
        la, wl = self.la, self.wl
        if self.cfg == 5:
            for t in range(self.E2E_DECODE_TOKENS):
                q = pinned["q"][t].to(self.dev, non_blocking=True)
                k = pinned["k"][t].to(self.dev, non_blocking=True)
                v = pinned["v"][t].to(self.dev, non_blocking=True)
                y = la.decode_step(q, k, v, self.S, self.z, 1, self.log_g, True, out=self.out)
                pinned["y"][t].copy_(y, non_blocking=True)
            return wl.B * wl.H * self.E2E_DECODE_TOKENS
        q, k, v = (pinned[n].to(self.dev, non_blocking=True) for n in ("q", "k", "v"))
        lg = pinned["log_g"].to(self.dev, non_blocking=True) if pinned.get("log_g") is not None else None
        if self.direction == "bidirectional":
            y = la.bidirectional(q, k, v, self.kind, lg, wl.normalize, out=self.out)
            pinned["y"].copy_(y, non_blocking=True)
            return tokens_per_step(wl, self.cfg)
        if self.direction == "backward":
            dy = pinned["dy"].to(self.dev, non_blocking=True)
            if wl.normalize:
                dq, dk, dv, dlg, _, _ = la.chunk_backward_normalized(q, k, v, dy, self.kind, lg, self.S0, self.z0,
                                                                     workspace=self.bws)
            else:
                dq, dk, dv, dlg, _ = la.chunk_backward(q, k, v, dy, self.kind, lg, self.S0, None,
                                                       workspace=self.bws, out=self.grads)
            for n, t in (("dq", dq), ("dk", dk), ("dv", dv), ("dlog", dlg)):
                if t is not None:
                    pinned[n].copy_(t, non_blocking=True)
            return tokens_per_step(wl, self.cfg)
        y, S, _ = la.chunk_forward(q, k, v, self.kind, lg, wl.normalize, self.S0, self.z0,
                                   out=self.out, final_state=self.S, final_z=self.z,
                                   reverse=self.direction == "reverse", feature_map=self.fmap)
        pinned["y"].copy_(y, non_blocking=True)
        pinned["S"].copy_(S, non_blocking=True)
        return tokens_per_step(wl, self.cfg)

    def make_pinned(self):
        wl = self.wl
        if self.cfg == 5:
            n_tok = self.E2E_DECODE_TOKENS
            p = {n: getattr(self, n)[:n_tok].cpu().pin_memory() for n in ("q", "k", "v")}
            p["y"] = torch.empty(n_tok, wl.B, wl.H, wl.Dv, dtype=wl.torch_dtype).pin_memory()
            h2d = sum(p[n].numel() * p[n].element_size() for n in ("q", "k", "v"))
            d2h = p["y"].numel() * p["y"].element_size()
            return p, h2d, d2h
        p = {n: self.host[n].pin_memory() for n in ("q", "k", "v")}
        p["log_g"] = self.host["log_g"].pin_memory() if self.host["log_g"] is not None else None
        p["y"] = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        p["S"] = torch.empty(self.S.shape, dtype=torch.float32).pin_memory()
        if self.direction == "backward":
            p["dy"] = self.dy.cpu().pin_memory()
            for n, t in zip(("dq", "dk", "dv", "dlog"), self.grads[:4]):
                if t is not None:
                    p[n] = torch.empty(t.shape, dtype=t.dtype).pin_memory()
            h2d = sum(p[n].numel() * p[n].element_size() for n in ("q", "k", "v", "log_g", "dy")
                      if p[n] is not None)
            d2h = sum(p[n].numel() * p[n].element_size() for n in ("dq", "dk", "dv", "dlog") if n in p)
            return p, h2d, d2h
        h2d = sum(p[n].numel() * p[n].element_size() for n in ("q", "k", "v", "log_g") if p[n] is not None)
        d2h = p["y"].numel() * p["y"].element_size()
        if self.direction != "bidirectional":
            d2h += p["S"].numel() * 4
        return p, h2d, d2h


def backward_launches(la, wl, kind, carried):
    """Kernel launches of one backward call, as the library issues them: its
    scans (two launches each when T-segmented) and its small kernels."""
    def scan(dk, dv):
        return 2 if (wl.dtype != "f32" and la.workspace_size(wl.B, wl.H, wl.T, dk, dv, wl.torch_dtype, False) > 0) \
            else 1
    decay = kind != 0
    dlog = (3 + (1 if kind == 1 else 0)) if decay else 0  # block scan, block suffixes, offsets, per-head sum
    n = (1 if decay else 0) * 2 + dlog                    # shifted decay, d_init_state scaled by g_1
    if not wl.normalize:
        return n + (1 if carried else 0) + 2 * scan(wl.Dv, wl.Dk) + scan(wl.Dk, wl.Dv)
    if wl.Dv + 1 > 128:  # numerator and denominator terms from separate scans
        return (n + (1 if carried else 0) + (2 if carried else 0) + 1 + scan(wl.Dk, wl.Dv) + scan(wl.Dk, 16) + 1
                + scan(wl.Dv, wl.Dk) + scan(16, wl.Dk) + 1 + scan(wl.Dv, wl.Dk) + scan(16, wl.Dk)
                + scan(wl.Dk, wl.Dv) + 1)
    W = wl.Dv + 16 if wl.dtype != "f32" else wl.Dv + 1
    return (n + (2 if carried else 0) + 1 + scan(wl.Dk, W) + 1 + 2 * scan(W, wl.Dk) + scan(wl.Dk, wl.Dv) + 1)


def decode_graph_timing(job, device, dist_on, reps=3):
    """The decode workload's 1024 token steps captured once in a CUDA graph
    and replayed (the launch overhead of the per-token calls removed), timed
    like the plain steps: CUDA events around each replay, max over ranks."""
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream(device))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        job.step()  # warm the stream before capture
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            job.step()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    barrier(dist_on)
    ms = []
    cur = torch.cuda.current_stream(device)
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        g.replay()
        e1.record(cur)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    barrier(dist_on)
    assert job.la.device_error(device) == 0
    per_token = max_over_ranks(statistics.median(ms), dist_on, device) / job.wl.steps
    del g
    return {"ms_per_token": round(per_token, 5), "launches_per_replay": job.wl.steps,
            "tokens_per_s": job.wl.B * job.wl.H / (per_token / 1e3)}


def barrier(dist_on):
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, dist_on, device):
    """The slowest rank's value (the job's time is set by its slowest GPU)."""
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank):
    """Each rank processes its own batch of independent sequences (weak
    scaling): same shapes and distributions, rank-specific seed."""
    return wl.seed + 7919 * rank


SPIN_UP_S = 0.5
SPACER_CYCLES = 2_000_000  # about 1 ms at the B200's clocks


def spin_up(job, flush, device, min_s=SPIN_UP_S):
    """Untimed steps until the GPU has run them for min_s seconds of wall
    time (at least one), so that the timed steps do not see the SM clock
    ramping up from idle.  Returns the number of steps run."""
    n = 0
    t0 = time.perf_counter()
    while True:
        if flush is not None:
            flush.add_(1)
        job.step()
        n += 1
        if n % 4 == 0 or n == 1:
            torch.cuda.synchronize(device)
            if time.perf_counter() - t0 >= min_s:
                return n


def step_stats(per):
    """Median, minimum and maximum of the per-step event times (ms)."""
    return {"median": round(statistics.median(per), 5), "min": round(min(per), 5), "max": round(max(per), 5)}


def config_dict(wl, cfg, direction, world):
    """The JSON line's `config`: the workload and how it is timed (shared by
    both arms, so that their lines name the same configuration)."""
    if cfg == 5:
        in_l2 = False
    else:
        in_l2 = algorithmic_bytes(wl, cfg, direction) < 2 * L2_BYTES
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "T": wl.T if cfg != 5 else 1,
            "Dk": wl.Dk, "Dv": wl.Dv, "decay": wl.decay, "normalize": wl.normalize,
            "direction": direction,
            "decode_steps": wl.steps if cfg == 5 else None,
            "l2": "flushed before every step (512 MB write)" if in_l2 else "inputs larger than L2",
            "parallelism": f"replicas x{world}; batch sharded across GPUs (weak scaling), no collective"}


def time_steps(job, steps, flush, dist_on, device):
    """Sum of per-step CUDA-event times (ms) over `steps` steps; L2 flushed
    before each step outside the events when `flush` is not None."""
    stream = torch.cuda.current_stream(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches = 0
    barrier(dist_on)
    wall0 = time.time()
    # the device waits about a millisecond (no memory traffic) while the host
    # enqueues the first steps, so that the first step's events time its
    # kernels, not the host's launch latency (the steady state of a queue)
    torch.cuda._sleep(SPACER_CYCLES)
    for i in range(steps):
        if flush is not None:
            flush.add_(1)
        starts[i].record(stream)
        launches += job.step()
        ends[i].record(stream)
    barrier(dist_on)
    wall1 = time.time()
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return per, launches, wall0, wall1


def cpu_baseline(cfg, budget_s=15.0, direction="forward"):
    """The float64 oracle, as it stands, on a bounded sample of the workload:
    whole (b, h) sequences (every token) until about budget_s of CPU work."""
    import oracle
    wl = W.WORKLOADS[cfg]
    oracle.build()
    cores = os.cpu_count() or 1
    if cfg == 5:
        # a sample of heads for a sample of decode tokens
        nh = min(wl.B * wl.H, 64 * cores)
        heads = list(range(nh))
        S, z = W.decode_initial_state(wl, heads=heads)
        S, z = S.double().numpy(), z.double().numpy()
        inps = [W.decode_step_inputs(wl, s, heads=heads) for s in range(4)]
        t0 = time.perf_counter()
        n = 0
        while True:
            inp = inps[n % len(inps)]
            _, S, z = oracle.decode_step(inp["q"], inp["k"], inp["v"], S, z, 1, inp["log_g"], True)
            n += 1
            if time.perf_counter() - t0 > budget_s / 2:
                break
        dt = time.perf_counter() - t0
        return {"value": nh * n / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": f"{nh} of {wl.B * wl.H} (b,h) states, {n} decode tokens, single thread"}
    total = wl.B * wl.H
    # estimate: ~1 GFLOP/s per core for the plain f64 loops
    per_head_s = 4.0 * wl.Dk * wl.Dv * (wl.T + wl.prefix_T) / 1e9
    if direction == "bidirectional":
        per_head_s *= 2
    if direction == "backward":
        per_head_s *= 4  # a checkpointed forward sweep and the backward sweep
    nh = max(1, min(total, int(budget_s * cores / max(per_head_s, 1e-9))))
    nh = min(nh, total)
    heads = list(range(nh))
    inp = W.forward_inputs(wl, heads=heads)
    threads = min(cores, nh)
    init = {}
    if wl.prefix_T and direction != "bidirectional":
        pre = W.prefix_inputs(wl, heads=heads)
        _, S0, z0 = oracle.forward(pre["q"], pre["k"], pre["v"], 0, None, True, nthreads=threads)
        init = dict(init_state=S0, init_z=z0)
    fn = {"forward": oracle.forward, "reverse": oracle.reverse}.get(direction)
    if direction == "backward":
        g = torch.Generator().manual_seed(wl.seed + 500)
        dy = torch.randn(nh, wl.T, wl.Dv, generator=g).reshape(1, nh, wl.T, wl.Dv).to(wl.torch_dtype)
        dy = dy.reshape(inp["q"].shape[:3] + (wl.Dv,))
    t0 = time.perf_counter()
    if direction == "backward":
        oracle.backward(inp["q"], inp["k"], inp["v"], dy, inp["decay_kind"], inp["log_g"], wl.normalize,
                        nthreads=threads, **init)
    elif fn is None:
        oracle.bidirectional(inp["q"], inp["k"], inp["v"], inp["decay_kind"], inp["log_g"], wl.normalize,
                             nthreads=threads)
    else:
        fn(inp["q"], inp["k"], inp["v"], inp["decay_kind"], inp["log_g"], wl.normalize, nthreads=threads, **init)
    dt = time.perf_counter() - t0
    return {"value": nh * wl.T / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{nh} of {total} (b,h) sequences, all {wl.T} tokens each, {threads} threads"}


def sized_workload(args, cfg):
    """The workload of config `cfg`, with --tokens / --batch overrides
    (smaller cases for profiler captures); an override renames the workload."""
    wl = W.WORKLOADS[cfg]
    if args.tokens and cfg != 5:
        wl = wl.with_sizes(T=args.tokens, name=f"{wl.name}_T{args.tokens}")
    if args.batch:
        wl = wl.with_sizes(B=args.batch, name=f"{wl.name}_B{args.batch}")
    return wl


def run_ours(args, rank, world, dist_on, device, cfg=None, prologue=False):
    cfg = args.config if cfg is None else cfg
    wl = sized_workload(args, cfg)
    job = Job(cfg, device, wl, rank, args.direction, prologue=prologue)
    if job.prologue:
        wl = job.wl = wl.with_sizes(name=wl.name + "_raw_qk_elu1_in_kernel")
    torch.cuda.synchronize()
    in_bytes = algorithmic_bytes(wl, cfg, args.direction) * (wl.steps if cfg == 5 else 1)
    flush = None
    if in_bytes < 2 * L2_BYTES and cfg != 5:
        flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    for _ in range(args.warmup):
        if flush is not None:
            flush.add_(1)
        job.step()
    torch.cuda.synchronize()
    spun = spin_up(job, flush, device)
    assert job.la.device_error(device) == 0

    sampler = ClockSampler(bus_id_of(device)) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    per, launches, w0, w1 = time_steps(job, args.steps, flush, dist_on, device)
    if sampler:
        time.sleep(0.3)
        sampler.stop()
    assert job.la.device_error(device) == 0
    total_ms = max_over_ranks(sum(per), dist_on, device)
    ms_per_step = total_ms / args.steps
    tokens = tokens_per_step(wl, cfg) * world
    value = tokens / (ms_per_step / 1e3)
    graph = decode_graph_timing(job, device, dist_on) if cfg == 5 and not args.skip_e2e else None

    # the path's kernels: one decode call, or one forward (a T-segmented forward
    # is a state pass and an output pass of the same kernel, timed together)
    launch_ms = ms_per_step / (wl.steps if cfg == 5 else 1)
    pk, pk_kind = peaks()
    bytes_launch = algorithmic_bytes(wl, cfg, args.direction)
    achieved_gbs = bytes_launch / (launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved_gbs / pk["hbm_gbs"], 4),
                # the committed counters are the forward instances' (other directions: none taken)
                "traffic": measured_traffic(wl.name) if args.direction == "forward" else None,
                "peak_source": pk_kind,
                "kernel": "la_decode (decode_vec_kernel)" if cfg == 5 else
                ("la_fwd_f32 (fwd_f32_kernel)" if wl.dtype == "f32" else
                 ("fwd_ws_kernel (three scans) and the backward's small kernels"
                  if args.direction == "backward" else
                  {1: "fwd_ws_kernel", 2: "fwd_ws_kernel (state pass + output pass)"
                   if args.direction != "bidirectional" else "fwd_ws_kernel (forward + reverse scan)",
                   4: "fwd_ws_kernel (state + output pass, forward and reverse)"}[job.fwd_launches])),
                "algorithmic_bytes_per_launch": bytes_launch,
                "tensor_frac": round(algorithmic_flops(wl, cfg, args.direction) / (launch_ms / 1e3) / 1e12 / pk.get("bf16_tflops", 1590.0), 4)}

    # end to end through the public API with host buffers
    e2e = None
    if not args.skip_e2e:
        pinned, h2d, d2h = job.make_pinned()
        stream = torch.cuda.current_stream(device)
        e_steps = max(1, min(args.steps, 20))
        for _ in range(2):
            job.e2e_step(pinned, stream)
        barrier(dist_on)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        e_tokens = 0
        for _ in range(e_steps):
            e_tokens += job.e2e_step(pinned, stream)
        ev1.record(stream)
        barrier(dist_on)
        e_ms = max_over_ranks(ev0.elapsed_time(ev1), dist_on, device) / e_steps
        e2e = {"value": e_tokens / e_steps * world / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4)}

    clocks = sampler.summary(w0, w1) if sampler else None
    # per-step statistics, the slowest rank's (max over ranks of each)
    stats = {k: max_over_ranks(v, dist_on, device) for k, v in step_stats(per).items()}
    line = {
        "metric": metric_for(args.direction), "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if wl.dtype == "f32" else "bf16", "data": "synthetic",
        "config": config_dict(wl, cfg, args.direction, world),
        "roofline": roofline, "e2e": e2e, "clocks": clocks,
        "gpu_launches": launches,
        "ms_per_step_stats": stats,
        "spin_up": {"steps": spun, "min_s": SPIN_UP_S},
        "plan": ("decode: one CTA per (b, h)" if cfg == 5 else
                 "one CTA per (b, h)" if wl.dtype == "f32" else
                 "per GPU (b, h) spread over CTAs by value slices"
                 + (" and T-segments (state pass + output pass)" if job.fwd_launches in (2, 4) and
                    (args.direction != "bidirectional" or job.fwd_launches == 4) else "")),
    }
    if graph:
        line["decode_graph"] = graph
    if job.prologue:
        # the same step with the feature map applied by a caller pass instead
        # (it reads and writes q and k once more: 4 B H T Dk bf16 bytes)
        for _ in range(3):
            job.caller_mapped_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(torch.cuda.current_stream(device))
        for _ in range(args.steps):
            job.caller_mapped_step()
        e1.record(torch.cuda.current_stream(device))
        barrier(dist_on)
        caller_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist_on, device)
        line["feature_map"] = {"where": "in the forward kernel (la_chunk_forward_pro_ws, FEATURE_ELU1) on raw q, k",
                               "caller_pass_ms_per_step": round(caller_ms, 5),
                               "caller_pass_extra_hbm_bytes": 4 * wl.B * wl.H * wl.T * wl.Dk * 2,
                               "saving_ms_per_step": round(caller_ms - ms_per_step, 5)}
    return line


# ---------------------------------------------------------------- RWKV-4 WKV (config 6)

WKV4_METRIC = "rwkv4-wkv forward tokens/s (B·T/s) and % of roofline (HBM GB/s)"


def wkv4_bytes(wl):
    """Bytes one la_wkv4_forward call must move: k, v read and out written
    once, w and u read, the fp32 final state written."""
    es = 2 if wl.dtype == "bf16" else 4
    return wl.B * wl.T * wl.C * 3 * es + 2 * wl.C * 4 + wl.B * 3 * wl.C * 4


EMA_METRIC = "cumulative-ema tokens/s (B·T/s) and % of roofline (HBM GB/s)"


def ema_bytes(wl):
    """Bytes one la_ema_scan call must move: x, f read and out written once,
    the fp32 final state written."""
    es = 2 if wl.dtype == "bf16" else 4
    return wl.B * wl.T * wl.C * 3 * es + wl.B * wl.C * 4


class EmaJob:
    def __init__(self, device, wl, rank=0, reverse=False):
        import retention_scan_b200 as la
        self.la, self.wl, self.dev, self.reverse = la, wl, device, reverse
        self.host = W.ema_inputs(wl.with_sizes(seed=wl.seed + 7919 * rank))
        self.x, self.f = (self.host[n].to(device) for n in ("x", "f"))
        self.out = torch.empty(wl.B, wl.T, wl.C, dtype=wl.torch_dtype, device=device)
        self.fin = torch.empty(wl.B, wl.C, dtype=torch.float32, device=device)
        self.launches = 1

    def step(self):
        self.la.ema_scan(self.x, self.f, out=self.out, final_state=self.fin, reverse=self.reverse)
        return 1

    def e2e(self, steps, dist_on):
        p = {n: self.host[n].pin_memory() for n in ("x", "f")}
        y = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        stream = torch.cuda.current_stream(self.dev)

        def one():
            x, f = (p[n].to(self.dev, non_blocking=True) for n in ("x", "f"))
            o, _ = self.la.ema_scan(x, f, out=self.out, final_state=self.fin, reverse=self.reverse)
            y.copy_(o, non_blocking=True)
        for _ in range(2):
            one()
        barrier(dist_on)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            one()
        ev1.record(stream)
        barrier(dist_on)
        h2d = sum(p[n].numel() * p[n].element_size() for n in p)
        return ev0.elapsed_time(ev1) / steps, h2d, y.numel() * y.element_size()


def cpu_baseline_ema(wl, budget_s=15.0, reverse=False):
    """The float64 oracle (single-threaded C loop) on whole batch rows."""
    import oracle
    oracle.build()
    per_row_s = wl.T * wl.C * 6 / 1e9
    nb = max(1, min(wl.B, int(budget_s / max(per_row_s, 1e-9))))
    inp = W.ema_inputs(wl, batches=range(nb))
    t0 = time.perf_counter()
    oracle.ema(inp["x"], inp["f"], reverse=reverse)
    dt = time.perf_counter() - t0
    return {"value": nb * wl.T / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{nb} of {wl.B} batch rows, all {wl.T} tokens x {wl.C} channels, single thread"}


class Wkv4Job:
    def __init__(self, device, wl, rank=0):
        import retention_scan_b200 as la
        self.la, self.wl, self.dev = la, wl, device
        self.host = W.wkv4_inputs(wl.with_sizes(seed=wl.seed + 7919 * rank))
        self.k, self.v, self.w, self.u = (self.host[n].to(device) for n in ("k", "v", "w", "u"))
        self.out = torch.empty(wl.B, wl.T, wl.C, dtype=wl.torch_dtype, device=device)
        self.fin = torch.empty(wl.B, 3, wl.C, dtype=torch.float32, device=device)
        nb = la.wkv4_workspace_size(wl.B, wl.T, wl.C, wl.torch_dtype)
        self.ws = torch.empty(nb, dtype=torch.uint8, device=device) if nb else False
        self.launches = 2 if nb else 1  # a state pass before the output pass when segmented

    def step(self):
        self.la.wkv4_forward(self.k, self.v, self.w, self.u, out=self.out, final_state=self.fin, workspace=self.ws)
        return self.launches

    def e2e(self, steps, dist_on):
        p = {n: self.host[n].pin_memory() for n in ("k", "v", "w", "u")}
        y = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        stream = torch.cuda.current_stream(self.dev)

        def one():
            k, v, w, u = (p[n].to(self.dev, non_blocking=True) for n in ("k", "v", "w", "u"))
            o, _ = self.la.wkv4_forward(k, v, w, u, out=self.out, final_state=self.fin, workspace=self.ws)
            y.copy_(o, non_blocking=True)
        for _ in range(2):
            one()
        barrier(dist_on)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            one()
        ev1.record(stream)
        barrier(dist_on)
        h2d = sum(p[n].numel() * p[n].element_size() for n in p)
        return ev0.elapsed_time(ev1) / steps, h2d, y.numel() * y.element_size()


def cpu_baseline_wkv4(wl, budget_s=15.0):
    """The float64 oracle (single-threaded C loop) on whole batch rows of the
    workload until about budget_s of work."""
    import oracle
    oracle.build()
    per_row_s = wl.T * wl.C * 40 / 1e9  # rough: ~40 f64 operations per channel step
    nb = max(1, min(wl.B, int(budget_s / max(per_row_s, 1e-9))))
    inp = W.wkv4_inputs(wl, batches=range(nb))
    t0 = time.perf_counter()
    oracle.wkv4(inp["k"], inp["v"], inp["w"], inp["u"])
    dt = time.perf_counter() - t0
    return {"value": nb * wl.T / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{nb} of {wl.B} batch rows, all {wl.T} tokens x {wl.C} channels, single thread"}


def run_wkv4(args, rank, world, dist_on, device):
    """The per-channel scans on [B, T, C]: config 6 (RWKV-4 WKV), config 7
    (cumulative EMA)."""
    ema = args.config == 7
    wl = W.EMA if ema else W.WKV4
    if args.tokens:
        wl = wl.with_sizes(T=args.tokens, name=f"{wl.name}_T{args.tokens}")
    if args.batch:
        wl = wl.with_sizes(B=args.batch, name=f"{wl.name}_B{args.batch}")
    job = EmaJob(device, wl, rank, reverse=args.direction == "reverse") if ema else Wkv4Job(device, wl, rank)
    nbytes = (ema_bytes if ema else wkv4_bytes)(wl)
    flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=device) if nbytes < 2 * L2_BYTES else None
    for _ in range(args.warmup):
        if flush is not None:
            flush.add_(1)
        job.step()
    torch.cuda.synchronize()
    spun = spin_up(job, flush, device)
    assert job.la.device_error(device) == 0
    sampler = ClockSampler(bus_id_of(device)) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    per, launches, w0, w1 = time_steps(job, args.steps, flush, dist_on, device)
    if sampler:
        time.sleep(0.3)
        sampler.stop()
    assert job.la.device_error(device) == 0
    ms = max_over_ranks(sum(per), dist_on, device) / args.steps
    stats = {k: max_over_ranks(v, dist_on, device) for k, v in step_stats(per).items()}
    pk, pk_kind = peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    e2e = None
    if not args.skip_e2e:
        e_ms, h2d, d2h = job.e2e(max(1, min(args.steps, 20)), dist_on)
        e_ms = max_over_ranks(e_ms, dist_on, device)
        e2e = {"value": wl.B * wl.T * world / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4)}
    return {
        "metric": EMA_METRIC if ema else WKV4_METRIC, "value": wl.B * wl.T * world / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "C": wl.C,
                   **({"direction": args.direction} if ema else {}),
                   "l2": "flushed before every step (512 MB write)" if flush is not None
                   else "inputs larger than L2",
                   "parallelism": f"replicas x{world}; batch sharded across GPUs (weak scaling), no collective"},
        "plan": "per GPU one CTA per (batch row, 64 channels" + (", T-segment)" if job.launches == 2 else ")"),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / pk["hbm_gbs"], 4),
                     "traffic": measured_traffic(wl.name) if args.direction == "forward" else None,
                     "peak_source": pk_kind,
                     "kernel": "ema_kernel" if ema else
                     ("wkv4_kernel (state pass + output pass)" if job.launches == 2 else "wkv4_kernel"),
                     "algorithmic_bytes_per_launch": nbytes},
        "e2e": e2e, "clocks": sampler.summary(w0, w1) if sampler else None, "gpu_launches": launches,
        "ms_per_step_stats": stats, "spin_up": {"steps": spun, "min_s": SPIN_UP_S},
    }


# ---------------------------------------------------------------- reference arm (the oracle)

def run_reference(args, world):
    """The oracle as it stands on the host cores: each step a bounded sample of
    the workload, sized so that W + K steps take about two and a half minutes."""
    cfg = args.config
    per_step_s = min(8.0, max(1.0, 150.0 / max(1, args.steps + args.warmup)))
    if cfg in (6, 7):
        wl = W.WKV4 if cfg == 6 else W.EMA
        base = cpu_baseline_wkv4 if cfg == 6 else cpu_baseline_ema
        for _ in range(args.warmup):
            base(wl, budget_s=min(2.0, per_step_s))
        vals = [base(wl, budget_s=per_step_s) for _ in range(args.steps)]
        v = statistics.median(x["value"] for x in vals)
        cb = dict(vals[-1])
        cb["value"] = v
        return {"impl": "reference", "metric": WKV4_METRIC if cfg == 6 else EMA_METRIC, "value": v, "unit": "tokens/s",
                "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": wl.B * wl.T / v * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic",
                "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "C": wl.C,
                           **({"direction": args.direction} if cfg == 7 else {}),
                           "l2": "flushed before every step (512 MB write)"
                           if (ema_bytes if cfg == 7 else wkv4_bytes)(wl) < 2 * L2_BYTES else "inputs larger than L2",
                           "parallelism": f"replicas x{world}; batch sharded across GPUs (weak scaling), no collective"},
                "cpu_baseline": cb,
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                "gpu_launches": 0}
    wl = W.WORKLOADS[cfg]
    for _ in range(args.warmup):
        cpu_baseline(cfg, budget_s=min(2.0, per_step_s), direction=args.direction)
    vals = []
    for _ in range(args.steps):
        vals.append(cpu_baseline(cfg, budget_s=per_step_s, direction=args.direction))
    v = statistics.median(x["value"] for x in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    return {
        "impl": "reference", "metric": metric_for(args.direction), "value": v, "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tokens_per_step(wl, cfg) / v * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, cfg, args.direction, world),
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


EXTRA_CONFIGS = (3, 5, 2)  # measured beside the headline config 4 by the default run
# and, beside them, the gated workload's backward and the two per-channel scans
EXTRA_LINES = (("backward", 4), ("forward", 6), ("forward", 7))


def free_port():
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def launch_ranks(n):
    """`--gpus N` outside torchrun: run this command as N local ranks under
    torch.distributed.run (rank 0 prints the line) and return its status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__), *sys.argv[1:]]
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "1"))
    return subprocess.run(cmd, env=env).returncode


def cpu_selftest(rank, world):
    """The multi-rank timing path without a GPU (gloo): rank r times a host
    busy loop of (r + 1) * 20 ms per step, between barriers; the reported
    time is the maximum over ranks, as for the GPU steps."""
    import datetime
    torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        torch.distributed.barrier()
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 0.02 * (rank + 1):
            pass
        ms = (time.perf_counter() - t0) * 1e3
        torch.distributed.barrier()
        t = torch.tensor([ms], dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        mine = torch.tensor([ms], dtype=torch.float64)
        every = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        torch.distributed.all_gather(every, mine)
        if rank == 0:
            print(json.dumps({"selftest": True, "n_gpus": world, "ms_per_step": float(t.item()),
                              "per_rank_ms": [float(x.item()) for x in every]}), flush=True)
    finally:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--config", type=int, default=None, choices=[1, 2, 3, 4, 5, 6, 7],
                    help="time one workload only (default: config 4 with configs 3, 5 and 2 beside it, "
                         "the backward of config 4, and configs 6 and 7)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=0, help="override T (profiling a smaller case)")
    ap.add_argument("--batch", type=int, default=0, help="override B (profiling a smaller case)")
    ap.add_argument("--direction", default="forward", choices=["forward", "reverse", "bidirectional", "backward"])
    ap.add_argument("--cpu-selftest", action="store_true", help=argparse.SUPPRESS)
    args = ap.parse_args()
    combined = args.config is None
    if combined:
        args.config = 4
    if args.config in (5, 6) and args.direction != "forward":
        ap.error("--direction applies to the whole-sequence configs 1-4 and 7")
    if args.config == 7 and args.direction not in ("forward", "reverse"):
        ap.error("the cumulative EMA (config 7) scans forward or reverse")
    if combined and args.direction != "forward":
        combined = False  # the extra configs are forward lines
    default_steps = {1: 2000, 2: 2000, 3: 200, 4: 50, 5: 3, 6: 200, 7: 200}
    if args.steps is None:
        args.steps = default_steps[args.config] if args.impl == "ours" else 3
    if args.warmup is None:
        args.warmup = max(3, args.steps // 20) if args.impl == "ours" else 1
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(launch_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but {world} ranks were launched")

    if args.cpu_selftest:
        cpu_selftest(rank, world)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=device,
                                             timeout=datetime.timedelta(seconds=120))
    try:
        line = (run_wkv4 if args.config in (6, 7) else run_ours)(args, rank, world, dist_on, device)
        extra = {}   # name -> (line, config, direction)
        if combined:
            for cfg in EXTRA_CONFIGS:
                sub = run_ours(args, rank, world, dist_on, device, cfg=cfg)
                extra[sub["config"]["workload"]] = (sub, cfg, "forward")
                torch.cuda.empty_cache()
                if cfg == 3:  # the normalised workload once more, with the feature map in the kernel
                    sub = run_ours(args, rank, world, dist_on, device, cfg=cfg, prologue=True)
                    extra[sub["config"]["workload"]] = (sub, cfg, "forward")
                    torch.cuda.empty_cache()
            for direction, cfg in EXTRA_LINES:
                a2 = argparse.Namespace(**vars(args))
                a2.config, a2.direction = cfg, direction
                sub = (run_wkv4 if cfg in (6, 7) else run_ours)(a2, rank, world, dist_on, device)
                name = sub["config"]["workload"] + ("" if direction == "forward" else "_" + direction)
                extra[name] = (sub, cfg, direction)
                torch.cuda.empty_cache()
        if rank == 0:
            if world == 1 and not args.skip_cpu_baseline:
                line["cpu_baseline"] = (cpu_baseline_wkv4(W.WKV4) if args.config == 6 else
                                        cpu_baseline_ema(W.EMA, reverse=args.direction == "reverse")
                                        if args.config == 7 else
                                        cpu_baseline(args.config, direction=args.direction))
                for sub, cfg, direction in extra.values():
                    sub["cpu_baseline"] = (cpu_baseline_wkv4(W.WKV4, budget_s=8.0) if cfg == 6 else
                                           cpu_baseline_ema(W.EMA, budget_s=8.0) if cfg == 7 else
                                           cpu_baseline(cfg, budget_s=8.0, direction=direction))
            if extra:
                # each record keeps its metric and unit where they differ from the headline's
                line["configs"] = {name: {k: v for k, v in sub.items()
                                          if k not in ("higher_is_better", "scaling", "data")
                                          and not (k in ("metric", "unit") and v == line[k])}
                                   for name, (sub, _, _) in extra.items()}
            print(json.dumps(line), flush=True)
    finally:
        if dist_on:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
