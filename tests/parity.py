"""Shared helpers of the GPU parity tests: tolerance metric and oracle calls.

Tolerance (the stated bar): max relative error 1e-4 for fp32 inputs and 2e-2
for bf16 inputs with fp32 accumulation.  "Relative error" of an array is
measured per (b, h) slice as max |x - ref| / max |ref| and the worst slice is
reported, so values near zero inside a slice are judged against the slice's
scale rather than against themselves.
"""
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(x, ref):
    """Worst (b,h)-slice max|x-ref| / max|ref|; x and ref shaped [B,H,...]."""
    x = x.detach().to("cpu").double().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if x.size == 0:
        return 0.0
    B, H = ref.shape[:2]
    xs = x.reshape(B * H, -1)
    rs = ref.reshape(B * H, -1)
    worst = 0.0
    for a, r in zip(xs, rs):
        scale = float(np.max(np.abs(r)))
        err = float(np.max(np.abs(a - r)))
        if not np.isfinite(err):
            return float("inf")
        worst = max(worst, err / scale if scale > 0 else err)
    return worst


def oracle_forward(inp, normalize=False, init_state=None, init_z=None):
    """Oracle on the exact input bits of a workload dict (CPU tensors)."""
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["decay_kind"], inp["log_g"], normalize,
                          init_state, init_z)


def to_dev(inp, device="cuda"):
    out = dict(inp)
    for key in ("q", "k", "v", "log_g"):
        if out.get(key) is not None:
            out[key] = out[key].to(device).contiguous()
    return out


def gen_case(B, H, T, Dk, Dv, dtype=torch.bfloat16, kind=0, normalize=False, seed=0,
             decay_mean=2.0, init=False):
    """Random case: q, k ~ elu+1 of N(0,1) when normalised, else N(0,1) with q
    scaled by Dk^-1/2; v ~ N(0,1); per-step log g = logsigmoid(N(decay_mean,1));
    per-head log g = log(1 - 2^(-1-h)) (strong decays that the test can see)."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, T, Dk, generator=g)
    k = torch.randn(B, H, T, Dk, generator=g)
    v = torch.randn(B, H, T, Dv, generator=g)
    if normalize:
        q, k = F.elu(q) + 1, F.elu(k) + 1
    else:
        q = q * Dk ** -0.5
    log_g = None
    if kind == 1:
        log_g = torch.tensor([math.log1p(-2.0 ** (-1 - h)) for h in range(H)], dtype=torch.float32)
    elif kind == 2:
        log_g = F.logsigmoid(torch.randn(B, H, T, generator=g) + decay_mean)
    S0 = torch.randn(B, H, Dk, Dv, generator=g) if init else None
    z0 = (torch.rand(B, H, Dk, generator=g) * 4 + 0.5) if (init and normalize) else None
    return dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), log_g=log_g, decay_kind=kind), S0, z0
