"""Shared helpers of the GPU parity tests: tolerance metric and oracle calls.

Tolerance (the stated bar): max relative error 1e-4 for fp32 inputs and 2e-2
for bf16 inputs with fp32 accumulation.  "Relative error" of an array is
measured per (b, h) slice as max |x - ref| / max |ref| and the worst slice is
reported, so values near zero inside a slice are judged against the slice's
scale rather than against themselves.
"""
import numpy as np
import torch

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
