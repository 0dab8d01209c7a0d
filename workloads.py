"""Seeded synthetic workloads for causal linear attention.

This module only draws random inputs and applies the caller-side input
preparation that each workload names (feature map, query scale, decay
parametrisation).  It holds none of the attention arithmetic; tests, the
oracle and the benchmark all take their inputs from here.

Every (batch, head) slice has its own generator, seeded from
(workload seed, stream, b*H + h), so a single head can be regenerated without
drawing the others, and a sampled-head check sees exactly the bits that the
full-size run saw.  Streams: 0 q, 1 k, 2 v, 3 decay pre-activation a,
4 initial state, 5 initial key sum.

Workloads (sizes are the defaults; every builder takes overrides so tests can
run the same recipe at smaller sizes):

  plain      g = 1, no normaliser, fp32, q,k,v ~ N(0,1)/sqrt(Dk), zero start
             (B=1, H=1, T=64, Dk=Dv=16, seed 0)
  retention  per-head gamma_h = 1 - 2^(-5-h), bf16, q scaled by Dk^-1/2
             (B=4, H=8, T=2048, Dk=Dv=64, seed 2)
  normalized feature map elu(x)+1 on q and k, g = 1, normalised output, and a
             carried state / key sum from a 512-token prefix
             (B=8, H=16, T=4096, Dk=Dv=128, seed 3; prefix seed 103)
  gated      per-step g = sigmoid(a), a ~ N(4,1), passed as log g = logsigmoid(a)
             in fp32; q scaled by Dk^-1/2 (B=1, H=32, T=65536, Dk=Dv=128, seed 4)
  decode     one token per call, per-head gamma_h, normalised with elu(x)+1 on
             q and k, fp32 state ~ N(0, 0.01^2), key sum |N(0, 0.01^2)|
             (B=256, H=32, Dk=Dv=128, 1024 steps, seed 5)
  ema        RetNet issue 21's cumulative EMA: values x ~ N(0,1) and factors
             f = sigmoid(a), a ~ N(3,1) (the page's elementwise EMA uses
             sigmoid factors), bf16 [B,T,C]; zero start (B=8, T=4096,
             C=2048, seed 7)
  wkv4       the RWKV-4 WKV recurrence: k, v ~ N(0,1) bf16 [B,T,C]; per
             channel w = -exp(d), d ~ N(-1, 1.5^2) (decay factors from about
             0.99 to near 0) and bonus u ~ N(-0.6, 0.4^2), fp32; empty start
             (B=8, T=4096, C=2048, seed 6).  The page gives no sizes or
             values: these are a mid-sized RWKV-4 layer's shapes.
"""
import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch
import torch.nn.functional as F

Q, K, V, A, S0, Z0 = range(6)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    Dk: int
    Dv: int
    dtype: str                 # "f32" or "bf16": q, k, v, out
    decay: str                 # "none", "per_head", "per_step"
    normalize: bool
    q_scale: Optional[float]   # multiply q by this (None: 1)
    all_scale: Optional[float] = None  # multiply q, k, v by this (plain workload)
    feature_map: Optional[str] = None  # None or "elu1" on q and k
    prefix_T: int = 0          # tokens of the carried-state prefix (0: zero start)
    steps: int = 0             # decode workload: tokens per run
    seed: int = 0
    prefix_seed: int = 0
    extra: dict = field(default_factory=dict)

    def with_sizes(self, **kw):
        return replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


PLAIN = Workload("plain_b1h1t64d16_f32", 1, 1, 64, 16, 16, "f32", "none", False,
                 q_scale=None, all_scale=1.0 / math.sqrt(16), seed=0)
RETENTION = Workload("retention_b4h8t2048d64_bf16", 4, 8, 2048, 64, 64, "bf16", "per_head",
                     False, q_scale=64 ** -0.5, seed=2)
NORMALIZED = Workload("normalized_b8h16t4096d128_bf16", 8, 16, 4096, 128, 128, "bf16", "none",
                      True, q_scale=None, feature_map="elu1", prefix_T=512, seed=3,
                      prefix_seed=103)
GATED = Workload("gated_b1h32t65536d128_bf16", 1, 32, 65536, 128, 128, "bf16", "per_step",
                 False, q_scale=128 ** -0.5, seed=4)
DECODE = Workload("decode_b256h32d128_steps1024", 256, 32, 1, 128, 128, "bf16", "per_head",
                  True, q_scale=None, feature_map="elu1", steps=1024, seed=5)

WORKLOADS = {1: PLAIN, 2: RETENTION, 3: NORMALIZED, 4: GATED, 5: DECODE}


def _gen(seed, stream, bh, step=0):
    g = torch.Generator()
    g.manual_seed(((seed * 8 + stream) * 4096 + step) * 1_000_003 + bh)
    return g


def _normal(shape, seed, stream, bh, step=0, mean=0.0, std=1.0):
    x = torch.randn(shape, generator=_gen(seed, stream, bh, step), dtype=torch.float32)
    if std != 1.0:
        x = x * std
    if mean != 0.0:
        x = x + mean
    return x


def _prep_qk(x, wl, which):
    if wl.feature_map == "elu1":
        x = F.elu(x) + 1.0
    if wl.all_scale is not None:
        x = x * wl.all_scale
    if which == Q and wl.q_scale is not None:
        x = x * wl.q_scale
    return x


def per_head_log_gamma(H):
    """log(gamma_h) for gamma_h = 1 - 2^(-5-h), computed in float64 as
    log1p(-2^(-5-h)) and rounded once to fp32."""
    return torch.tensor([math.log1p(-2.0 ** (-5 - h)) for h in range(H)],
                        dtype=torch.float64).to(torch.float32)


def _heads(wl, heads):
    return list(range(wl.B * wl.H)) if heads is None else list(heads)


def forward_inputs(wl, heads=None, seed=None, T=None):
    """Inputs of a whole-sequence forward.

    heads: None for every (b, h), else a list of b*H + h indices; the result
    then has B=1, H=len(heads) and those slices in that order (decay per head
    follows each slice's own h).  Returns a dict of CPU tensors:
    q, k [B,H,T,Dk] and v [B,H,T,Dv] in the workload dtype; log_g (fp32, [H]
    or [B,H,T]) or None; decay_kind (0/1/2).
    """
    seed = wl.seed if seed is None else seed
    T = wl.T if T is None else T
    hs = _heads(wl, heads)
    qs, ks, vs, ls = [], [], [], []
    for bh in hs:
        qs.append(_prep_qk(_normal((T, wl.Dk), seed, Q, bh), wl, Q))
        ks.append(_prep_qk(_normal((T, wl.Dk), seed, K, bh), wl, K))
        vv = _normal((T, wl.Dv), seed, V, bh)
        if wl.all_scale is not None:
            vv = vv * wl.all_scale
        vs.append(vv)
        if wl.decay == "per_step":
            a = _normal((T,), seed, A, bh, mean=4.0)
            ls.append(F.logsigmoid(a))
    shape_bh = (wl.B, wl.H) if heads is None else (1, len(hs))
    dt = wl.torch_dtype
    out = {
        "q": torch.stack(qs).reshape(*shape_bh, T, wl.Dk).to(dt),
        "k": torch.stack(ks).reshape(*shape_bh, T, wl.Dk).to(dt),
        "v": torch.stack(vs).reshape(*shape_bh, T, wl.Dv).to(dt),
        "log_g": None,
        "decay_kind": {"none": 0, "per_head": 1, "per_step": 2}[wl.decay],
    }
    if wl.decay == "per_head":
        lg = per_head_log_gamma(wl.H)
        if heads is not None:
            lg = torch.stack([lg[bh % wl.H] for bh in hs])
        out["log_g"] = lg
    elif wl.decay == "per_step":
        out["log_g"] = torch.stack(ls).reshape(*shape_bh, T)
    return out


def prefix_inputs(wl, heads=None):
    """Inputs of the carried-state prefix (normalized workload): the same
    recipe as forward_inputs with the prefix seed and prefix_T tokens."""
    return forward_inputs(wl, heads=heads, seed=wl.prefix_seed, T=wl.prefix_T)


def decode_initial_state(wl, heads=None):
    """Decode workload start: state [B,H,Dk,Dv] ~ N(0, 0.01^2) and key sum
    [B,H,Dk] = |N(0, 0.01^2)|, both fp32."""
    hs = _heads(wl, heads)
    S = torch.stack([_normal((wl.Dk, wl.Dv), wl.seed, S0, bh, std=0.01) for bh in hs])
    z = torch.stack([_normal((wl.Dk,), wl.seed, Z0, bh, std=0.01).abs() for bh in hs])
    shape_bh = (wl.B, wl.H) if heads is None else (1, len(hs))
    return S.reshape(*shape_bh, wl.Dk, wl.Dv), z.reshape(*shape_bh, wl.Dk)


def decode_step_inputs(wl, step, heads=None):
    """Token `step` of the decode workload: q, k [B,H,Dk], v [B,H,Dv] in the
    workload dtype, plus log_g [H] (per-head gamma) and decay_kind."""
    hs = _heads(wl, heads)
    q = torch.stack([_prep_qk(_normal((wl.Dk,), wl.seed, Q, bh, step + 1), wl, Q) for bh in hs])
    k = torch.stack([_prep_qk(_normal((wl.Dk,), wl.seed, K, bh, step + 1), wl, K) for bh in hs])
    v = torch.stack([_normal((wl.Dv,), wl.seed, V, bh, step + 1) for bh in hs])
    shape_bh = (wl.B, wl.H) if heads is None else (1, len(hs))
    lg = per_head_log_gamma(wl.H)
    if heads is not None:
        lg = torch.stack([lg[bh % wl.H] for bh in hs])
    dt = wl.torch_dtype
    return {"q": q.reshape(*shape_bh, wl.Dk).to(dt), "k": k.reshape(*shape_bh, wl.Dk).to(dt),
            "v": v.reshape(*shape_bh, wl.Dv).to(dt), "log_g": lg, "decay_kind": 1}


def decode_pool_device(wl, steps, device, seed_offset=0):
    """Decode-benchmark tokens drawn on the device in one go (same
    distributions as decode_step_inputs, different bits): q, k [steps,B,H,Dk],
    v [steps,B,H,Dv] in the workload dtype."""
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed * 1_000_003 + seed_offset)
    shp_k = (steps, wl.B, wl.H, wl.Dk)
    shp_v = (steps, wl.B, wl.H, wl.Dv)
    q = torch.randn(shp_k, generator=g, device=device)
    k = torch.randn(shp_k, generator=g, device=device)
    v = torch.randn(shp_v, generator=g, device=device)
    q = _prep_qk(q, wl, Q).to(wl.torch_dtype)
    k = _prep_qk(k, wl, K).to(wl.torch_dtype)
    return q, k, v.to(wl.torch_dtype)


# ---------------------------------------------------------------- RWKV-4 WKV

@dataclass(frozen=True)
class Wkv4Workload:
    name: str
    B: int
    T: int
    C: int
    dtype: str   # "bf16" or "f32": k, v, out
    seed: int

    def with_sizes(self, **kw):
        return replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WKV4 = Wkv4Workload("wkv4_b8t4096c2048_bf16", B=8, T=4096, C=2048, dtype="bf16", seed=6)


def wkv4_inputs(wl, batches=None):
    """k, v [b, T, C] for the listed batch rows (all by default), each row
    from its own generators; w, u [C] fp32 from the workload seed."""
    rows = list(range(wl.B)) if batches is None else list(batches)
    k = torch.stack([_normal((wl.T, wl.C), wl.seed, Q, b) for b in rows]) if rows else \
        torch.zeros(0, wl.T, wl.C)
    v = torch.stack([_normal((wl.T, wl.C), wl.seed, V, b) for b in rows]) if rows else \
        torch.zeros(0, wl.T, wl.C)
    d = _normal((wl.C,), wl.seed, A, 0, mean=-1.0, std=1.5)
    w = -torch.exp(d)
    u = _normal((wl.C,), wl.seed, S0, 0, mean=-0.6, std=0.4)
    return dict(k=k.to(wl.torch_dtype), v=v.to(wl.torch_dtype), w=w.float(), u=u.float())


# ---------------------------------------------------------------- cumulative EMA

EMA = Wkv4Workload("ema_b8t4096c2048_bf16", B=8, T=4096, C=2048, dtype="bf16", seed=7)


def ema_inputs(wl, batches=None):
    """x, f [b, T, C] for the listed batch rows (all by default), each row
    from its own generators: x ~ N(0,1), f = sigmoid(N(3,1))."""
    rows = list(range(wl.B)) if batches is None else list(batches)
    x = torch.stack([_normal((wl.T, wl.C), wl.seed, V, b) for b in rows])
    f = torch.stack([torch.sigmoid(_normal((wl.T, wl.C), wl.seed, A, b, mean=3.0)) for b in rows])
    return dict(x=x.to(wl.torch_dtype), f=f.to(wl.torch_dtype))

