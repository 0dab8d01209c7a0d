"""GPU parity of the input prologue (la_chunk_forward_pro_ws,
la_decode_step_pro): the kernels read phi(q) * q_scale and phi(k), with
phi = elu(x) + 1 (flash-linear-attention issue 268 feeds the normalised
linear attention elu + 1 of its queries and keys, and passes q * scale).
The oracle gets the mapped inputs, computed in float64 from the same input
bits; bar as the forward: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs."""
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


def elu1(x):
    x = x.detach().cpu().double().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    return np.where(x > 0, x + 1.0, np.exp(x))


def raw(x):
    return x.detach().cpu().double().numpy()


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
def test_fp32_forward_with_feature_map_and_scale(kind, normalize):
    inp, S0, z0 = gen_case(2, 3, 77, 24, 40, dtype=torch.float32, kind=kind, normalize=False, init=True,
                           seed=5000 + kind * 2 + normalize)
    if normalize:
        z0 = torch.rand(2, 3, 24) * 4 + 0.5
    scale = 0.37
    d = to_dev(inp)
    y, S, z = la().chunk_forward(d["q"], d["k"], d["v"], kind, d["log_g"], normalize, S0.cuda(),
                                 z0.cuda() if normalize else None, feature_map=la().FEATURE_ELU1, q_scale=scale)
    torch.cuda.synchronize()
    yr, Sr, zr = oracle.forward(scale * elu1(inp["q"]), elu1(inp["k"]), inp["v"], kind, inp["log_g"], normalize,
                                S0, z0 if normalize else None)
    errs = {"y": rel_err(y, yr), "S": rel_err(S, Sr)}
    if normalize:
        errs["z"] = rel_err(z, zr)
    assert max(errs.values()) <= TOL[torch.float32], errs


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
@pytest.mark.parametrize("T", [300, 4096 + 77])
def test_bf16_forward_with_q_scale(kind, normalize, T):
    """The tensor-core path scales the unnormalised output (the normalised
    output does not depend on q's scale); long T also runs T-segments."""
    inp, S0, z0 = gen_case(1, 2, T, 64, 64, kind=kind, normalize=normalize, init=True,
                           seed=5100 + kind * 2 + normalize + T)
    scale = 64 ** -0.5
    d = to_dev(inp)
    y, S, z = la().chunk_forward(d["q"], d["k"], d["v"], kind, d["log_g"], normalize, S0.cuda(),
                                 None if z0 is None else z0.cuda(), q_scale=scale)
    torch.cuda.synchronize()
    yr, Sr, zr = oracle.forward(scale * raw(inp["q"]), inp["k"], inp["v"], kind, inp["log_g"], normalize, S0, z0)
    errs = {"y": rel_err(y, yr), "S": rel_err(S, Sr)}
    if normalize:
        errs["z"] = rel_err(z, zr)
    assert max(errs.values()) <= TOL[torch.bfloat16], errs


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("normalize", [False, True])
@pytest.mark.parametrize("T", [300, 4096 + 77])
def test_bf16_forward_with_feature_map(kind, normalize, T):
    """phi = elu + 1 on the Q and K tiles inside the tensor-core kernel (the
    raw q, k cross HBM once), with the q scale; long T also runs T-segments,
    whose state pass maps its K tiles the same way."""
    inp, S0, z0 = gen_case(1, 2, T, 64, 64, kind=kind, normalize=False, init=True,
                           seed=5300 + kind * 2 + normalize + T)
    if normalize:
        z0 = torch.rand(1, 2, 64) * 4 + 0.5
    scale = 0.37
    d = to_dev(inp)
    y, S, z = la().chunk_forward(d["q"], d["k"], d["v"], kind, d["log_g"], normalize, S0.cuda(),
                                 z0.cuda() if normalize else None, feature_map=la().FEATURE_ELU1, q_scale=scale)
    torch.cuda.synchronize()
    yr, Sr, zr = oracle.forward(scale * elu1(inp["q"]), elu1(inp["k"]), inp["v"], kind, inp["log_g"], normalize,
                                S0, z0 if normalize else None)
    errs = {"y": rel_err(y, yr), "S": rel_err(S, Sr)}
    if normalize:
        errs["z"] = rel_err(z, zr)
    assert max(errs.values()) <= TOL[torch.bfloat16], errs


@pytest.mark.parametrize("Dk,Dv", [(48, 80), (128, 128), (16, 32), (112, 64)])
def test_bf16_feature_map_widths(Dk, Dv):
    """Padded key widths: the zero columns past Dk must stay zero (phi(0) = 1)."""
    inp, S0, _ = gen_case(2, 3, 333, Dk, Dv, kind=2, normalize=False, init=True, seed=5400 + Dk + Dv)
    z0 = torch.rand(2, 3, Dk) * 4 + 0.5
    d = to_dev(inp)
    y, S, z = la().chunk_forward(d["q"], d["k"], d["v"], 2, d["log_g"], True, S0.cuda(), z0.cuda(),
                                 feature_map=la().FEATURE_ELU1)
    torch.cuda.synchronize()
    yr, Sr, zr = oracle.forward(elu1(inp["q"]), elu1(inp["k"]), inp["v"], 2, inp["log_g"], True, S0, z0)
    errs = {"y": rel_err(y, yr), "S": rel_err(S, Sr), "z": rel_err(z, zr)}
    assert max(errs.values()) <= TOL[torch.bfloat16], errs


def test_bf16_feature_map_equals_caller_side_map():
    """The normalised workload's recipe: phi in the kernel on the raw bf16
    q, k against phi applied by the caller in fp32 and rounded to bf16.  The
    kernel evaluates the exponential at the tiles' bf16 precision (argument
    and result), a bf16 rounding step or two from the fp32 value, so the
    outputs agree to about 0.3 %, far inside the bar."""
    g = torch.Generator().manual_seed(5500)
    B, H, T, D = 2, 4, 1000, 128
    q, k, v = (torch.randn(B, H, T, D, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    y1, S1, z1 = la().chunk_forward(q, k, v, normalize=True, feature_map=la().FEATURE_ELU1)
    phi = lambda x: (torch.nn.functional.elu(x.float()) + 1).to(torch.bfloat16)  # noqa: E731
    y2, S2, z2 = la().chunk_forward(phi(q), phi(k), v, normalize=True)
    torch.cuda.synchronize()
    for a, b in ((y1, y2), (S1, S2), (z1, z2)):
        assert rel_err(a, b.cpu().double().numpy()) <= 1e-2


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("normalize", [False, True])
@pytest.mark.parametrize("D", [64, 128, 40])
def test_decode_with_feature_map_and_scale(dtype, normalize, D):
    """Five tokens through the decode step with the prologue, against the
    oracle's decode on the mapped inputs (D = 40: the generic kernel)."""
    B, H = 3, 4
    g = torch.Generator().manual_seed(5200 + D + normalize)
    S = torch.randn(B, H, D, D, generator=g) * 0.1
    zz = torch.rand(B, H, D, generator=g) + 0.5
    lg = torch.log1p(-torch.rand(H, generator=g) * 0.2)
    Sd, zd = S.cuda(), zz.cuda()
    Sr, zr = S.double().numpy(), zz.double().numpy()
    scale = 0.5
    for t in range(5):
        q, k, v = (torch.randn(B, H, D, generator=g).to(dtype) for _ in range(3))
        y = la().decode_step(q.cuda(), k.cuda(), v.cuda(), Sd, zd if normalize else None, 1, lg.cuda(), normalize,
                             feature_map=la().FEATURE_ELU1, q_scale=scale)
        torch.cuda.synchronize()
        yr, Sr, zr2 = oracle.decode_step(scale * elu1(q), elu1(k), v, Sr, zr if normalize else None, 1, lg,
                                         normalize)
        if normalize:
            zr = zr2
        assert rel_err(y, yr) <= TOL[dtype], (t, rel_err(y, yr))
    assert rel_err(Sd, Sr) <= 1e-5
    if normalize:
        assert rel_err(zd, zr) <= 1e-5


def test_decode_prologue_equals_caller_side_map():
    """The fused prologue gives what a caller-side elu + 1 pass gives."""
    B, H, D = 2, 8, 128
    g = torch.Generator().manual_seed(5300)
    S0, z0 = torch.randn(B, H, D, D, generator=g) * 0.01, torch.rand(B, H, D, generator=g) + 0.1
    q, k, v = (torch.randn(B, H, D, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    Sa, za, Sb, zb = S0.cuda(), z0.cuda(), S0.cuda(), z0.cuda()
    ya = la().decode_step(q, k, v, Sa, za, 0, None, True, feature_map=la().FEATURE_ELU1)
    phi = lambda x: torch.where(x.float() > 0, x.float() + 1, torch.exp(x.float()))  # noqa: E731
    yb = la().decode_step(phi(q).contiguous(), phi(k).contiguous(), v.float().contiguous(), Sb, zb, 0, None, True)
    torch.cuda.synchronize()
    assert rel_err(ya, yb.cpu().double().numpy()) <= 2e-2
    assert rel_err(Sa, Sb.cpu().double().numpy()) <= 1e-6
