"""The derived bar of the normalised backward at Dv = 128 (shared by the GPU
parity test and the CPU check that the bar rejects plausible mistakes).

dq_t = S_t dn_t + dden_t z_t and dk_t = dS_t v_t + dz_t, with dn = dy / den
and dden = -(dy . y) / den, are differences of comparable terms.  At
Dv = 128 the library forms the two terms in two scans, each rounding its own
scores and state copy to bf16 relative to its own term, so the bar adds
4 u (|first| + |second|) elementwise to the relative bar (u = 2^-8 for bf16,
2^-20 for fp32), the terms' sizes taken from the float64 oracle's scans."""
import numpy as np

import oracle


def _np(x):
    return None if x is None else (x.detach().cpu().double().numpy() if hasattr(x, "detach") else np.asarray(x))


def shifted_decay(kind, lg, B, H, T):
    """The reverse scans' per-step log decay: that of the next token (0 after
    the last); None without a decay."""
    if kind == 0:
        return None
    lsh = np.broadcast_to(lg[None, :, None], (B, H, T)).copy() if kind == 1 else lg.copy()
    lsh[..., :-1] = lsh[..., 1:]
    lsh[..., -1] = 0.0
    return lsh


def terms(inp, S0, z0, dSf, dzf, dy):
    """The float64 terms: (dq1, dq2, dk1, dk2) with dq = dq1 + dq2, dk = dk1 + dk2."""
    q, k, v, g = _np(inp["q"]), _np(inp["k"]), _np(inp["v"]), _np(dy)
    kind, lg = inp["decay_kind"], _np(inp["log_g"])
    B, H, T, Dk = q.shape
    ones = np.ones((B, H, T, 1))
    n, _, _ = oracle.forward(q, k, v, kind, lg, False, _np(S0))
    den, _, _ = oracle.forward(q, k, ones, kind, lg, False, None if z0 is None else _np(z0)[..., None])
    den = den[..., 0]
    dn = g / den[..., None]
    dden = -(g * n).sum(-1) / den ** 2
    lsh = shifted_decay(kind, lg, B, H, T)
    rk = 0 if kind == 0 else 2
    sw = lambda x: None if x is None else np.swapaxes(_np(x), -1, -2)  # noqa: E731
    dq1, _, _ = oracle.forward(dn, v, k, kind, lg, False, sw(S0))
    dq2, _, _ = oracle.forward(dden[..., None], ones, k, kind, lg, False,
                               None if z0 is None else _np(z0)[:, :, None, :])
    dk1, _, _ = oracle.reverse(v, dn, q, rk, lsh, False, sw(dSf))
    dk2, _, _ = oracle.reverse(ones, dden[..., None], q, rk, lsh, False,
                               None if dzf is None else _np(dzf)[:, :, None, :])
    return dq1, dq2, dk1, dk2


def term_sizes(inp, S0, z0, dSf, dzf, dy):
    """|S_t dn_t| + |dden_t z_t| and |dS_t v_t| + |dz_t| from float64 scans."""
    dq1, dq2, dk1, dk2 = terms(inp, S0, z0, dSf, dzf, dy)
    return np.abs(dq1) + np.abs(dq2), np.abs(dk1) + np.abs(dk2)


def split_err(x, ref, sizes, tol, u):
    """max over elements of |x - ref| / (tol max|ref| + 4 u sizes), per slice."""
    x, ref = _np(x), np.asarray(ref)
    B, H = ref.shape[:2]
    worst = 0.0
    for a, r, t in zip(x.reshape(B * H, -1), ref.reshape(B * H, -1), sizes.reshape(B * H, -1)):
        worst = max(worst, float(np.max(np.abs(a - r) / (tol * np.max(np.abs(r)) + 4 * u * t))))
    return worst
