"""Pins of the oracle: checks that tie it to the pages and to mathematics, not
to itself.  Each check takes the oracle's forward / decode callables, so the
same checks run against the real oracle (test_oracle_pins.py) and against
deliberately broken copies of it (test_oracle_mutants.py).

What pins what:
  worked_examples      exact values printed on the tensortonic "CS336 L04
                       linear attention duality" page (golden fixture)
  parallel_form        the O(T^2) (Q K^T * D) V form of RetNet issue 21 via
                       numpy matmuls, all decay kinds, normaliser, carried state
  cumsum_form          g = 1: S_t is the prefix sum of k_s v_s^T (numpy cumsum)
  t1_closed_form       T = 1: y = (q.k) v + g q^T S_0
  t2_closed_form       T = 2 written out by hand
  one_hot_keys         k_t = e_{i_t}: row i of S_T is a decayed sum of v's,
                       decay written as explicit products of g's
  zero_keys            k = 0: y_t = (prod_{r<=t} g_r) q_t^T S_0
  scalar_powers        Dk = Dv = 1, constant gamma: sum of gamma^(t-s) k_s v_s
                       with integer powers
  normaliser_unity     Dv = 1, v = 1, S_0 = z_0: y = 1 exactly
  normaliser_scale     normalised output is invariant to scaling q
  split_carry          run(T) == run(T1) -> carry (S, z) -> run(T - T1)
                       (flash-linear-attention issue 268: cache and Z-state)
  ema_operator         segment summaries folded with RetNet issue 21's
                       (xa, fa) o (xb, fb) = (xa fb + xb, fa fb) in random
                       bracketings equal the full run's final state
  decode_matches       decode step == forward with T = 1; n steps == forward
                       over n tokens; page example 1 through decode
"""
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "linear_attention_duality_examples.json")
TOL = 1e-11


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} (scale {scale:.3e})"


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _log_g(rng, kind, B, H, T):
    if kind == 0:
        return None
    if kind == 1:
        return np.log(rng.uniform(0.5, 0.99, size=H))
    return np.log(rng.uniform(0.5, 1.0, size=(B, H, T)))


def _positive(rng, *shape):
    x = rng.standard_normal(shape)
    return np.where(x > 0, x + 1.0, np.exp(x))  # elu(x) + 1


# -- checks ---------------------------------------------------------------

def worked_examples(fwd, dec):
    ex = json.load(open(GOLDEN))["examples"]
    for e in ex:
        q = np.array(e["q"], np.float64)[:, None]  # (B,S,D) -> (B,1,S,D)
        k = np.array(e["k"], np.float64)[:, None]
        v = np.array(e["v"], np.float64)[:, None]
        y, S, _ = fwd(q, k, v)
        _close(y[:, 0], e["output"], 0.0, e["name"] + " output")
        _close(S[:, 0], e["final_state"], 0.0, e["name"] + " final_state")
    # example 1 token by token: the state is 6 then 36
    e = ex[0]
    q = np.array(e["q"], np.float64)[:, None]
    k = np.array(e["k"], np.float64)[:, None]
    v = np.array(e["v"], np.float64)[:, None]
    S = np.zeros((1, 1, 1, 1))
    for t, want in enumerate(e["states_after_each_token"]):
        y, S, _ = dec(q[:, :, t], k[:, :, t], v[:, :, t], S)
        _close(S.reshape(()), want, 0.0, "example 1 state after token")
        _close(y.reshape(()), np.array(e["output"]).reshape(-1)[t], 0.0, "example 1 decode output")


def parallel_form(fwd, dec, parallel):
    rng = np.random.default_rng(11)
    for kind in (0, 1, 2):
        for normalize in (False, True):
            for with_init in (False, True):
                B, H, T, Dk, Dv = 2, 3, 37, 5, 4
                if normalize:
                    q, k = _positive(rng, B, H, T, Dk), _positive(rng, B, H, T, Dk)
                else:
                    q, k = _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dk)
                v = _rand(rng, B, H, T, Dv)
                lg = _log_g(rng, kind, B, H, T)
                S0 = _rand(rng, B, H, Dk, Dv) if with_init else None
                z0 = np.abs(_rand(rng, B, H, Dk)) if (with_init and normalize) else None
                y, S, z = fwd(q, k, v, kind, lg, normalize, S0, z0)
                yp, Sp, zp = parallel(q, k, v, kind, lg, normalize, S0, z0)
                tag = f"kind={kind} norm={normalize} init={with_init}"
                _close(y, yp, 1e-10, "parallel y " + tag)
                _close(S, Sp, 1e-10, "parallel S " + tag)
                if normalize:
                    _close(z, zp, 1e-10, "parallel z " + tag)


def cumsum_form(fwd, dec):
    rng = np.random.default_rng(12)
    B, H, T, Dk, Dv = 1, 2, 23, 3, 4
    q, k, v = _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dv)
    y, S, _ = fwd(q, k, v)
    outer = k[..., :, None] * v[..., None, :]          # [B,H,T,Dk,Dv]
    states = np.cumsum(outer, axis=2)
    _close(y, np.einsum("bhti,bhtij->bhtj", q, states), TOL, "cumsum y")
    _close(S, states[:, :, -1], TOL, "cumsum final state")


def t1_closed_form(fwd, dec):
    rng = np.random.default_rng(13)
    Dk, Dv = 4, 3
    q, k, v = _rand(rng, 1, 1, 1, Dk), _rand(rng, 1, 1, 1, Dk), _rand(rng, 1, 1, 1, Dv)
    S0 = _rand(rng, 1, 1, Dk, Dv)
    g = 0.7
    y, S, _ = fwd(q, k, v, 1, np.array([np.log(g)]), False, S0)
    qv, kv, vv, S0v = q[0, 0, 0], k[0, 0, 0], v[0, 0, 0], S0[0, 0]
    _close(y[0, 0, 0], (qv @ kv) * vv + g * (qv @ S0v), TOL, "T=1 output")
    _close(S[0, 0], g * S0v + np.outer(kv, vv), TOL, "T=1 state")


def t2_closed_form(fwd, dec):
    rng = np.random.default_rng(14)
    Dk, Dv = 3, 2
    q, k, v = _rand(rng, 1, 1, 2, Dk), _rand(rng, 1, 1, 2, Dk), _rand(rng, 1, 1, 2, Dv)
    S0 = _rand(rng, 1, 1, Dk, Dv)
    z0 = np.abs(_rand(rng, 1, 1, Dk))
    g1, g2 = 0.9, 0.6
    lg = np.log(np.array([g1, g2]))[None, None]
    q1, q2 = q[0, 0]
    k1, k2 = k[0, 0]
    v1, v2 = v[0, 0]
    S0v, z0v = S0[0, 0], z0[0, 0]
    y, S, _ = fwd(q, k, v, 2, lg, False, S0)
    y1 = g1 * (q1 @ S0v) + (q1 @ k1) * v1
    y2 = g1 * g2 * (q2 @ S0v) + g2 * (q2 @ k1) * v1 + (q2 @ k2) * v2
    _close(y[0, 0, 0], y1, TOL, "T=2 y1")
    _close(y[0, 0, 1], y2, TOL, "T=2 y2")
    _close(S[0, 0], g1 * g2 * S0v + g2 * np.outer(k1, v1) + np.outer(k2, v2), TOL, "T=2 state")
    qp, kp = np.abs(q) + 0.1, np.abs(k) + 0.1
    q1, q2 = qp[0, 0]
    k1, k2 = kp[0, 0]
    y, S, z = fwd(qp, kp, v, 2, lg, True, S0, z0)
    d2 = g1 * g2 * (q2 @ z0v) + g2 * (q2 @ k1) + (q2 @ k2)
    n2 = g1 * g2 * (q2 @ S0v) + g2 * (q2 @ k1) * v1 + (q2 @ k2) * v2
    _close(y[0, 0, 1], n2 / d2, TOL, "T=2 normalised y2")
    _close(z[0, 0], g1 * g2 * z0v + g2 * k1 + k2, TOL, "T=2 key sum")


def one_hot_keys(fwd, dec):
    rng = np.random.default_rng(15)
    T, Dk, Dv = 17, 4, 3
    idx = rng.integers(0, Dk, size=T)
    k = np.zeros((1, 1, T, Dk))
    k[0, 0, np.arange(T), idx] = 1.0
    q, v = _rand(rng, 1, 1, T, Dk), _rand(rng, 1, 1, T, Dv)
    g = rng.uniform(0.5, 1.0, size=T)
    y, S, _ = fwd(q, k, v, 2, np.log(g)[None, None])
    want = np.zeros((Dk, Dv))
    for t in range(T):
        want[idx[t]] += np.prod(g[t + 1:]) * v[0, 0, t]
    _close(S[0, 0], want, TOL, "one-hot keys state")


def zero_keys(fwd, dec):
    rng = np.random.default_rng(16)
    T, Dk, Dv = 9, 3, 5
    q, v = _rand(rng, 1, 1, T, Dk), _rand(rng, 1, 1, T, Dv)
    k = np.zeros((1, 1, T, Dk))
    S0 = _rand(rng, 1, 1, Dk, Dv)
    g = rng.uniform(0.3, 1.0, size=T)
    y, S, _ = fwd(q, k, v, 2, np.log(g)[None, None], False, S0)
    for t in range(T):
        _close(y[0, 0, t], np.prod(g[:t + 1]) * (q[0, 0, t] @ S0[0, 0]), TOL, "zero keys y")


def scalar_powers(fwd, dec):
    rng = np.random.default_rng(17)
    T, gamma = 25, 0.85
    q, k, v = _rand(rng, 1, 1, T, 1), _rand(rng, 1, 1, T, 1), _rand(rng, 1, 1, T, 1)
    S0 = _rand(rng, 1, 1, 1, 1)
    y, S, _ = fwd(q, k, v, 1, np.array([np.log(gamma)]), False, S0)
    kk, vv, qq, s0 = k[0, 0, :, 0], v[0, 0, :, 0], q[0, 0, :, 0], S0.item()
    for t in range(T):
        st = sum(gamma ** (t - s) * kk[s] * vv[s] for s in range(t + 1)) + gamma ** (t + 1) * s0
        _close(y[0, 0, t, 0], qq[t] * st, TOL, "scalar EMA y")


def normaliser_unity(fwd, dec):
    rng = np.random.default_rng(18)
    for kind in (0, 1, 2):
        B, H, T, Dk = 1, 2, 31, 6
        q, k = _positive(rng, B, H, T, Dk), _positive(rng, B, H, T, Dk)
        v = np.ones((B, H, T, 1))
        z0 = np.abs(_rand(rng, B, H, Dk))
        lg = _log_g(rng, kind, B, H, T)
        y, S, z = fwd(q, k, v, kind, lg, True, z0[..., None], z0)
        _close(y, np.ones_like(y), 1e-13, f"v=1 gives y=1 (kind {kind})")
        _close(S[..., 0], z, 1e-13, f"v=1 state equals key sum (kind {kind})")


def normaliser_scale(fwd, dec):
    rng = np.random.default_rng(19)
    B, H, T, Dk, Dv = 1, 2, 13, 4, 3
    q, k, v = _positive(rng, B, H, T, Dk), _positive(rng, B, H, T, Dk), _rand(rng, B, H, T, Dv)
    y1, _, _ = fwd(q, k, v, 0, None, True)
    y2, _, _ = fwd(q * 8.0, k, v, 0, None, True)
    _close(y1, y2, 1e-13, "normalised output invariant to q scale")
    y3, _, _ = fwd(q, k, v, 0, None, False)
    assert np.max(np.abs(y3 - y1)) > 1e-3, "normalize flag has no effect"


def split_carry(fwd, dec):
    rng = np.random.default_rng(20)
    for kind in (0, 1, 2):
        for normalize in (False, True):
            B, H, T, Dk, Dv, T1 = 2, 2, 29, 4, 3, 11
            q, k = _positive(rng, B, H, T, Dk), _positive(rng, B, H, T, Dk)
            v = _rand(rng, B, H, T, Dv)
            lg = _log_g(rng, kind, B, H, T)
            lg1 = lg[..., :T1] if kind == 2 else lg
            lg2 = lg[..., T1:] if kind == 2 else lg
            y, S, z = fwd(q, k, v, kind, lg, normalize)
            ya, Sa, za = fwd(q[:, :, :T1], k[:, :, :T1], v[:, :, :T1], kind, lg1, normalize)
            yb, Sb, zb = fwd(q[:, :, T1:], k[:, :, T1:], v[:, :, T1:], kind, lg2, normalize, Sa, za)
            tag = f"kind={kind} norm={normalize}"
            _close(np.concatenate([ya, yb], axis=2), y, 1e-12, "split y " + tag)
            _close(Sb, S, 1e-12, "split S " + tag)
            if normalize:
                _close(zb, z, 1e-12, "split z " + tag)


def ema_operator(fwd, dec):
    rng = np.random.default_rng(21)
    T, Dk, Dv, nseg = 40, 3, 2, 5
    q, k, v = _rand(rng, 1, 1, T, Dk), _rand(rng, 1, 1, T, Dk), _rand(rng, 1, 1, T, Dv)
    lg = np.log(rng.uniform(0.6, 1.0, size=(1, 1, T)))
    _, S_full, _ = fwd(q, k, v, 2, lg)
    cuts = np.sort(rng.choice(np.arange(1, T), size=nseg - 1, replace=False))
    bounds = [0, *cuts.tolist(), T]
    segs = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        _, Sx, _ = fwd(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], 2, lg[..., a:b])
        segs.append((Sx[0, 0], float(np.exp(lg[0, 0, a:b].sum()))))

    def op(x, y):  # (xa, fa) o (xb, fb) = (xa * fb + xb, fa * fb)
        return (x[0] * y[1] + y[0], x[1] * y[1])

    def fold(items):  # a random bracketing of the ordered sequence
        if len(items) == 1:
            return items[0]
        m = int(rng.integers(1, len(items)))
        return op(fold(items[:m]), fold(items[m:]))

    for _ in range(4):
        Sx, _ = fold(segs)
        _close(Sx, S_full[0, 0], 1e-12, "EMA operator bracketing")


def decode_matches(fwd, dec):
    rng = np.random.default_rng(22)
    for kind in (0, 1, 2):
        for normalize in (False, True):
            B, H, n, Dk, Dv = 2, 3, 7, 4, 5
            q, k = _positive(rng, B, H, n, Dk), _positive(rng, B, H, n, Dk)
            v = _rand(rng, B, H, n, Dv)
            S0 = _rand(rng, B, H, Dk, Dv)
            z0 = np.abs(_rand(rng, B, H, Dk)) if normalize else None
            lg = _log_g(rng, kind, B, H, n)
            y, S, z = fwd(q, k, v, kind, lg, normalize, S0, z0)
            St, zt = S0, z0
            for t in range(n):
                lgt = lg[..., t] if kind == 2 else lg
                yt, St, zt = dec(q[:, :, t], k[:, :, t], v[:, :, t], St, zt, kind, lgt, normalize)
                _close(yt, y[:, :, t], 1e-12, f"decode step {t} kind={kind} norm={normalize}")
            _close(St, S, 1e-12, "decode final state")
            if normalize:
                _close(zt, z, 1e-12, "decode final key sum")


ALL = [worked_examples, cumsum_form, t1_closed_form, t2_closed_form, one_hot_keys,
       zero_keys, scalar_powers, normaliser_unity, normaliser_scale, split_carry,
       ema_operator, decode_matches]


# -- reverse scan (S_t = g_t S_{t+1} + k_t v_t^T) and bidirectional sum -----

def reverse_parallel_form(rev, parallel_rev):
    rng = np.random.default_rng(31)
    for kind in (0, 1, 2):
        for normalize in (False, True):
            for with_init in (False, True):
                B, H, T, Dk, Dv = 2, 2, 29, 4, 3
                if normalize:
                    q, k = _positive(rng, B, H, T, Dk), _positive(rng, B, H, T, Dk)
                else:
                    q, k = _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dk)
                v = _rand(rng, B, H, T, Dv)
                lg = _log_g(rng, kind, B, H, T)
                S0 = _rand(rng, B, H, Dk, Dv) if with_init else None
                z0 = np.abs(_rand(rng, B, H, Dk)) if (with_init and normalize) else None
                y, S, z = rev(q, k, v, kind, lg, normalize, S0, z0)
                yp, Sp, zp = parallel_rev(q, k, v, kind, lg, normalize, S0, z0)
                tag = f"reverse kind={kind} norm={normalize} init={with_init}"
                _close(y, yp, 1e-10, "y " + tag)
                _close(S, Sp, 1e-10, "S " + tag)
                if normalize:
                    _close(z, zp, 1e-10, "z " + tag)


def reverse_cumsum_form(rev):
    # g = 1: the state at t is the suffix sum of k_s v_s^T
    rng = np.random.default_rng(32)
    B, H, T, Dk, Dv = 1, 2, 19, 3, 4
    q, k, v = _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dv)
    y, S, _ = rev(q, k, v)
    outer = k[..., :, None] * v[..., None, :]
    states = np.flip(np.cumsum(np.flip(outer, 2), axis=2), 2)
    _close(y, np.einsum("bhti,bhtij->bhtj", q, states), TOL, "reverse cumsum y")
    _close(S, states[:, :, 0], TOL, "reverse cumsum state at token 1")


def reverse_t2_closed_form(rev):
    # T = 2, per-step g: S_2 = g_2 S0 + k_2 v_2^T, S_1 = g_1 S_2 + k_1 v_1^T
    rng = np.random.default_rng(33)
    Dk, Dv = 3, 2
    q, k, v = _rand(rng, 1, 1, 2, Dk), _rand(rng, 1, 1, 2, Dk), _rand(rng, 1, 1, 2, Dv)
    S0 = _rand(rng, 1, 1, Dk, Dv)
    g = np.array([0.6, 0.8])
    y, S, _ = rev(q, k, v, 2, np.log(g)[None, None, :], False, S0)
    q1, q2, k1, k2, v1, v2, S0v = q[0, 0, 0], q[0, 0, 1], k[0, 0, 0], k[0, 0, 1], v[0, 0, 0], v[0, 0, 1], S0[0, 0]
    S2 = g[1] * S0v + np.outer(k2, v2)
    S1 = g[0] * S2 + np.outer(k1, v1)
    _close(y[0, 0, 1], q2 @ S2, TOL, "reverse T=2 y_2")
    _close(y[0, 0, 0], q1 @ S1, TOL, "reverse T=2 y_1")
    _close(S[0, 0], S1, TOL, "reverse T=2 state at token 1")


def bidirectional_closed_form(bi):
    # g = 1: forward counts s <= t and reverse s >= t, so their sum is
    # (Q K^T) V plus the diagonal term (q_t . k_t) v_t once more
    rng = np.random.default_rng(34)
    B, H, T, Dk, Dv = 1, 2, 17, 3, 4
    q, k, v = _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dv)
    y = bi(q, k, v)
    A = np.einsum("bhti,bhsi->bhts", q, k)
    diag = np.einsum("bhti,bhti->bht", q, k)[..., None] * v
    _close(y, A @ v + diag, TOL, "bidirectional g=1")


# -- backward: gradients of L = sum dy . y + <dS_T, S_T> + <dz_T, z_T> -------
#
#   backward_finite_differences  central differences of L through the
#                                (pinned) forward, every input, all decay kinds,
#                                normaliser and carried state
#   backward_t1_closed_form      T = 1 differentiated by hand
#   backward_parallel_form       g-weighted matrices: dQ = (dY V^T o M) K,
#                                dK = (dY V^T o M)^T Q, dV = (Q K^T o M)^T dY
#                                with M_ts = G_t / G_s (s <= t); the decay
#                                gradient as the suffix sum of
#                                q_t . dq_t - k_t . dk_t (plus <S_T, dS_T> at T)

def _loss(fwd, normalize, dy, dST, dzT):
    def L(q, k, v, kind, lg, S0, z0):
        y, S, z = fwd(q, k, v, kind, lg, normalize, S0, z0)
        r = float(np.sum(y * dy)) + float(np.sum(S * dST))
        if normalize:
            r += float(np.sum(z * dzT))
        return r
    return L


def backward_finite_differences(bwd, fwd):
    rng = np.random.default_rng(41)
    h = 1e-6
    for kind in (0, 1, 2):
        for normalize in (False, True):
            for with_init in (False, True):
                B, H, T, Dk, Dv = 1, 2, 7, 3, 4
                if normalize:
                    q, k = _positive(rng, B, H, T, Dk), _positive(rng, B, H, T, Dk)
                else:
                    q, k = _rand(rng, B, H, T, Dk), _rand(rng, B, H, T, Dk)
                v = _rand(rng, B, H, T, Dv)
                lg = _log_g(rng, kind, B, H, T)
                S0 = _rand(rng, B, H, Dk, Dv) if with_init else None
                z0 = np.abs(_rand(rng, B, H, Dk)) + 0.5 if (with_init and normalize) else None
                dy, dST = _rand(rng, B, H, T, Dv), _rand(rng, B, H, Dk, Dv)
                dzT = _rand(rng, B, H, Dk) if normalize else None
                L = _loss(fwd, normalize, dy, dST, dzT)
                grads = bwd(q, k, v, dy, kind, lg, normalize, S0, z0, dST, dzT)
                args = {"q": q, "k": k, "v": v, "lg": lg, "S0": S0, "z0": z0}
                slot = {"q": 0, "k": 1, "v": 2, "lg": 3, "S0": 4, "z0": 5}
                tag = f"kind={kind} norm={normalize} init={with_init}"
                for name, x in args.items():
                    if x is None:
                        continue
                    flat = x.reshape(-1)
                    for idx in rng.choice(flat.size, size=min(flat.size, 6), replace=False):
                        a = dict(args)
                        xp, xm = x.copy(), x.copy()
                        xp.reshape(-1)[idx] += h
                        xm.reshape(-1)[idx] -= h
                        a[name] = xp
                        lp = L(a["q"], a["k"], a["v"], kind, a["lg"], a["S0"], a["z0"])
                        a[name] = xm
                        lm = L(a["q"], a["k"], a["v"], kind, a["lg"], a["S0"], a["z0"])
                        fd = (lp - lm) / (2 * h)
                        got = np.asarray(grads[slot[name]]).reshape(-1)[idx]
                        assert abs(got - fd) <= 1e-6 * max(1.0, abs(fd)), \
                            f"d{name}[{idx}] {tag}: {got} vs finite difference {fd}"


def backward_t1_closed_form(bwd):
    # y = g q^T S0 + (q.k) v,  S_1 = g S0 + k v^T,  L = dy.y + <dS, S_1>
    rng = np.random.default_rng(42)
    Dk, Dv = 3, 4
    q, k, v, dy = _rand(rng, Dk), _rand(rng, Dk), _rand(rng, Dv), _rand(rng, Dv)
    S0, dS = _rand(rng, Dk, Dv), _rand(rng, Dk, Dv)
    g = 0.7
    sh = lambda x: x[None, None, None]  # noqa: E731
    dq, dk, dv, dlg, dS0, _ = bwd(sh(q), sh(k), sh(v), sh(dy), 2, np.full((1, 1, 1), np.log(g)), False,
                                  S0[None, None], None, dS[None, None], None)
    _close(dq[0, 0, 0], g * S0 @ dy + k * (v @ dy), TOL, "T=1 dq")
    _close(dk[0, 0, 0], q * (v @ dy) + dS @ v, TOL, "T=1 dk")
    _close(dv[0, 0, 0], (q @ k) * dy + dS.T @ k, TOL, "T=1 dv")
    _close(dS0[0, 0], g * (np.outer(q, dy) + dS), TOL, "T=1 dS0")
    _close(dlg[0, 0, 0], g * (q @ S0 @ dy + np.sum(S0 * dS)), TOL, "T=1 dlog g")


def backward_parallel_form(bwd, fwd):
    rng = np.random.default_rng(43)
    for kind in (0, 1, 2):
        for with_init in (False, True):
            B, H, T, Dk, Dv = 2, 2, 23, 4, 3
            q, k, v, dy = (_rand(rng, B, H, T, D) for D in (Dk, Dk, Dv, Dv))
            lg = _log_g(rng, kind, B, H, T)
            S0 = _rand(rng, B, H, Dk, Dv) if with_init else np.zeros((B, H, Dk, Dv))
            dST = _rand(rng, B, H, Dk, Dv)
            dq, dk, dv, dlg, dS0, _ = bwd(q, k, v, dy, kind, lg, False, S0 if with_init else None, None,
                                          dST, None)
            _, ST, _ = fwd(q, k, v, kind, lg, False, S0 if with_init else None, None)
            tag = f"kind={kind} init={with_init}"
            dA_all = np.zeros((B, H, T))
            for b in range(B):
                for hh in range(H):
                    a = np.zeros(T) if kind == 0 else (np.full(T, lg[hh]) if kind == 1 else lg[b, hh])
                    A = np.cumsum(a)                      # log of G_t = g_1 ... g_t
                    M = np.tril(np.exp(A[:, None] - A[None, :]))
                    Q, K, V, dY = q[b, hh], k[b, hh], v[b, hh], dy[b, hh]
                    GT = np.exp(A[-1] - A)                # G_T / G_s
                    eq = (dY @ V.T * M) @ K + np.exp(A)[:, None] * (dY @ S0[b, hh].T)
                    ek = (dY @ V.T * M).T @ Q + GT[:, None] * (V @ dST[b, hh].T)
                    ev = (Q @ K.T * M).T @ dY + GT[:, None] * (K @ dST[b, hh])
                    _close(dq[b, hh], eq, 1e-10, "parallel dq " + tag)
                    _close(dk[b, hh], ek, 1e-10, "parallel dk " + tag)
                    _close(dv[b, hh], ev, 1e-10, "parallel dv " + tag)
                    dS1 = (np.exp(A)[:, None] * Q).T @ dY + np.exp(A[-1]) * dST[b, hh]
                    _close(dS0[b, hh], dS1, 1e-10, "parallel dS0 " + tag)
                    dA = np.sum(Q * eq, axis=1) - np.sum(K * ek, axis=1)
                    dA[-1] += np.sum(ST[b, hh] * dST[b, hh])
                    dA_all[b, hh] = np.flip(np.cumsum(np.flip(dA)))
            if kind == 1:
                _close(dlg, dA_all.sum(axis=(0, 2)), 1e-9, "parallel dlog g " + tag)
            elif kind == 2:
                _close(dlg, dA_all, 1e-9, "parallel dlog g " + tag)



# -- RWKV-4 WKV (BlinkDL/RWKV-LM issue 167, formula 14) ----------------------
#
#   wkv4_direct_form   the online weighted mean against the definition written
#                      out (O(T^2), numpy exponentials), with and without a
#                      carried state
#   wkv4_t1_t2         T = 1: out = v; T = 2 expanded by hand
#   wkv4_invariants    constant v gives constant out; adding s to every key
#                      leaves out and (aa, bb) unchanged and moves pp by s
#   wkv4_split_carry   run(T) == run(T1) -> carry (aa, bb, pp) -> run(T - T1)
#   wkv4_large_keys    keys near 300 (e^300 overflows fp32) and near -800
#                      (e^-800 underflows f64): the loop stays finite and
#                      exact, equal to the definition on the keys shifted
#                      back (the ratio ignores the shift)
#   wkv4_no_bonus      u = -1e30: out_t (t >= 1) is the decayed average of the
#                      earlier values only

def _wkv4_inputs(rng, B, T, C, init=False, kshift=0.0):
    k = rng.standard_normal((B, T, C)) + kshift
    v = rng.standard_normal((B, T, C))
    w = -np.exp(rng.standard_normal(C) - 0.5)
    u = rng.standard_normal(C) - 0.5
    S0 = None
    if init:
        S0 = np.stack([rng.standard_normal((B, C)), np.abs(rng.standard_normal((B, C))) + 0.1,
                       rng.standard_normal((B, C)) + kshift], axis=1)
    return k, v, w, u, S0


def wkv4_direct_form(wkv, direct):
    rng = np.random.default_rng(51)
    for init in (False, True):
        for T in (1, 2, 3, 17, 40):
            k, v, w, u, S0 = _wkv4_inputs(rng, 2, T, 5, init)
            out, _ = wkv(k, v, w, u, S0)
            _close(out, direct(k, v, w, u, S0), 1e-12, f"direct form T={T} init={init}")


def wkv4_t1_t2(wkv, direct):
    rng = np.random.default_rng(52)
    k, v, w, u, _ = _wkv4_inputs(rng, 1, 2, 3)
    out, fin = wkv(k[:, :1], v[:, :1], w, u)
    _close(out, v[:, :1], 1e-15, "T=1 out = v")
    _close(fin[:, 0] * np.exp(fin[:, 2]), np.exp(k[:, 0]) * v[:, 0], 1e-12, "T=1 state numerator")
    _close(fin[:, 1] * np.exp(fin[:, 2]), np.exp(k[:, 0]), 1e-12, "T=1 state denominator")
    out, _ = wkv(k, v, w, u)
    a, b = np.exp(k[0, 0]), np.exp(u + k[0, 1])
    _close(out[0, 1], (a * v[0, 0] + b * v[0, 1]) / (a + b), 1e-12, "T=2 by hand")


def wkv4_invariants(wkv, direct):
    rng = np.random.default_rng(53)
    k, v, w, u, _ = _wkv4_inputs(rng, 2, 30, 4)
    out, _ = wkv(k, np.full_like(v, 1.75), w, u)
    _close(out, np.full_like(v, 1.75), 1e-13, "constant v")
    o1, f1 = wkv(k, v, w, u)
    o2, f2 = wkv(k + 3.25, v, w, u)
    _close(o2, o1, 1e-12, "key shift: out")
    _close(f2[:, :2], f1[:, :2], 1e-12, "key shift: aa, bb")
    _close(f2[:, 2], f1[:, 2] + 3.25, 1e-12, "key shift: pp")


def wkv4_split_carry(wkv, direct):
    rng = np.random.default_rng(54)
    k, v, w, u, S0 = _wkv4_inputs(rng, 2, 33, 6, init=True)
    full, ffin = wkv(k, v, w, u, S0)
    for T1 in (1, 10, 32):
        a, fa = wkv(k[:, :T1], v[:, :T1], w, u, S0)
        b, fb = wkv(k[:, T1:], v[:, T1:], w, u, fa)
        _close(np.concatenate([a, b], axis=1), full, 1e-12, f"split at {T1}: out")
        _close(fb, ffin, 1e-12, f"split at {T1}: state")


def wkv4_large_keys(wkv, direct):
    rng = np.random.default_rng(55)
    for shift in (300.0, -800.0):
        k, v, w, u, _ = _wkv4_inputs(rng, 2, 25, 4, kshift=shift)
        out, fin = wkv(k, v, w, u)
        assert np.all(np.isfinite(out)) and np.all(np.isfinite(fin)), f"keys near {shift}: non-finite values"
        _close(out, direct(k - shift, v, w, u), 1e-12, f"keys near {shift}")


def wkv4_no_bonus(wkv, direct):
    rng = np.random.default_rng(56)
    k, v, w, u, _ = _wkv4_inputs(rng, 1, 12, 3)
    u = np.full_like(u, -1e30)
    out, _ = wkv(k, v, w, u)
    for t in range(1, 12):
        wt = np.exp((t - 1 - np.arange(t))[:, None] * w[None, :] + k[0, :t])
        _close(out[0, t], (wt * v[0, :t]).sum(0) / wt.sum(0), 1e-12, f"no bonus t={t}")


WKV4 = [wkv4_direct_form, wkv4_t1_t2, wkv4_invariants, wkv4_split_carry, wkv4_large_keys, wkv4_no_bonus]


# -- cumulative EMA (RetNet issue 21, cumulative_ema) -------------------------
#
#   ema_constant_factor  f = gamma everywhere: out_t = sum_i gamma^(t-i) x_i
#                        + gamma^(t+1) s0 with integer powers
#   ema_cumsum           f = 1: numpy cumsum;  f = 0: out = x
#   ema_operator         segment summaries (state from 0, product of
#                        factors) folded with (xa, fa) o (xb, fb) =
#                        (xa fb + xb, fa fb) in random bracketings equal the
#                        full run's final state
#   ema_reverse          reverse == flip(forward(flip(x), flip(f)))
#   ema_split_carry      run(T) == run(T1) -> carry -> run(T - T1)

def _ema_inputs(rng, B, T, C):
    return rng.standard_normal((B, T, C)), rng.uniform(0.3, 1.0, (B, T, C)), rng.standard_normal((B, C))


def ema_constant_factor(ema):
    rng = np.random.default_rng(71)
    x, _, s0 = _ema_inputs(rng, 2, 19, 3)
    g = 0.83
    out, fin = ema(x, np.full_like(x, g), s0)
    t = np.arange(19)
    P = np.tril(g ** (t[:, None] - t[None, :]).clip(min=0)) * (t[:, None] >= t[None, :])
    want = np.einsum("ts,bsc->btc", P, x) + (g ** (t + 1))[None, :, None] * s0[:, None, :]
    _close(out, want, 1e-12, "constant factor")
    _close(fin, want[:, -1], 1e-12, "constant factor final")


def ema_cumsum(ema):
    rng = np.random.default_rng(72)
    x, _, _ = _ema_inputs(rng, 2, 23, 4)
    out, _ = ema(x, np.ones_like(x))
    _close(out, np.cumsum(x, axis=1), 1e-12, "f = 1 is a cumsum")
    out, _ = ema(x, np.zeros_like(x))
    _close(out, x, 0.0, "f = 0 is the identity")


def ema_operator(ema):
    rng = np.random.default_rng(73)
    x, f, _ = _ema_inputs(rng, 1, 40, 2)
    _, full = ema(x, f)
    cuts = np.sort(rng.choice(np.arange(1, 40), size=5, replace=False))
    spans = np.split(np.arange(40), cuts)
    items = []
    for sp in spans:
        _, fin = ema(x[:, sp], f[:, sp])
        items.append((fin, np.prod(f[:, sp], axis=1)))

    def op(a, b):  # RetNet issue 21's pairing of (value, factor)
        return a[0] * b[1] + b[0], a[1] * b[1]

    for trial in range(6):
        seq = list(items)
        while len(seq) > 1:  # a random bracketing
            j = rng.integers(0, len(seq) - 1)
            seq[j:j + 2] = [op(seq[j], seq[j + 1])]
        _close(seq[0][0], full, 1e-12, f"bracketing {trial}")


def ema_reverse(ema):
    rng = np.random.default_rng(74)
    x, f, s0 = _ema_inputs(rng, 2, 17, 3)
    out, fin = ema(x, f, s0, reverse=True)
    o2, f2 = ema(x[:, ::-1].copy(), f[:, ::-1].copy(), s0)
    _close(out, o2[:, ::-1], 1e-12, "reverse = flip forward flip")
    _close(fin, f2, 1e-12, "reverse final state")


def ema_split_carry(ema):
    rng = np.random.default_rng(75)
    x, f, s0 = _ema_inputs(rng, 2, 31, 3)
    for rev in (False, True):
        full, ffin = ema(x, f, s0, reverse=rev)
        for T1 in (1, 12, 30):
            if not rev:
                a, fa = ema(x[:, :T1], f[:, :T1], s0)
                b, fb = ema(x[:, T1:], f[:, T1:], fa)
                got = np.concatenate([a, b], axis=1)
            else:
                b, fb0 = ema(x[:, T1:], f[:, T1:], s0, reverse=True)
                a, fb = ema(x[:, :T1], f[:, :T1], fb0, reverse=True)
                got = np.concatenate([a, b], axis=1)
            _close(got, full, 1e-12, f"split at {T1} reverse={rev}")
            _close(fb, ffin, 1e-12, f"split at {T1} reverse={rev}: state")


EMA = [ema_constant_factor, ema_cumsum, ema_operator, ema_reverse, ema_split_carry]
