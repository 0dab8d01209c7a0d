"""The oracle against its pins (CPU only)."""
import functools

import numpy as np
import pytest

import oracle
import oracle_pins as pins


def _fwd(*a, **kw):
    return oracle.forward(*a, nthreads=2, **kw)


@pytest.mark.parametrize("check", pins.ALL, ids=lambda f: f.__name__)
def test_recurrent_oracle(oracle_lib, check):
    check(_fwd, oracle.decode_step)


def test_recurrent_matches_parallel_form(oracle_lib):
    pins.parallel_form(_fwd, oracle.decode_step, oracle.parallel_forward)


# The parallel form is itself pinned by the checks that need no decode step.
@pytest.mark.parametrize("check", [pins.cumsum_form, pins.t1_closed_form, pins.t2_closed_form,
                                   pins.one_hot_keys, pins.zero_keys, pins.scalar_powers,
                                   pins.normaliser_unity, pins.split_carry],
                         ids=lambda f: f.__name__)
def test_parallel_form(check):
    check(oracle.parallel_forward, None)


def test_parallel_form_worked_examples():
    import json
    for e in json.load(open(pins.GOLDEN))["examples"]:
        q = np.array(e["q"], np.float64)[:, None]
        k = np.array(e["k"], np.float64)[:, None]
        v = np.array(e["v"], np.float64)[:, None]
        y, S, _ = oracle.parallel_forward(q, k, v)
        assert np.array_equal(y[:, 0], np.array(e["output"], np.float64))
        assert np.array_equal(S[:, 0], np.array(e["final_state"], np.float64))


def test_threads_do_not_change_results(oracle_lib):
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((3, 5, 19, 4)) for _ in range(3))
    lg = np.log(rng.uniform(0.5, 1, size=(3, 5, 19)))
    a = oracle.forward(q, k, v, 2, lg, nthreads=1)
    b = oracle.forward(q, k, v, 2, lg, nthreads=7)
    for x, y in zip(a[:2], b[:2]):
        assert np.array_equal(x, y)


def test_empty_sequence(oracle_lib):
    rng = np.random.default_rng(4)
    S0 = rng.standard_normal((2, 3, 4, 5))
    z0 = np.abs(rng.standard_normal((2, 3, 4)))
    q = np.zeros((2, 3, 0, 4))
    v = np.zeros((2, 3, 0, 5))
    y, S, z = oracle.forward(q, q, v, 0, None, True, S0, z0)
    assert y.shape == (2, 3, 0, 5)
    assert np.array_equal(S, S0) and np.array_equal(z, z0)


def test_rejects_bad_arguments(oracle_lib):
    q = np.zeros((1, 1, 2, 2))
    with pytest.raises(ValueError):
        oracle.forward(q, q, q, 3, np.zeros(1))
    with pytest.raises(ValueError):
        oracle.forward(q, q, q, 1, None)


# ---------------------------------------------------------------- reverse scan
def _rev(*a, **kw):
    return oracle.reverse(*a, nthreads=2, **kw)


def test_reverse_matches_anticausal_form(oracle_lib):
    pins.reverse_parallel_form(_rev, oracle.parallel_reverse)


@pytest.mark.parametrize("check", [pins.reverse_cumsum_form, pins.reverse_t2_closed_form],
                         ids=lambda f: f.__name__)
def test_reverse_closed_forms(oracle_lib, check):
    check(_rev)          # the recurrent reverse (forward of the time-reversed arguments)
    check(oracle.parallel_reverse)  # and the independent anti-causal form


def test_bidirectional_closed_form(oracle_lib):
    pins.bidirectional_closed_form(lambda q, k, v: oracle.bidirectional(q, k, v, nthreads=2))


# ---------------------------------------------------------------- backward
def _bwd(*a, **kw):
    return oracle.backward(*a, nthreads=2, **kw)


def test_backward_matches_finite_differences(oracle_lib):
    pins.backward_finite_differences(_bwd, _fwd)


def test_backward_t1_closed_form(oracle_lib):
    pins.backward_t1_closed_form(_bwd)


def test_backward_matches_parallel_form(oracle_lib):
    pins.backward_parallel_form(_bwd, _fwd)


def test_backward_empty_sequence(oracle_lib):
    rng = np.random.default_rng(5)
    dST = rng.standard_normal((1, 2, 3, 4))
    q = np.zeros((1, 2, 0, 3))
    v = np.zeros((1, 2, 0, 4))
    dq, dk, dv, dlg, dS0, _ = oracle.backward(q, q, v, v, 2, np.zeros((1, 2, 0)), False, None, None, dST)
    assert dq.shape == (1, 2, 0, 3) and dv.shape == (1, 2, 0, 4) and dlg.shape == (1, 2, 0)
    assert np.array_equal(dS0, dST)


@pytest.mark.parametrize("check", pins.WKV4, ids=lambda f: f.__name__)
def test_wkv4_oracle(oracle_lib, check):
    check(oracle.wkv4, oracle.wkv4_direct)


def test_wkv4_direct_form_by_brute_force():
    """The numpy definition itself, against a scalar loop over (t, i)."""
    import math
    rng = np.random.default_rng(57)
    B, T, C = 1, 6, 2
    k, v = rng.standard_normal((B, T, C)), rng.standard_normal((B, T, C))
    w, u = -np.exp(rng.standard_normal(C)), rng.standard_normal(C)
    d = oracle.wkv4_direct(k, v, w, u)
    for c in range(C):
        for t in range(T):
            num = math.exp(u[c] + k[0, t, c]) * v[0, t, c]
            den = math.exp(u[c] + k[0, t, c])
            for i in range(t):
                e = math.exp((t - 1 - i) * w[c] + k[0, i, c])
                num += e * v[0, i, c]
                den += e
            assert abs(d[0, t, c] - num / den) <= 1e-13 * max(1.0, abs(num / den))


def test_wkv4_rejects_bad_arguments(oracle_lib):
    lib = oracle.load_library()
    assert lib.la_ref_wkv4(None, None, None, None, None, None, None, 1, 1, 1) == -1


@pytest.mark.parametrize("check", pins.EMA, ids=lambda f: f.__name__)
def test_ema_oracle(oracle_lib, check):
    check(oracle.ema)
