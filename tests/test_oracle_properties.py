"""Property checks of the fp64 oracle over random small shapes (hypothesis): the routes the
pages equate agree, the magnitude scale bounds the output, and a sequence cut anywhere and
resumed from the returned state gives the whole.  The fixed-case pins are in oracle_pins.py."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


@SETTINGS
@given(B=st.integers(1, 2), T=st.integers(1, 24), C=st.integers(1, 5), w_hi=st.floats(-4.0, 2.0),
       k_std=st.floats(0.1, 6.0), seed=st.integers(0, 2**31 - 1))
def test_wkv_routes_agree(B, T, C, w_hi, k_std, seed):
    """The direct sum (eq. 1 as written) and the running-maximum recurrence are the same
    arithmetic regrouped; the magnitude scale s bounds |y|."""
    g = np.random.default_rng(seed)
    w = np.exp(g.uniform(w_hi - 3.0, w_hi, C))
    u = g.normal(0, 0.5, C)
    k = g.normal(0, k_std, (B, T, C))
    v = g.normal(0, 1, (B, T, C))
    yd, sd = oracle.wkv_direct(w, u, k, v)
    yr, sr, _, _ = oracle.wkv_recurrent(w, u, k, v)
    assert np.all(np.abs(yd - yr) <= 1e-11 * sd)
    assert np.all(sr >= np.abs(yr) * (1 - 1e-12))


@SETTINGS
@given(B=st.integers(1, 2), T=st.integers(2, 24), C=st.integers(1, 4), cut=st.floats(0.0, 1.0),
       seed=st.integers(0, 2**31 - 1))
def test_wkv_resume_anywhere(B, T, C, cut, seed):
    g = np.random.default_rng(seed)
    w = np.exp(g.uniform(-3, 1, C))
    u = g.normal(0, 0.5, C)
    k = g.normal(0, 2, (B, T, C))
    v = g.normal(0, 1, (B, T, C))
    c = min(T - 1, max(1, int(cut * T)))
    y, s, st_all, _ = oracle.wkv_recurrent(w, u, k, v)
    y1, _, st1, sa1 = oracle.wkv_recurrent(w, u, k[:, :c], v[:, :c])
    y2, _, st2, _ = oracle.wkv_recurrent(w, u, k[:, c:], v[:, c:], state_in=st1, sacc_in=sa1)
    assert np.all(np.abs(np.concatenate([y1, y2], axis=1) - y) <= 1e-13 * s)
    assert np.allclose(st2, st_all, rtol=1e-13, atol=0)


@SETTINGS
@given(B=st.integers(1, 2), T=st.integers(1, 10), H=st.integers(1, 3), N=st.integers(1, 5),
       w_hi=st.floats(-4.0, 3.0), given_state=st.booleans(), seed=st.integers(0, 2**31 - 1))
def test_eagle_routes_agree(B, T, H, N, w_hi, given_state, seed):
    """Eagle's matrix recurrence and its unrolled sum agree, from the empty or a given state;
    the magnitude scale bounds |y|."""
    g = np.random.default_rng(seed)
    C = H * N
    w = np.exp(g.uniform(w_hi - 4.0, w_hi, C))
    r, k, v = (g.normal(0, 1, (B, T, C)) for _ in range(3))
    S0 = g.normal(0, 1, (B, H, N, N)) if given_state else None
    y, s, _ = oracle.eagle_recurrent(w, r, k, v, N=N, state_in=S0)
    yd = oracle.eagle_direct(w, r, k, v, N=N, state_in=S0)
    assert np.all(np.abs(y - yd) <= 1e-12 * s + 1e-300)
    assert np.all(s >= np.abs(y) * (1 - 1e-12))


@SETTINGS
@given(T=st.integers(2, 16), N=st.integers(1, 4), cut=st.floats(0.0, 1.0), seed=st.integers(0, 2**31 - 1))
def test_eagle_resume_anywhere(T, N, cut, seed):
    g = np.random.default_rng(seed)
    B, H = 2, 2
    C = H * N
    w = np.exp(g.uniform(-3, 1, C))
    r, k, v = (g.normal(0, 1, (B, T, C)) for _ in range(3))
    c = min(T - 1, max(1, int(cut * T)))
    y, s, st_all = oracle.eagle_recurrent(w, r, k, v, N=N)
    y1, _, st1 = oracle.eagle_recurrent(w, r[:, :c], k[:, :c], v[:, :c], N=N)
    y2, _, st2 = oracle.eagle_recurrent(w, r[:, c:], k[:, c:], v[:, c:], N=N, state_in=st1)
    assert np.all(np.abs(np.concatenate([y1, y2], axis=1) - y) <= 1e-13 * s + 1e-300)
    assert np.allclose(st2, st_all, rtol=1e-12, atol=1e-12)


@settings(max_examples=20, deadline=None, derandomize=True)
@given(B=st.integers(1, 2), T=st.integers(1, 6), C=st.integers(1, 3), seed=st.integers(0, 2**31 - 1))
def test_backward_matches_finite_differences(B, T, C, seed):
    """Every gradient of L = sum(gy * y) against central differences of the direct forward."""
    g = np.random.default_rng(seed)
    w = np.exp(g.uniform(-3, 1, C))
    u = g.normal(0, 0.5, C)
    k = g.normal(0, 1, (B, T, C))
    v = g.normal(0, 1, (B, T, C))
    gy = g.normal(0, 1, (B, T, C))
    gk, gv, gw, gu, (sk, sv, sw, su) = oracle.wkv_backward(w, u, k, v, gy)

    def loss(w_, u_, k_, v_):
        return float((oracle.wkv_direct(w_, u_, k_, v_)[0] * gy).sum())

    h = 1e-6
    for arr, grad, scale, pos in ((k, gk, sk, 2), (v, gv, sv, 3), (w, gw, sw, 0), (u, gu, su, 1)):
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args_p = [w, u, k, v]
            args_m = [w, u, k, v]
            args_p[pos], args_m[pos] = plus, minus
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * (scale[idx] + 1e-9)


@SETTINGS
@given(n=st.integers(1, 64), seed=st.integers(0, 2**31 - 1))
def test_gate_symmetry(n, seed):
    """sigma(r) + sigma(-r) = 1: gate(r, x) + gate(-r, x) = x."""
    g = np.random.default_rng(seed)
    r = g.normal(0, 4, n)
    x = g.normal(0, 1, n)
    assert np.allclose(oracle.gate(r, x) + oracle.gate(-r, x), x, rtol=1e-14, atol=1e-15)


@SETTINGS
@given(B=st.integers(1, 2), T=st.integers(1, 8), C=st.integers(1, 5), seed=st.integers(0, 2**31 - 1))
def test_token_shift3_is_three_lerps(B, T, C, seed):
    """The three-mu shift is the one-mu shift with each projection's mu, and a lerp: linear in
    mu with the current token at mu = 1."""
    g = np.random.default_rng(seed)
    mus = [g.uniform(0, 1, C) for _ in range(3)]
    x = g.normal(0, 1, (B, T, C))
    xl = g.normal(0, 1, (B, C))
    outs = oracle.token_shift3(*mus, x, xl)
    for o, mu in zip(outs, mus):
        assert np.array_equal(o, oracle.token_shift(mu, x, xl))
    ones = oracle.token_shift(np.ones(C), x, xl)
    assert np.array_equal(ones, x)
