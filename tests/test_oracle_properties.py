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
