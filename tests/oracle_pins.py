"""Pins for the fp64 oracle: facts the pages and the mathematics fix, checked
without trusting the oracle itself.

Each ``pin_*`` takes a loaded oracle library handle (so the same pins can be run
against deliberately broken copies of the oracle, see test_oracle_mutants.py)
and raises AssertionError when the oracle disagrees with the fact.

Sources: the RWKV transformer-math page (aicassindra.com, tm_rwkv_math) --
sections "The WKV operator: attention with a fixed decay", "Why it collapses
into a recurrence", "Numerical stability: carry the exponent", "A worked
example, one channel", "Token shift: a two-tap causal convolution"; the aiwiki
"RWKV" page (eq. 1 and its one-token decode step); the vanos001 "RWKV
(Attention-RNN Hybrid)" page (decode step written with a negative stored decay).
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_example.txt")


def read_golden(path=GOLDEN):
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (x.strip() for x in line.split("=", 1))
            nums = [float(x) for x in val.split()]
            vals[key] = nums if len(nums) > 1 else nums[0]
    return vals


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_case(seed, B=2, T=17, C=5, k_std=1.0, w_lo=-3.0, w_hi=1.0):
    r = _rng(seed)
    w = np.exp(r.uniform(w_lo, w_hi, C))
    u = r.normal(0.0, 0.5, C)
    k = r.normal(0.0, k_std, (B, T, C))
    v = r.normal(0.0, 1.0, (B, T, C))
    return w, u, k, v


def _accum(st):
    """True accumulators (A, B) = (a e^p, b e^p) of a [3, ...] state."""
    return st[0] * np.exp(st[2]), st[1] * np.exp(st[2])


# ----------------------------------------------------------------------------
# The page's worked example
# ----------------------------------------------------------------------------

def pin_worked_example(L):
    g = read_golden()
    w = np.array([g["w"]])
    u = np.array([g["u"]])
    k = np.array(g["k"]).reshape(1, 3, 1)
    v = np.array(g["v"]).reshape(1, 3, 1)
    tol = 5e-5  # the page prints 4 decimals
    yd, _ = oracle.wkv_direct(w, u, k, v, L=L)
    yr, _, _, _ = oracle.wkv_recurrent(w, u, k, v, L=L)
    yn = oracle.wkv_naive(w, u, k, v, L=L)
    for y in (yd, yr, yn):
        assert abs(y[0, 2, 0] - g["wkv_last"]) <= tol, (y[0, 2, 0], g["wkv_last"])
    # the page's intermediate accumulators, through the stored state
    _, _, st1, _ = oracle.wkv_recurrent(w, u, k[:, :1], v[:, :1], L=L)
    A0, B0 = _accum(st1)
    assert abs(A0[0, 0] - g["A_0"]) <= tol and abs(B0[0, 0] - g["B_0"]) <= tol, (A0, B0)
    _, _, st2, _ = oracle.wkv_recurrent(w, u, k[:, :2], v[:, :2], L=L)
    A1, B1 = _accum(st2)
    assert abs(A1[0, 0] - g["A_1"]) <= tol and abs(B1[0, 0] - g["B_1"]) <= tol, (A1, B1)
    # the page's numerator and denominator are sums of three terms each printed to
    # 4 decimals, so each carries up to 2e-4 of rounding; their ratio then agrees
    # with y to 3.9 * (2e-4/19.6 + 2e-4/5.07) < 2e-4
    assert abs(g["numerator"] / g["denominator"] - yd[0, 2, 0]) <= 2e-4
    assert abs(math.exp(-g["w"]) - g["decay"]) <= tol


# ----------------------------------------------------------------------------
# Three routes to the same number
# ----------------------------------------------------------------------------

def pin_routes_agree(L):
    for seed, (B, T, C) in enumerate([(1, 1, 1), (2, 17, 5), (1, 64, 64), (3, 33, 7)]):
        w, u, k, v = _rand_case(100 + seed, B, T, C)
        yd, sd = oracle.wkv_direct(w, u, k, v, L=L)
        yr, sr, _, _ = oracle.wkv_recurrent(w, u, k, v, L=L)
        yn = oracle.wkv_naive(w, u, k, v, L=L)
        assert np.all(np.isfinite(yd)) and np.all(np.isfinite(yr))
        scale = np.maximum(sd, 1e-300)
        assert np.max(np.abs(yd - yr) / scale) <= 1e-12
        assert np.max(np.abs(yd - yn) / scale) <= 1e-12
        assert np.max(np.abs(sd - sr) / scale) <= 1e-12


def pin_brute_force_high_precision(L):
    """eq. 1 in 40-digit arithmetic (mpmath) on tiny inputs; the fp64 routes must sit
    within a few hundred ulps of the exact value."""
    import mpmath
    mpmath.mp.dps = 40
    w, u, k, v = _rand_case(7, B=1, T=9, C=3, k_std=2.0)
    yd, sd = oracle.wkv_direct(w, u, k, v, L=L)
    yr, _, _, _ = oracle.wkv_recurrent(w, u, k, v, L=L)
    for c in range(3):
        for t in range(9):
            num = mpmath.mpf(0)
            den = mpmath.mpf(0)
            for i in range(t):
                e = mpmath.exp(-(t - 1 - i) * mpmath.mpf(w[c]) + mpmath.mpf(k[0, i, c]))
                num += e * mpmath.mpf(v[0, i, c])
                den += e
            e = mpmath.exp(mpmath.mpf(u[c]) + mpmath.mpf(k[0, t, c]))
            num += e * mpmath.mpf(v[0, t, c])
            den += e
            exact = float(num / den)
            assert abs(yd[0, t, c] - exact) <= 1e-13 * sd[0, t, c], (t, c)
            assert abs(yr[0, t, c] - exact) <= 1e-13 * sd[0, t, c], (t, c)


# ----------------------------------------------------------------------------
# Special cases and closed forms
# ----------------------------------------------------------------------------

def pin_first_position_is_v(L):
    """The sum over the past is empty at the first position, so y = v (any k, u, w)."""
    w, u, k, v = _rand_case(11, B=2, T=5, C=9, k_std=5.0)
    yr, _, _, _ = oracle.wkv_recurrent(w, u, k, v, L=L)
    assert np.array_equal(yr[:, 0, :], v[:, 0, :])
    yd, _ = oracle.wkv_direct(w, u, k, v, L=L)
    assert np.max(np.abs(yd[:, 0, :] - v[:, 0, :]) / np.maximum(np.abs(v[:, 0, :]), 1e-300)) <= 4e-16
    yr1, _, _, _ = oracle.wkv_recurrent(w, u, k[:, :1], v[:, :1], L=L)
    assert np.array_equal(yr1[:, 0, :], v[:, 0, :])


def pin_convex_bound(L):
    """Numerator and denominator share their weights: y_t lies within [min v, max v] of i <= t."""
    w, u, k, v = _rand_case(12, B=2, T=50, C=8, k_std=3.0)
    for y in (oracle.wkv_direct(w, u, k, v, L=L)[0], oracle.wkv_recurrent(w, u, k, v, L=L)[0]):
        lo = np.minimum.accumulate(v, axis=1)
        hi = np.maximum.accumulate(v, axis=1)
        assert np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12)


def pin_running_mean(L):
    """w = 0, u = 0, constant k: every weight is equal, so y_t is the mean of v_0..v_t."""
    B, T, C = 2, 40, 6
    r = _rng(13)
    v = r.normal(0, 1, (B, T, C))
    k = np.full((B, T, C), 0.3)
    w = np.zeros(C)
    u = np.zeros(C)
    mean = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None]
    for y in (oracle.wkv_direct(w, u, k, v, L=L)[0], oracle.wkv_recurrent(w, u, k, v, L=L)[0],
              oracle.wkv_naive(w, u, k, v, L=L)):
        assert np.max(np.abs(y - mean)) <= 1e-13


def pin_two_tap_softmax(L):
    """Huge decay (w = 1e4): only the most recent past token (undecayed, i = t-1) and the
    current token survive, so y_t is a two-way softmax of (k_{t-1}, u + k_t) over
    (v_{t-1}, v_t).  Pins the off-by-one in the decay exponent."""
    B, T, C = 1, 12, 4
    r = _rng(14)
    k = r.normal(0, 1.5, (B, T, C))
    v = r.normal(0, 1, (B, T, C))
    u = r.normal(0, 0.5, C)
    w = np.full(C, 1e4)
    ep = np.exp(k[:, :-1])
    ec = np.exp(u[None, None, :] + k[:, 1:])
    want = (ep * v[:, :-1] + ec * v[:, 1:]) / (ep + ec)
    for y in (oracle.wkv_direct(w, u, k, v, L=L)[0], oracle.wkv_recurrent(w, u, k, v, L=L)[0]):
        assert np.max(np.abs(y[:, 1:] - want)) <= 1e-13
        assert np.array_equal(y[:, 0], v[:, 0]) or np.max(np.abs(y[:, 0] - v[:, 0])) <= 1e-15


def pin_bonus_to_minus_infinity(L):
    """u -> -inf removes the current token: with w = 1e4 the output is then v_{t-1} for
    t >= 1; the first position keeps its limit y_0 = v_0."""
    B, T, C = 1, 10, 3
    r = _rng(15)
    k = r.normal(0, 1, (B, T, C))
    v = r.normal(0, 1, (B, T, C))
    w = np.full(C, 1e4)
    yr = oracle.wkv_recurrent(w, np.full(C, -1e4), k, v, L=L)[0]
    assert np.array_equal(yr[:, 0], v[:, 0])
    assert np.max(np.abs(yr[:, 1:] - v[:, :-1])) <= 1e-15
    yd = oracle.wkv_direct(w, np.full(C, -600.0), k, v, L=L)[0]  # e^-600 is tiny but not 0
    assert np.max(np.abs(yd[:, 1:] - v[:, :-1])) <= 1e-15
    # with an ordinary decay, u = -1e4 gives the past-only average: check against
    # the same case with the current token's key pushed to -inf by hand
    w2 = np.exp(r.uniform(-3, 1, C))
    y_cut = oracle.wkv_recurrent(w2, np.full(C, -1e4), k, v, L=L)[0]
    for t in range(1, T):
        kk = k.copy()
        kk[:, t] = -1e4  # current key removed; past unchanged
        y_ref = oracle.wkv_recurrent(w2, np.zeros(C), kk[:, : t + 1], v[:, : t + 1], L=L)[0]
        assert np.max(np.abs(y_cut[:, t] - y_ref[:, t])) <= 1e-13


def pin_key_shift_invariance(L):
    """k -> k + c scales every weight by e^c: y is unchanged and the running maximum
    shifts by exactly c (keys up to 40 plus a shift of 100: no inf/NaN)."""
    w, u, k, v = _rand_case(16, B=2, T=60, C=5, k_std=3.0, w_lo=-5)
    k = k.copy()
    k[:, ::7, ::2] = 40.0
    y0, _, st0, _ = oracle.wkv_recurrent(w, u, k, v, L=L)
    y1, _, st1, _ = oracle.wkv_recurrent(w, u, k + 100.0, v, L=L)
    assert np.all(np.isfinite(y1)) and np.all(np.isfinite(st1))
    assert np.max(np.abs(y1 - y0)) <= 1e-12
    assert np.max(np.abs(st1[2] - st0[2] - 100.0)) <= 1e-11
    assert np.max(np.abs(st1[:2] - st0[:2]) / np.maximum(np.abs(st0[:2]), 1e-300)) <= 1e-11
    yd0, _ = oracle.wkv_direct(w, u, k, v, L=L)
    yd1, _ = oracle.wkv_direct(w, u, k + 100.0, v, L=L)
    assert np.all(np.isfinite(yd1)) and np.max(np.abs(yd1 - yd0)) <= 1e-12


def pin_value_affine(L):
    """Weights sum to one after normalising: y(alpha v + beta) = alpha y(v) + beta."""
    w, u, k, v = _rand_case(17, B=1, T=30, C=4)
    y0 = oracle.wkv_recurrent(w, u, k, v, L=L)[0]
    y1 = oracle.wkv_recurrent(w, u, k, -2.5 * v + 3.0, L=L)[0]
    assert np.max(np.abs(y1 - (-2.5 * y0 + 3.0))) <= 1e-12
    yd0 = oracle.wkv_direct(w, u, k, v, L=L)[0]
    yd1 = oracle.wkv_direct(w, u, k, -2.5 * v + 3.0, L=L)[0]
    assert np.max(np.abs(yd1 - (-2.5 * yd0 + 3.0))) <= 1e-12


def pin_running_max_closed_form(L):
    """The stored exponent after t tokens is max_{i<=t} (k_i - (t - i) w), and b >= 1
    (the maximising token contributes e^0)."""
    w, u, k, v = _rand_case(18, B=2, T=25, C=6, k_std=2.0)
    for T in (1, 2, 7, 25):
        _, _, st, _ = oracle.wkv_recurrent(w, u, k[:, :T], v[:, :T], L=L)
        i = np.arange(T)[None, :, None]
        want = np.max(k[:, :T] - (T - 1 - i) * w[None, None, :], axis=1)
        assert np.max(np.abs(st[2] - want)) <= 1e-12
        assert np.all(st[1] >= 1.0 - 1e-15)


def pin_naive_accumulators(L):
    """The stored state's true accumulators equal the plain two-accumulator sums
    a_t = sum_i e^{-(t-i) w + k_i} v_i, b_t = sum_i e^{-(t-i) w + k_i}."""
    w, u, k, v = _rand_case(19, B=1, T=15, C=4)
    _, _, st, _ = oracle.wkv_recurrent(w, u, k, v, L=L)
    A, Bs = _accum(st)
    i = np.arange(15)[None, :, None]
    wt = np.exp(-(14 - i) * w[None, None, :] + k)
    assert np.max(np.abs(A - np.sum(wt * v, axis=1)) / np.sum(wt * np.abs(v), axis=1)) <= 1e-13
    assert np.max(np.abs(Bs - np.sum(wt, axis=1)) / np.sum(wt, axis=1)) <= 1e-13


def pin_prefill_then_decode(L):
    """Prefill produces the state, decode steps continue from it: the sequence cut at any
    point and resumed from the stored state gives the uncut result, bit for bit."""
    w, u, k, v = _rand_case(20, B=2, T=21, C=3, k_std=3.0)
    y, s, st, sa = oracle.wkv_recurrent(w, u, k, v, L=L)
    for cut in (0, 1, 8, 20):
        y1, _, st1, sa1 = oracle.wkv_recurrent(w, u, k[:, :cut], v[:, :cut], L=L)
        y2, _, st2, sa2 = oracle.wkv_recurrent(w, u, k[:, cut:], v[:, cut:], state_in=st1, sacc_in=sa1, L=L)
        assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
        assert np.array_equal(st2, st) and np.array_equal(sa2, sa)
    # token by token, as a decode loop does
    stt, sat = None, None
    for t in range(21):
        yt, _, stt, sat = oracle.wkv_recurrent(w, u, k[:, t:t + 1], v[:, t:t + 1], state_in=stt,
                                               sacc_in=sat, L=L)
        assert np.array_equal(yt[:, 0], y[:, t])
    assert np.array_equal(stt, st)


def pin_decode_layer_indexing(L):
    """Decode rows are [N, L, C] with parameters [L, C]: row (n, l) uses layer l's w, u."""
    N, Ly, C = 3, 4, 5
    r = _rng(21)
    w = np.exp(r.uniform(-3, 1, (Ly, C)))
    u = r.normal(0, 0.5, (Ly, C))
    k = r.normal(0, 1, (N, Ly, C))
    v = r.normal(0, 1, (N, Ly, C))
    st = np.stack([r.normal(0, 1, (N, Ly, C)), 1 + np.abs(r.normal(0, 1, (N, Ly, C))),
                   r.normal(0, 1, (N, Ly, C))])
    y, _, st2, _ = oracle.decode_step(w, u, k, v, st, L=L)
    for l in range(Ly):
        yl, _, stl, _ = oracle.wkv_recurrent(w[l], u[l], k[:, l:l + 1], v[:, l:l + 1], state_in=st[:, :, l],
                                             L=L)
        assert np.array_equal(yl[:, 0], y[:, l])
        assert np.array_equal(stl, st2[:, :, l])


def pin_negative_decay_convention(L):
    """One page writes the step with a stored decay that is negative and added
    (p + w_stored).  With w_stored = -w it is the same step; read as +w it no longer
    reproduces the worked example's 3.8619."""
    g = read_golden()

    def step_added_decay(state, kk, vv, w_stored, uu):
        a, b, p = state
        m = max(p, uu + kk)
        y = (a * math.exp(p - m) + math.exp(uu + kk - m) * vv) / (b * math.exp(p - m) + math.exp(uu + kk - m))
        m2 = max(p + w_stored, kk)
        a = a * math.exp(p + w_stored - m2) + vv * math.exp(kk - m2)
        b = b * math.exp(p + w_stored - m2) + math.exp(kk - m2)
        return y, (a, b, m2)

    def run(w_stored):
        st = (0.0, 0.0, oracle.P_EMPTY)
        ys = []
        for kk, vv in zip(g["k"], g["v"]):
            y, st = step_added_decay(st, kk, vv, w_stored, g["u"])
            ys.append(y)
        return ys, st

    w = np.array([g["w"]])
    u = np.array([g["u"]])
    k = np.array(g["k"]).reshape(1, 3, 1)
    v = np.array(g["v"]).reshape(1, 3, 1)
    yr, _, st, _ = oracle.wkv_recurrent(w, u, k, v, L=L)
    ys, stp = run(-g["w"])
    assert ys == list(yr[0, :, 0]) and stp == (st[0, 0, 0], st[1, 0, 0], st[2, 0, 0])
    ys_wrong, _ = run(+g["w"])
    assert abs(ys_wrong[2] - g["wkv_last"]) > 1e-2


def pin_token_shift(L):
    """xbar_t = mu x_t + (1 - mu) x_{t-1}: mu = 1 passes x_t, mu = 0 passes the previous token,
    mu = 1/2 is the exact midpoint; the token before t = 0 is x_last, else zero."""
    B, T, C = 2, 7, 5
    r = _rng(22)
    x = r.normal(0, 1, (B, T, C))
    xl = r.normal(0, 1, (B, C))
    prev = np.concatenate([xl[:, None], x[:, :-1]], axis=1)
    prev0 = np.concatenate([np.zeros((B, 1, C)), x[:, :-1]], axis=1)
    assert np.array_equal(oracle.token_shift(np.ones(C), x, xl, L=L), x)
    assert np.array_equal(oracle.token_shift(np.zeros(C), x, xl, L=L), prev)
    assert np.array_equal(oracle.token_shift(np.full(C, 0.5), x, xl, L=L), (x + prev) / 2)
    assert np.array_equal(oracle.token_shift(np.full(C, 0.5), x, None, L=L), (x + prev0) / 2)
    mu = r.uniform(0, 1, C)
    xb = oracle.token_shift(mu, x, xl, L=L)
    # per channel the result lies between the two taps
    assert np.all(xb >= np.minimum(x, prev) - 1e-15) and np.all(xb <= np.maximum(x, prev) + 1e-15)
    # decode form: one token from the previous one, [N, L, C] rows with [L, C] mu
    mu2 = r.uniform(0, 1, (3, C))
    xt = r.normal(0, 1, (B, 3, C))
    xp = r.normal(0, 1, (B, 3, C))
    xb2 = oracle.decode_token_shift(mu2, xt, xp, L=L)
    for l in range(3):
        want = oracle.token_shift(mu2[l], xt[:, l:l + 1], xp[:, l], L=L)[:, 0]
        assert np.array_equal(xb2[:, l], want)
    assert np.array_equal(oracle.decode_token_shift(np.ones((3, C)), xt, xp, L=L), xt)


def pin_gate(L):
    """The receptance gate sigma(r) * wkv ("Receptance: the gate on the way out"): sigma(0) =
    1/2 exactly, the limits r -> +inf (pass) and r -> -inf (mute), the reflection
    sigma(r) + sigma(-r) = 1, sigma against scipy's logistic function, and a gate that acts
    channel by channel (each output depends only on its own r)."""
    from scipy.special import expit
    r = _rng(31)
    wkv = r.normal(0, 2, (2, 9, 6))
    assert np.array_equal(oracle.gate(np.zeros_like(wkv), wkv, L=L), wkv / 2)
    assert np.allclose(oracle.gate(np.full_like(wkv, 60.0), wkv, L=L), wkv, rtol=1e-25, atol=0)
    assert np.array_equal(oracle.gate(np.full_like(wkv, -800.0), wkv, L=L), np.zeros_like(wkv))
    rr = r.normal(0, 3, wkv.shape)
    g, gm = oracle.gate(rr, wkv, L=L), oracle.gate(-rr, wkv, L=L)
    assert np.allclose(g + gm, wkv, rtol=1e-14, atol=1e-14)
    assert np.allclose(g, wkv * expit(rr), rtol=1e-14, atol=1e-300)
    # channel by channel: changing r at one position changes only that output
    rr2 = rr.copy()
    rr2[1, 4, 2] += 1.0
    diff = oracle.gate(rr2, wkv, L=L) != g
    assert diff.sum() == 1 and diff[1, 4, 2]


def pin_token_shift3(L):
    """The three projections' lerps ("Token shift": separate mu_r, mu_k, mu_v): each output
    follows its own mu only (mu = 1 passes x_t, mu = 0 the previous token), in the order
    (r, k, v)."""
    B, T, C = 2, 6, 4
    r = _rng(32)
    x = r.normal(0, 1, (B, T, C))
    xl = r.normal(0, 1, (B, C))
    prev = np.concatenate([xl[:, None], x[:, :-1]], axis=1)
    one, zero, half = np.ones(C), np.zeros(C), np.full(C, 0.5)
    xr, xk, xv = oracle.token_shift3(one, zero, half, x, xl, L=L)
    assert np.array_equal(xr, x) and np.array_equal(xk, prev) and np.array_equal(xv, (x + prev) / 2)
    xr, xk, xv = oracle.token_shift3(zero, half, one, x, None, L=L)
    prev0 = np.concatenate([np.zeros((B, 1, C)), x[:, :-1]], axis=1)
    assert np.array_equal(xr, prev0) and np.array_equal(xk, (x + prev0) / 2) and np.array_equal(xv, x)


def _loss(L, w, u, k, v, gy):
    return float((oracle.wkv_direct(w, u, k, v, L=L)[0] * gy).sum())


def pin_backward_finite_differences(L):
    """The gradient of L = sum(gy * y) against central finite differences of the (pinned)
    direct forward, for every k and v element and every channel's w and u."""
    for seed, (B, T, C) in ((41, (1, 6, 2)), (42, (2, 4, 3))):
        w, u, k, v = _rand_case(seed, B, T, C)
        gy = _rng(seed + 100).normal(0, 1, k.shape)
        gk, gv, gw, gu, (sk, sv, sw, su) = oracle.wkv_backward(w, u, k, v, gy, L=L)
        h = 1e-6

        def fd(arr, idx, fn):
            a1, a0 = arr.copy(), arr.copy()
            a1[idx] += h
            a0[idx] -= h
            return (fn(a1) - fn(a0)) / (2 * h)

        for idx in np.ndindex(k.shape):
            assert abs(fd(k, idx, lambda x: _loss(L, w, u, x, v, gy)) - gk[idx]) <= 1e-7 * (sk[idx] + 1e-12)
            assert abs(fd(v, idx, lambda x: _loss(L, w, u, k, x, gy)) - gv[idx]) <= 1e-7 * (sv[idx] + 1e-12)
        for c in range(C):
            assert abs(fd(w, (c,), lambda x: _loss(L, x, u, k, v, gy)) - gw[c]) <= 1e-7 * (sw[c] + 1e-12)
            assert abs(fd(u, (c,), lambda x: _loss(L, w, x, k, v, gy)) - gu[c]) <= 1e-7 * (su[c] + 1e-12)


def pin_backward_closed_forms(L):
    """T = 1: y = v exactly, so gv = gy and every other gradient is zero.  Key shift: y does not
    change when every key of a channel moves by the same amount, so the k-gradients of each
    (b, c) sum to zero.  Value shift: y moves by exactly the shift (a convex combination), so
    the v-gradients of each (b, c) sum to the sum of gy."""
    w, u, k, v = _rand_case(43, 2, 1, 4)
    gy = _rng(143).normal(0, 1, k.shape)
    gk, gv, gw, gu, _ = oracle.wkv_backward(w, u, k, v, gy, L=L)
    tiny = 1e-15 * np.abs(gy * v)  # y = (alpha v) / alpha is v up to one rounding
    assert np.allclose(gv, gy, rtol=1e-15, atol=0) and np.all(gw == 0)
    assert np.all(np.abs(gk) <= tiny) and np.all(np.abs(gu) <= tiny.sum(axis=(0, 1)))
    w, u, k, v = _rand_case(44, 2, 9, 3)
    gy = _rng(144).normal(0, 1, k.shape)
    gk, gv, gw, gu, (sk, sv, _, _) = oracle.wkv_backward(w, u, k, v, gy, L=L)
    assert np.all(np.abs(gk.sum(axis=1)) <= 1e-12 * sk.sum(axis=1))
    assert np.allclose(gv.sum(axis=1), gy.sum(axis=1), rtol=1e-12, atol=1e-12)


def pin_backward_magnitude_scales(L):
    """The backward's magnitude scales (each gradient's terms added up with |gy| for gy and
    |v| + |y| for v - y) where every sign is fixed: with gy >= 0 and v >= 0 (so y >= 0, a convex
    combination) they follow from the gradients and the pinned forward alone.  y_t is linear in
    v (y_t = sum_i beta_{t,i} v_i / D_t with D_t independent of v), so running the direct forward
    on a value sequence zeroed outside a set of tokens picks out those tokens' weighted values:
      sv = gv,   sk = 2 v gv - gk,
      su = 2 sum_t gy_t y_t(v kept at token t only) - gu,
      sw = 2 sum_t gy_t [(t - 1) y_t(v kept before t) - y_t(i v_i kept before t)] + gw."""
    for seed, (B, T, C) in ((45, (1, 7, 3)), (46, (2, 5, 2))):
        w, u, k, v = _rand_case(seed, B, T, C)
        v = np.abs(v) + 0.1
        gy = np.abs(_rng(seed + 100).normal(0, 1, k.shape)) + 0.05
        gk, gv, gw, gu, (sk, sv, sw, su) = oracle.wkv_backward(w, u, k, v, gy, L=L)
        assert np.allclose(sv, gv, rtol=1e-13, atol=0)
        assert np.allclose(sk, 2 * v * gv - gk, rtol=1e-11, atol=1e-14 * np.max(sk))
        cur = np.zeros(C)
        past = np.zeros(C)
        idx = np.arange(T, dtype=np.float64)[None, :, None]
        for t in range(T):
            only = np.zeros_like(v)
            only[:, t] = v[:, t]
            cur += (gy[:, t] * oracle.wkv_direct(w, u, k, only, L=L)[0][:, t]).sum(axis=0)
            if t > 0:
                before = v.copy()
                before[:, t:] = 0.0
                yb = oracle.wkv_direct(w, u, k, before, L=L)[0][:, t]
                yi = oracle.wkv_direct(w, u, k, idx * before, L=L)[0][:, t]
                past += (gy[:, t] * ((t - 1) * yb - yi)).sum(axis=0)
        assert np.allclose(su, 2 * cur - gu, rtol=1e-11, atol=0)
        assert np.allclose(sw, 2 * past + gw, rtol=1e-10, atol=1e-13 * np.max(sw))


# ----------------------------------------------------------------------------
# Eagle (RWKV-5) matrix-state WKV ("RWKV (Attention-RNN Hybrid)", section
# "Versions: RWKV-4 -> Eagle -> Finch"): S_t = diag(d) S_{t-1} + k_t v_t^T,
# y_t = r_t^T S_t per head, d = exp(-w) on the key index
# ----------------------------------------------------------------------------

EAGLE_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "eagle_hand_example.txt")


def _eagle_case(seed, B=2, T=9, H=2, N=4, w_lo=-3.0, w_hi=1.0):
    g = _rng(seed)
    C = H * N
    w = np.exp(g.uniform(w_lo, w_hi, C))
    r, k, v = (g.normal(0.0, 1.0, (B, T, C)) for _ in range(3))
    return w, r, k, v


def pin_eagle_hand_example(L):
    """One head of two channels over three tokens, worked by hand (exact in binary)."""
    g = read_golden(EAGLE_GOLDEN)
    w = -np.log(np.array(g["d"]))
    r, k, v = (np.array(g[x]).reshape(1, 3, 2) for x in "rkv")
    y, s, st = oracle.eagle_recurrent(w, r, k, v, N=2, L=L)
    assert np.allclose(y.ravel(), g["y"], rtol=0, atol=1e-14)
    assert np.allclose(st.ravel(), g["S"], rtol=0, atol=1e-14)
    assert np.allclose(oracle.eagle_direct(w, r, k, v, N=2, L=L).ravel(), g["y"], rtol=0, atol=1e-14)


def pin_eagle_linear_attention(L):
    """No decay (w = 0, d = 1): the state is the running sum of k_i v_i^T, so each head's
    output is causal linear attention, tril(R K^T) V, here by matrix products."""
    B, T, H, N = 2, 11, 3, 4
    w, r, k, v = _eagle_case(50, B, T, H, N)
    w = np.zeros_like(w)
    y, s, _ = oracle.eagle_recurrent(w, r, k, v, N=N, L=L)
    yd = oracle.eagle_direct(w, r, k, v, N=N, L=L)
    mask = np.tril(np.ones((T, T)))
    for b in range(B):
        for h in range(H):
            sl = slice(h * N, (h + 1) * N)
            ref = ((r[b, :, sl] @ k[b, :, sl].T) * mask) @ v[b, :, sl]
            assert np.allclose(y[b, :, sl], ref, rtol=1e-12, atol=1e-12)
            assert np.allclose(yd[b, :, sl], ref, rtol=1e-12, atol=1e-12)


def pin_eagle_no_memory(L):
    """Total decay (w = 1e4: exp(-1e4) is exactly 0): only the current token survives, so
    y_t = (r_t . k_t) v_t per head, and the state is k_{T-1} v_{T-1}^T."""
    B, T, H, N = 2, 5, 2, 3
    w, r, k, v = _eagle_case(51, B, T, H, N)
    w = np.full_like(w, 1e4)
    y, _, st = oracle.eagle_recurrent(w, r, k, v, N=N, L=L)
    for h in range(H):
        sl = slice(h * N, (h + 1) * N)
        dot = (r[:, :, sl] * k[:, :, sl]).sum(-1, keepdims=True)
        assert np.allclose(y[:, :, sl], dot * v[:, :, sl], rtol=1e-13, atol=1e-13)
        assert np.allclose(st[:, h], k[:, -1, sl][:, :, None] * v[:, -1, sl][:, None, :], rtol=0, atol=0)


def pin_eagle_one_token_from_state(L):
    """One token from a given state S: y = r^T (diag(d) S + k v^T) written out per element, and
    the state that comes back is that matrix."""
    B, H, N = 2, 2, 3
    w, r, k, v = _eagle_case(52, B, 1, H, N)
    S0 = _rng(152).normal(0, 1, (B, H, N, N))
    y, _, st = oracle.eagle_recurrent(w, r, k, v, N=N, state_in=S0, L=L)
    for b in range(B):
        for h in range(H):
            sl = slice(h * N, (h + 1) * N)
            d = np.exp(-w[sl])
            S1 = np.array([[d[m] * S0[b, h, m, j] + k[b, 0, sl][m] * v[b, 0, sl][j] for j in range(N)]
                           for m in range(N)])
            assert np.allclose(st[b, h], S1, rtol=1e-14, atol=1e-14)
            yj = [sum(r[b, 0, sl][m] * S1[m, j] for m in range(N)) for j in range(N)]
            assert np.allclose(y[b, 0, sl], yj, rtol=1e-13, atol=1e-13)


def pin_eagle_routes_and_split(L):
    """The recurrence and the direct sum agree (the same arithmetic regrouped), also from a
    given state; running T1 tokens, then the rest from the returned state, gives the whole."""
    B, T, H, N = 2, 13, 2, 4
    w, r, k, v = _eagle_case(53, B, T, H, N)
    S0 = _rng(153).normal(0, 1, (B, H, N, N))
    for st_in in (None, S0):
        y, s, st = oracle.eagle_recurrent(w, r, k, v, N=N, state_in=st_in, L=L)
        yd = oracle.eagle_direct(w, r, k, v, N=N, state_in=st_in, L=L)
        assert np.all(np.abs(y - yd) <= 1e-12 * s)
        assert np.all(s >= np.abs(y) * (1 - 1e-12))
    y, s, st = oracle.eagle_recurrent(w, r, k, v, N=N, L=L)
    cut = 6
    y1, _, st1 = oracle.eagle_recurrent(w, r[:, :cut], k[:, :cut], v[:, :cut], N=N, L=L)
    y2, _, st2 = oracle.eagle_recurrent(w, r[:, cut:], k[:, cut:], v[:, cut:], N=N, state_in=st1, L=L)
    assert np.all(np.abs(np.concatenate([y1, y2], axis=1) - y) <= 1e-13 * s)
    assert np.allclose(st2, st, rtol=1e-13, atol=1e-13)


def pin_eagle_bilinear_and_heads(L):
    """y is linear in v and in r (each alone), and a head's output depends on its own
    channels only: changing one head's inputs leaves every other head's outputs as they were."""
    B, T, H, N = 1, 7, 3, 4
    w, r, k, v = _eagle_case(54, B, T, H, N)
    _, _, v2 = (x for x in _eagle_case(55, B, T, H, N)[1:])
    y1 = oracle.eagle_recurrent(w, r, k, v, N=N, L=L)[0]
    y2, s2, _ = oracle.eagle_recurrent(w, r, k, v2, N=N, L=L)
    y12, s12, _ = oracle.eagle_recurrent(w, r, k, 2 * v - 3 * v2, N=N, L=L)
    assert np.all(np.abs(y12 - (2 * y1 - 3 * y2)) <= 1e-12 * (s12 + s2))
    yr = oracle.eagle_recurrent(w, -0.5 * r, k, v, N=N, L=L)[0]
    assert np.allclose(yr, -0.5 * y1, rtol=1e-14, atol=0)
    k3 = k.copy()
    k3[:, :, N:2 * N] += 1.0  # head 1's keys only
    y3 = oracle.eagle_recurrent(w, r, k3, v, N=N, L=L)[0]
    assert np.array_equal(y3[:, :, :N], y1[:, :, :N]) and np.array_equal(y3[:, :, 2 * N:], y1[:, :, 2 * N:])
    assert not np.allclose(y3[:, :, N:2 * N], y1[:, :, N:2 * N])


def pin_eagle_magnitude_scale(L):
    """Eagle's magnitude scale s is the read-out of |r|, |k|, |v| and |S_in|: it equals the
    (pinned) direct sum evaluated on those absolute values, and with non-negative inputs it is
    y itself, bit for bit (the same products in the same order)."""
    B, T, H, N = 2, 10, 2, 4
    w, r, k, v = _eagle_case(56, B, T, H, N)
    S0 = _rng(156).normal(0, 1, (B, H, N, N))
    for st_in in (None, S0):
        _, s, _ = oracle.eagle_recurrent(w, r, k, v, N=N, state_in=st_in, L=L)
        sd = oracle.eagle_direct(w, np.abs(r), np.abs(k), np.abs(v), N=N,
                                 state_in=None if st_in is None else np.abs(st_in), L=L)
        assert np.allclose(s, sd, rtol=1e-12, atol=0)
    y, s, _ = oracle.eagle_recurrent(w, np.abs(r), np.abs(k), np.abs(v), N=N, state_in=np.abs(S0), L=L)
    assert np.array_equal(s, y)


ALL_PINS = [
    pin_worked_example,
    pin_routes_agree,
    pin_brute_force_high_precision,
    pin_first_position_is_v,
    pin_convex_bound,
    pin_running_mean,
    pin_two_tap_softmax,
    pin_bonus_to_minus_infinity,
    pin_key_shift_invariance,
    pin_value_affine,
    pin_running_max_closed_form,
    pin_naive_accumulators,
    pin_prefill_then_decode,
    pin_decode_layer_indexing,
    pin_negative_decay_convention,
    pin_token_shift,
    pin_gate,
    pin_token_shift3,
    pin_backward_finite_differences,
    pin_backward_closed_forms,
    pin_backward_magnitude_scales,
    pin_eagle_hand_example,
    pin_eagle_linear_attention,
    pin_eagle_no_memory,
    pin_eagle_one_token_from_state,
    pin_eagle_routes_and_split,
    pin_eagle_bilinear_and_heads,
    pin_eagle_magnitude_scale,
]
