"""The fp64 oracle against what the pages and the mathematics fix (no GPU)."""
import numpy as np
import pytest

import oracle
import synth
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(oracle.lib())


def test_oracle_reports_threads():
    assert oracle.num_threads() >= 1


# ----------------------------------------------------------------------------
# The shared input generator (no WKV arithmetic): definition and distributions
# ----------------------------------------------------------------------------

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def _mix64(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def test_splitmix64_definition():
    # Vigna's reference splitmix64 seeded with 0 first outputs 0xE220A8397B1DCDAF
    assert _mix64(GAMMA) == 0xE220A8397B1DCDAF
    seed, stream = 1234, 5
    key = _mix64((_mix64((seed + GAMMA) & M64) + (stream + 1) * GAMMA) & M64)
    want = [_mix64((key + (i + 1) * GAMMA) & M64) for i in range(10, 20)]
    got = synth.words(seed, stream, 10, offset=10)
    assert [int(x) for x in got] == want


def test_generator_distributions():
    n = 1 << 20
    z = synth.normal(7, 3, (n,), 0.0, 1.0)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1.0) < 5e-3
    z3 = synth.normal(7, 3, (n,), 0.0, 3.0)
    assert np.allclose(z3, 3.0 * z, rtol=1e-6, atol=1e-6)
    uu = synth.uniform(7, 4, (n,), -3.0, 1.0)
    assert uu.min() > -3.0 and uu.max() < 1.0 and abs(uu.mean() + 1.0) < 1e-2
    w = synth.exp_uniform(7, 4, (n,), -3.0, 1.0)
    assert np.allclose(np.log(w.astype(np.float64)), uu, atol=1e-6)
    k = np.zeros(n, np.float32)
    synth.spike(7, 5, k, 0.01, 40.0)
    frac = np.mean(k == 40.0)
    assert abs(frac - 0.01) < 1e-3


def test_generator_is_counter_based():
    a = synth.normal(11, 3, (1000,))
    b = synth.normal(11, 3, (600,), offset=400)
    assert np.array_equal(a[400:], b)
    idx = np.array([5, 999, 0, 17])
    assert np.array_equal(synth.normal_at(11, 3, idx), a[idx])


def test_bf16_rounding_is_nearest_even():
    import torch
    x = synth.normal(3, 3, (4096,), 0.0, 2.0)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5 - 2 ** -9, 3.0]
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(synth.to_bf16_exact(x), want)


def test_forward_sampled_inputs_match_full():
    spec = synth.forward_spec_like("fwd_8x1024x768", 2, 50, 24)
    w, u, k, v = synth.forward_inputs(spec)
    b = np.array([0, 1, 1])
    c = np.array([3, 0, 23])
    ks, vs = synth.forward_inputs_at(spec, b, c)
    assert np.array_equal(ks, k[b, :, c]) and np.array_equal(vs, v[b, :, c])
    assert np.any(k == 40.0)
