"""CPU checks of the GPU-test harness's own arithmetic (no GPU): the perturbation bound
the end-to-end attention check relies on holds, and is not vacuous."""
import numpy as np

from oracle import lc_oracle as O
from tests.oracle_ref import perturbation_bound


def _normalised(rng, shape):
    return O.rms_norm(rng.standard_normal(shape))


def test_perturbation_bound_holds_for_grid_step_changes():
    """Keys and query moved by one E4M3 / BF16 grid step at random elements (what a
    rounding-midpoint flip does to a stored intermediate): the output moves by no more
    than the bound, and the bound is within a modest factor of the actual change."""
    rng = np.random.default_rng(7)
    H, D, n = 16, 576, 300
    for trial in range(6):
        q = _normalised(rng, (H, D))
        keys = _normalised(rng, (n, D))
        sink = rng.standard_normal(H)
        q2, keys2 = q.copy(), keys.copy()
        hit = rng.random(keys.shape) < 0.01 * (trial + 1)
        keys2[hit] += np.sign(rng.standard_normal(hit.sum())) * O.ulp_e4m3(keys[hit])
        hq = rng.random(q.shape) < 0.002
        q2[hq] += O.ulp_e4m3(q[hq])
        scale = 1 / np.sqrt(D)
        o1, _ = O.attend(q, keys, sink, scale)
        o2, _ = O.attend(q2, keys2, sink, scale)
        b = perturbation_bound(q, keys, q2, keys2, sink, scale)
        d = np.abs(o2 - o1)
        assert np.all(d <= b)
        assert np.max(d) > 0 and np.max(d) >= 0.05 * np.max(b)


def test_perturbation_bound_is_zero_for_identical_inputs():
    rng = np.random.default_rng(8)
    q = _normalised(rng, (4, 64))
    keys = _normalised(rng, (10, 64))
    b = perturbation_bound(q, keys, q, keys, np.zeros(4), 0.125)
    assert np.all(b <= 1e-12 + 1e-15)
