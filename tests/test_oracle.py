"""The FP64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
from oracle_pins import PINS


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(name):
    fn, bound = PINS[name]
    err = fn(oracle.load())
    assert err <= bound, f"{name}: error {err:.3e} above {bound:.1e}"


def test_decode_regrouping_matches_step_by_step():
    """oracle.decode (steps regrouped per sequence) == one recurrence call per step."""
    rng = np.random.default_rng(3)
    steps, N, H, D = 4, 3, 2, 4
    q = rng.standard_normal((steps, N, H, D))
    k = rng.standard_normal((steps, N, H, D))
    v = rng.standard_normal((steps, N, H, D))
    g = -rng.uniform(0, 5, (steps, N, H, D))
    b = rng.uniform(0, 1, (steps, N, H))
    S = rng.standard_normal((N, H, D, D))
    out, fin = oracle.decode(q, k, v, g, b, S)
    cu = np.arange(N + 1)
    state = S
    for t in range(steps):
        o_t, state, _ = oracle.prefill(q[t], k[t], v[t], g[t], b[t], cu, state)
        assert np.abs(o_t - out[t]).max() == 0.0
    assert np.abs(state - fin).max() == 0.0


def test_rejects_bad_arguments():
    q = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, q, np.zeros((4, 1)), [0, 4], None, 3, chunk=2)  # interval % C


def test_empty_sequences():
    q = np.zeros((0, 1, 2))
    S = np.ones((2, 1, 2, 2))
    out, fin, ck = oracle.prefill(q, q, q, q, np.zeros((0, 1)), [0, 0, 0], S, 4)
    assert out.shape == (0, 1, 2) and np.array_equal(fin, S) and ck.shape[0] == 0
