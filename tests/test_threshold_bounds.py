"""The facts the one-pass sparse threshold kernels rely on, checked against
the float64 oracle's exact thresholds on seeded random rows (CPU only).

tau(S) is the threshold of sparsemax (sum relu(u - tau) = 1) or 1.5-entmax
(sum relu(u - tau)^2 = 1, u = z/2) over a key set S.

1. Adding keys never lowers tau, so the threshold of the keys seen so far
   (or of any subset, e.g. one half of a split row) bounds the final one.
2. tau >= max u - 1.
3. For a buffer B that contains the support of the keys seen so far:
   sparsemax tau >= (sum_B u - 1) / |B|, 1.5-entmax tau >= mean_B u - 1/sqrt|B|.
4. One Newton step from the left on g(t) = sum relu(u - t)^k - 1 from any
   t <= tau stays <= tau (g is convex and decreasing).
5. Dropping keys at or below a lower bound of tau leaves tau unchanged.
"""

import numpy as np
import pytest

import oracle

NORMS = ("sparsemax", "entmax15")


def _tau(u, normalizer):
    """Exact threshold in units u (z for sparsemax, z/2 for 1.5-entmax)."""
    if normalizer == "sparsemax":
        return oracle.sparsemax_row(u)[1]
    return oracle.entmax15_row(2.0 * u)[1]


def _rows(seed, n_rows=200):
    rng = np.random.default_rng(seed)
    for _ in range(n_rows):
        n = int(rng.integers(1, 400))
        gain = float(rng.choice([0.25, 1.0, 4.0]))
        yield rng.standard_normal(n) * gain


@pytest.mark.parametrize("normalizer", NORMS)
def test_tau_grows_with_keys_and_is_at_least_max_minus_one(normalizer):
    rng = np.random.default_rng(1)
    for u in _rows(2):
        t = _tau(u, normalizer)
        assert t >= u.max() - 1.0 - 1e-12
        cut = int(rng.integers(1, u.size + 1))
        assert _tau(u[:cut], normalizer) <= t + 1e-12          # prefix
        half = u[rng.permutation(u.size)[: max(1, u.size // 2)]]
        assert _tau(half, normalizer) <= t + 1e-12             # any subset


@pytest.mark.parametrize("normalizer", NORMS)
def test_buffer_moment_bounds(normalizer):
    rng = np.random.default_rng(3)
    for u in _rows(4):
        t = _tau(u, normalizer)
        support = u[u > t]
        extra = u[u <= t]
        # any buffer containing the support (plus some non-support keys)
        k = int(rng.integers(0, extra.size + 1))
        buf = np.concatenate([support, rng.choice(extra, k, replace=False)]) if k else support
        n = buf.size
        if normalizer == "sparsemax":
            bound = (buf.sum() - 1.0) / n
        else:
            bound = buf.mean() - 1.0 / np.sqrt(n)
        assert bound <= t + 1e-12


def _newton_step(u, t, normalizer):
    w = u[u > t] - t
    if normalizer == "sparsemax":
        return t + (w.sum() - 1.0) / w.size
    return t + ((w * w).sum() - 1.0) / (2.0 * w.sum())


@pytest.mark.parametrize("normalizer", NORMS)
def test_newton_step_from_the_left_stays_below(normalizer):
    rng = np.random.default_rng(5)
    for u in _rows(6):
        t_star = _tau(u, normalizer)
        lo = u.max() - 1.0
        t = lo + (t_star - lo) * float(rng.uniform(0.0, 1.0))
        for _ in range(4):
            t_next = _newton_step(u, t, normalizer)
            assert t - 1e-12 <= t_next <= t_star + 1e-9
            t = t_next


@pytest.mark.parametrize("normalizer", NORMS)
def test_dropping_keys_below_a_lower_bound_keeps_tau(normalizer):
    for u in _rows(7):
        t = _tau(u, normalizer)
        lb = max(u.max() - 1.0, t - 0.5)
        kept = u[u > lb]
        assert abs(_tau(kept, normalizer) - t) <= 1e-9


def test_planted_wrong_bound_is_caught():
    """A bound with the wrong sign of the correction term (mean + 1/sqrt|B|)
    must fail the same check: the property test can see a mistake."""
    bad = 0
    for u in _rows(9, 60):
        t = _tau(u, "entmax15")
        support = u[u > t]
        if support.mean() + 1.0 / np.sqrt(support.size) > t + 1e-9:
            bad += 1
    assert bad > 0
