"""Property tests of the oracle on tiny generated rows (hypothesis, CPU only).

Each property follows from the definitions, not from the oracle's code:
probability rows (non-negative, sum 1; softmax1 sums to S/(1+S) < 1), the
optimality conditions of the sparse projections (support members at
exactly p = u - tau or (u - tau)^2, everything else at or below tau), the
shift invariance of all four normalizers, and the visible-key rule of the
masks checked position by position."""

import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

rows = st.lists(st.floats(min_value=-20.0, max_value=20.0, allow_nan=False,
                          allow_infinity=False, width=64), min_size=1, max_size=12)


@settings(max_examples=300, deadline=None)
@given(rows)
def test_sparsemax_row_optimality(z):
    z = np.array(z)
    p, tau = oracle.sparsemax_row(z)
    assert np.all(p >= 0) and abs(p.sum() - 1.0) <= 1e-9
    on = p > 0
    assert np.allclose(p[on], z[on] - tau, atol=1e-9)
    assert np.all(z[~on] <= tau + 1e-9)


@settings(max_examples=300, deadline=None)
@given(rows)
def test_entmax15_row_optimality(z):
    z = np.array(z)
    p, tau = oracle.entmax15_row(z)
    u = z / 2.0
    assert np.all(p >= 0) and abs(p.sum() - 1.0) <= 1e-9
    on = p > 0
    assert np.allclose(p[on], (u[on] - tau) ** 2, atol=1e-9)
    assert np.all(u[~on] <= tau + 1e-9)


@settings(max_examples=300, deadline=None)
@given(rows)
def test_softmax_and_softmax1_rows(z):
    z = np.array(z)
    p, lse = oracle.softmax_row(z)
    assert np.all(p > 0) and abs(p.sum() - 1.0) <= 1e-9
    assert abs(lse - math.log(np.exp(z - z.max()).sum()) - z.max()) <= 1e-9
    p1, lse1 = oracle.softmax1_row(z)
    s = np.exp(z).sum()
    assert abs(p1.sum() - s / (1.0 + s)) <= 1e-9 and p1.sum() < 1.0
    assert abs(lse1 - math.log1p(s)) <= 1e-9 * max(1.0, abs(lse1))


@settings(max_examples=200, deadline=None)
@given(rows, st.floats(min_value=-5.0, max_value=5.0, allow_nan=False, width=64))
def test_shift_invariance(z, c):
    z = np.array(z)
    for fn in (oracle.sparsemax_row, oracle.entmax15_row, oracle.softmax_row):
        p0, _ = fn(z)
        p1, _ = fn(z + c)
        assert np.allclose(p0, p1, atol=1e-9)


@settings(max_examples=200, deadline=None)
@given(st.integers(1, 9), st.integers(1, 9), st.booleans(), st.integers(0, 6))
def test_mask_rule_position_by_position(Tq, Tk, causal, window):
    m = oracle.allowed_matrix(Tq, Tk, causal, window)
    for i in range(Tq):
        pos = i + Tk - Tq  # bottom-right alignment
        for j in range(Tk):
            ok = True
            if causal and j > pos:
                ok = False
            if window > 0:
                if causal and pos - j >= window:
                    ok = False
                if not causal and abs(pos - j) >= window:
                    ok = False
            assert bool(m[i, j]) == ok, (i, j)
