"""Shared helpers for the parity tests: library build, tolerance checks,
row sampling.  The tolerances are the ones the attention forward is held to:
output max-abs <= 2e-2 and mean-abs <= 2e-3 against the float64 oracle,
per-row log-sum-exp / threshold within 1e-3, masked weights exactly 0."""

import numpy as np

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
STAT_ABS = 1e-3


def ensure_built():
    from alternative_normalizers_b200 import build
    return build.build()


def cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def check_out(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want)
    assert err.max() <= OUT_MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= OUT_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"


def check_stat(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    inf = ~np.isfinite(want)
    assert np.array_equal(got[inf], want[inf]), f"{what}: infinite stats differ"
    if (~inf).any():
        err = np.abs(got[~inf] - want[~inf])
        assert err.max() <= STAT_ABS, f"{what}: max stat err {err.max():.3e}"


def sample_rows(B, Hq, Tq, n, seed, group=1, extra=()):
    """Seeded (b, h, i) rows: first/last rows of every 128-row tile edge of a
    few heads, all heads of one KV group, plus uniform picks."""
    rng = np.random.default_rng(seed)
    rows = set()
    for e in extra:
        rows.add(tuple(e))
    h0 = int(rng.integers(0, Hq // group)) * group
    for h in range(h0, h0 + group):
        for i in (0, 1, 127, 128, Tq // 2, Tq - 2, Tq - 1):
            if 0 <= i < Tq:
                rows.add((0, h, i))
    while len(rows) < n:
        rows.add((int(rng.integers(0, B)), int(rng.integers(0, Hq)),
                  int(rng.integers(0, Tq))))
    return np.array(sorted(rows), dtype=np.int64)
