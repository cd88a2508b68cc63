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


def workload_seed(name):
    """Fixed per-workload seed for row sampling (crc32 of the name): the same
    rows are checked on every run and in every process."""
    import zlib
    return zlib.crc32(name.encode()) & 0xFFFF


def fullsize_rows(w, n=1024):
    """At least ``n`` seeded (b, h, i) rows of a full-size dense workload:
    every head of one GQA group at the first and last rows of the first,
    middle and last 128-row tiles; first/last rows of a few more tiles;
    rows at and around the window edge when there is a window; then uniform
    picks up to ``n``."""
    rng = np.random.default_rng(workload_seed(w.name))
    group = w.Hq // w.Hkv
    extra = []
    ntile = (w.Tq + 127) // 128
    tiles = sorted({0, ntile // 2, ntile - 1} |
                   set(rng.choice(ntile, min(ntile, 6), replace=False).tolist()))
    h_edge = int(rng.integers(0, w.Hq))
    for t in tiles:
        for i in (128 * t, 128 * t + 127):
            if i < w.Tq:
                extra.append((int(rng.integers(0, w.B)), h_edge, i))
    if w.window:
        for i in (w.window - 2, w.window - 1, w.window, w.window + 1,
                  w.window + 127, w.window + 128):
            if 0 <= i < w.Tq:
                for h in (0, w.Hq - 1):
                    extra.append((w.B - 1, h, i))
    return sample_rows(w.B, w.Hq, w.Tq, n, seed=workload_seed(w.name) + 1,
                       group=group, extra=extra)


def compact_pool(k_pool, v_pool, block_table, seqlens, seqs, page_size):
    """The pages the sequences ``seqs`` use, copied into a small pool with a
    renumbered block table (rows of other sequences left as they are), so
    the oracle upcasts only what it reads.  Pure re-indexing."""
    import torch
    lens = [int(x) for x in seqlens]
    pages = sorted({int(block_table[b, p]) for b in seqs
                    for p in range(-(-lens[b] // page_size))})
    remap = {p: i for i, p in enumerate(pages)}
    table = block_table.clone()
    for b in seqs:
        for p in range(-(-lens[b] // page_size)):
            table[b, p] = remap[int(block_table[b, p])]
    idx = torch.tensor(pages, dtype=torch.long)
    return k_pool[idx], v_pool[idx], table
