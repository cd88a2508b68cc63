"""Pins for the oracle's block mask (whole 128 x 128 blocks of (query, key)
pairs kept or dropped on top of the causal / window rule; "Attention
variants", TensorCAD, section "C. Keep the fused kernel": a mask yields a
block mask whose masked-out blocks are skipped), independent of its code:

* an all-ones block mask changes nothing;
* a block-diagonal mask over documents whose boundaries fall on block edges
  (document masking for packed sequences) equals attention run separately
  on each document's slice of the inputs;
* a row whose blocks are all dropped has no visible key (output 0, the
  normalizer's empty-row statistic);
* the expanded mask, brute force over (i, j), is the elementwise AND.
A planted mistake (block index taken from the key for the query) is caught.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import attention_fwd, block_allowed

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")


def _rand(rng, *shape):
    return rng.normal(size=shape)


def test_block_allowed_brute_force():
    rng = np.random.default_rng(1)
    bm = rng.integers(0, 2, size=(3, 4))
    got = block_allowed(bm, 300, 450)
    for i in range(0, 300, 7):
        for j in range(0, 450, 11):
            assert got[i, j] == bool(bm[i // 128, j // 128])


def _planted(bm, Tq, Tk):
    bm = np.asarray(bm) != 0
    return bm[np.arange(Tq)[:, None] // 128, np.arange(Tk)[None, :] // 128].T \
        if Tq == Tk else None


def test_planted_transposed_block_index_is_caught():
    bm = np.array([[1, 0], [1, 1]])
    assert not np.array_equal(block_allowed(bm, 256, 256), _planted(bm, 256, 256))


@pytest.mark.parametrize("normalizer", NORMS)
def test_all_ones_block_mask_is_no_mask(normalizer):
    rng = np.random.default_rng(2)
    q, k, v = _rand(rng, 1, 2, 200, 8), _rand(rng, 1, 1, 200, 8), _rand(rng, 1, 1, 200, 8)
    bm = np.ones((1, 2, 2, 2), dtype=np.uint8)
    a = attention_fwd(q, k, v, 0.4, normalizer, True)
    b = attention_fwd(q, k, v, 0.4, normalizer, True, block_mask=bm)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("normalizer", NORMS)
def test_block_diagonal_mask_is_document_masking(normalizer):
    """Two documents of 256 and 128 tokens packed into one sequence of 384:
    the block-diagonal block mask gives each document's rows exactly the
    attention over its own keys."""
    rng = np.random.default_rng(3)
    T, d = 384, 8
    q, k, v = _rand(rng, 1, 2, T, d), _rand(rng, 1, 1, T, d), _rand(rng, 1, 1, T, d)
    bm = np.zeros((1, 2, 3, 3), dtype=np.uint8)
    bm[..., :2, :2] = 1
    bm[..., 2, 2] = 1
    for causal in (False, True):
        o, s, _ = attention_fwd(q, k, v, 0.5, normalizer, causal, block_mask=bm)
        for lo, hi in ((0, 256), (256, 384)):
            od, sd, _ = attention_fwd(q[:, :, lo:hi], k[:, :, lo:hi], v[:, :, lo:hi], 0.5,
                                      normalizer, causal)
            np.testing.assert_allclose(o[:, :, lo:hi], od, atol=1e-12)
            np.testing.assert_allclose(s[:, :, lo:hi], sd, atol=1e-12)


def test_fully_dropped_rows_are_empty():
    rng = np.random.default_rng(4)
    q, k, v = _rand(rng, 1, 1, 256, 8), _rand(rng, 1, 1, 256, 8), _rand(rng, 1, 1, 256, 8)
    bm = np.ones((1, 1, 2, 2), dtype=np.uint8)
    bm[0, 0, 1, :] = 0                      # rows 128..255 keep no block
    want_stat = {"softmax": -math.inf, "softmax1": 0.0, "sparsemax": math.inf,
                 "entmax15": math.inf}
    for n, st in want_stat.items():
        o, s, w = attention_fwd(q, k, v, 0.3, n, False, want_weights=True, block_mask=bm)
        assert np.all(o[0, 0, 128:] == 0) and np.all(s[0, 0, 128:] == st)
        assert np.all(w[0, 0, :128, :] >= 0) and np.all(w[0, 0, 128:] == 0)
