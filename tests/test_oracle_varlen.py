"""Pins for the oracle's packed variable-length attention
(``varlen_attention``; "HF Attention Normalizers", section "Packed
Variable-Length Attention"), independent of its code:

* sequences of equal lengths are the batched dense problem with the packed
  layout [total, H, d] transposed to [B, H, T, d];
* a single sequence with Tq != Tk keeps the dense oracle's bottom-right
  causal alignment;
* with equal query and key lengths per sequence, packed attention is
  attention over the concatenation under a token-level document mask
  (block-diagonal AND causal inside each document), computed here by brute
  force row by row from the row normalizers.
"""

import numpy as np
import pytest

import oracle
from oracle import attention_fwd, varlen_attention

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")


def _packed(rng, lens_q, lens_k, Hq, Hkv, d):
    tq, tk = sum(lens_q), sum(lens_k)
    return (rng.normal(size=(tq, Hq, d)), rng.normal(size=(tk, Hkv, d)),
            rng.normal(size=(tk, Hkv, d)), np.concatenate([[0], np.cumsum(lens_q)]),
            np.concatenate([[0], np.cumsum(lens_k)]))


@pytest.mark.parametrize("normalizer", NORMS)
def test_equal_lengths_are_the_batched_problem(normalizer):
    rng = np.random.default_rng(1)
    B, T, Hq, Hkv, d = 3, 11, 4, 2, 5
    q, k, v, cq, ck = _packed(rng, [T] * B, [T] * B, Hq, Hkv, d)
    o, s = varlen_attention(q, k, v, cq, ck, 0.6, normalizer, True)
    qb = q.reshape(B, T, Hq, d).transpose(0, 2, 1, 3)
    kb = k.reshape(B, T, Hkv, d).transpose(0, 2, 1, 3)
    vb = v.reshape(B, T, Hkv, d).transpose(0, 2, 1, 3)
    od, sd, _ = attention_fwd(qb, kb, vb, 0.6, normalizer, True)
    np.testing.assert_allclose(o, od.transpose(0, 2, 1, 3).reshape(B * T, Hq, d), atol=1e-12)
    np.testing.assert_allclose(s, sd.transpose(0, 2, 1).reshape(B * T, Hq), atol=1e-12)


@pytest.mark.parametrize("normalizer", NORMS)
def test_single_sequence_bottom_right(normalizer):
    rng = np.random.default_rng(2)
    q, k, v, cq, ck = _packed(rng, [7], [12], 2, 1, 4)
    o, s = varlen_attention(q, k, v, cq, ck, 0.5, normalizer, True, window=4)
    od, sd, _ = attention_fwd(q.transpose(1, 0, 2)[None], k.transpose(1, 0, 2)[None],
                              v.transpose(1, 0, 2)[None], 0.5, normalizer, True, 4)
    np.testing.assert_allclose(o, od[0].transpose(1, 0, 2), atol=1e-12)
    np.testing.assert_allclose(s, sd[0].T, atol=1e-12)


@pytest.mark.parametrize("normalizer", NORMS)
def test_document_mask_brute_force(normalizer):
    rng = np.random.default_rng(3)
    lens = [5, 9, 3]
    q, k, v, cq, ck = _packed(rng, lens, lens, 2, 1, 4)
    o, s = varlen_attention(q, k, v, cq, ck, 0.7, normalizer, True)
    T = sum(lens)
    doc = np.repeat(np.arange(len(lens)), lens)
    ok = (doc[:, None] == doc[None, :]) & (np.arange(T)[None, :] <= np.arange(T)[:, None])
    for h in range(2):
        z = 0.7 * q[:, h] @ k[:, 0].T
        for i in range(T):
            p, st = oracle.normalize_row(z[i][ok[i]], normalizer)
            np.testing.assert_allclose(o[i, h], p @ v[ok[i], 0], atol=1e-12)
            assert abs(s[i, h] - st) < 1e-12
