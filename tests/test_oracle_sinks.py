"""Pins for the oracle's learned-sink softmax (``softmax_sink_row``), each
independent of the oracle's code.

The sink is a learned per-head logit in the softmax's denominator ("Attention
variants: what to open up, and how far", TensorCAD, variants table, row
"Attention sinks").  Fixed by the definition and the mathematics:

* torch's float64 softmax / logsumexp over the row with the sink logit
  appended (a library routine) gives the weights and the row statistic;
* the weight left for the sink, 1 - sum p, is exp(s - row_stat);
* shifting every logit and the sink together changes nothing but the
  row statistic (by the shift);
* s = 0 reduces to softmax1 and s = -inf to softmax (both pinned elsewhere);
* in attention, the sink of head h is one more key whose score is exactly
  s_h and whose value row is zero (built here with one-hot query and key
  columns), which also pins the per-head indexing of the sinks.
A planted mistake (sink term in the numerator as well) is rejected.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention_fwd, softmax_sink_row

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


@pytest.mark.parametrize("seed", range(6))
def test_sink_row_matches_torch_softmax_of_appended_row(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    z = rng.normal(0, 3, n)
    s = float(rng.normal(0, 3))
    p, st = softmax_sink_row(z, s)
    full = torch.tensor(np.append(z, s), dtype=torch.float64)
    want = torch.softmax(full, 0).numpy()
    np.testing.assert_allclose(p, want[:n], rtol=1e-13, atol=1e-16)
    assert abs(st - float(torch.logsumexp(full, 0))) < 1e-12
    # what the sink keeps for itself
    assert abs((1 - p.sum()) - math.exp(s - st)) < 1e-12
    # shift invariance
    p2, st2 = softmax_sink_row(z + 7.5, s + 7.5)
    np.testing.assert_allclose(p2, p, rtol=1e-12)
    assert abs(st2 - st - 7.5) < 1e-12


def test_sink_row_special_cases():
    z = np.array([1.0, -0.5, 2.25, 0.0])
    np.testing.assert_allclose(softmax_sink_row(z, 0.0)[0], oracle.softmax1_row(z)[0],
                               rtol=1e-14)
    np.testing.assert_allclose(softmax_sink_row(z, -math.inf)[0],
                               oracle.softmax_row(z)[0], rtol=1e-14)
    # empty row: no weights, the statistic is the sink itself
    p, st = softmax_sink_row(np.zeros(0), 1.25)
    assert p.size == 0 and st == 1.25
    p, st = softmax_sink_row(np.zeros(0), -math.inf)
    assert p.size == 0 and st == -math.inf
    # a very large sink takes almost all the mass
    p, _ = softmax_sink_row(z, 60.0)
    assert p.sum() < 1e-20


@pytest.mark.parametrize("causal", [False, True])
def test_sink_attention_equals_softmax_with_a_sink_key(causal):
    """Head h's sink as a real key: key 0 is one-hot in column 0 with a zero
    value row, the other keys have column 0 zeroed, and query column 0 holds
    s_h (scale 1), so key 0 scores exactly s_h for every row of head h and no
    other score changes.  Softmax over that input equals the sink softmax over
    the original keys (bottom-right causal keeps key 0 visible to all)."""
    rng = np.random.default_rng(21)
    B, Hq, Hkv, T, d = 2, 4, 2, 9, 6
    q = rng.normal(size=(B, Hq, T, d))
    k = rng.normal(size=(B, Hkv, T, d))
    v = rng.normal(size=(B, Hkv, T, d))
    sinks = np.array([0.7, -1.3, 2.2, -0.4])
    k[..., 0] = 0.0
    q[..., 0] = sinks[None, :, None]
    o1, s1, _ = attention_fwd(q, k, v, 1.0, "softmax", causal, sinks=sinks)
    k0 = np.zeros((B, Hkv, 1, d))
    k0[..., 0] = 1.0
    kk = np.concatenate([k0, k], axis=2)
    vv = np.concatenate([np.zeros((B, Hkv, 1, d)), v], axis=2)
    o0, s0, _ = attention_fwd(q, kk, vv, 1.0, "softmax", causal)
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    np.testing.assert_allclose(s1, s0, atol=1e-12)


def _sink_in_numerator_too(z, s):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(np.append(z, s))
    return e[:-1] / e.sum() + math.exp(s) / e.sum() / max(1, z.size), 0.0


def test_planted_sink_mistake_is_caught():
    z = np.array([0.4, -1.0, 1.5])
    s = 0.9
    full = torch.tensor(np.append(z, s), dtype=torch.float64)
    want = torch.softmax(full, 0).numpy()[:3]
    assert np.abs(softmax_sink_row(z, s)[0] - want).max() < 1e-14
    assert np.abs(_sink_in_numerator_too(z, s)[0] - want).max() > 1e-3
    assert np.abs(oracle.softmax_row(z)[0] - want).max() > 1e-3
