"""Pins for the float64 oracle, each independent of the oracle's own code.

The oracle restates the definitions of the "HF Attention Normalizers" page
("Supported Normalizers" table, "Important Limitations") and the masking /
soft-cap rules of the other pages.  These tests tie it to facts fixed by the
mathematics or by an independent library, never to itself:

* hand-derived worked rows (tests/golden/worked_rows.json),
* two-element closed forms, uniform rows, shift invariance,
* brute-force support enumeration with the KKT conditions (n <= 8),
* the variational definitions (projection onto the simplex; Tsallis-1.5
  regularised argmax) checked against random feasible points,
* independent float64 bisection on the threshold equation,
* torch's float64 ``scaled_dot_product_attention`` (math backend) for the
  softmax attention wiring (scale, transpose, mask, GQA expansion),
* the softmax1 <-> softmax-with-a-zero-key identity,
* the worked ``and_masks(causal, window)`` example, brute-force masks,
* the paged gather against the dense layout it stores.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import (allowed_matrix, attention_fwd, attention_rows,
                    entmax15_row, normalize_row, paged_decode, softmax1_row,
                    softmax_row, sparsemax_row, transform_scores)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ------------------------------------------------------------------ golden

def test_worked_rows():
    with open(os.path.join(GOLDEN, "worked_rows.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        p, st = normalize_row(np.array(c["z"]), c["normalizer"])
        np.testing.assert_allclose(p, c["p"], atol=1e-12, err_msg=c["why"])
        assert abs(st - c["stat"]) < 1e-12, c["why"]


def test_mask_worked_example():
    path = os.path.join(GOLDEN, "mask_causal_window4_6x6.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    want = np.array(rows, dtype=int).astype(bool)
    got = allowed_matrix(6, 6, causal=True, window=4)
    assert got.shape == (6, 6)
    np.testing.assert_array_equal(got, want)


def test_mask_brute_force():
    rng = np.random.default_rng(0)
    for _ in range(40):
        Tq = int(rng.integers(1, 12))
        Tk = int(rng.integers(1, 12))
        causal = bool(rng.integers(0, 2))
        window = int(rng.integers(0, 6))
        got = allowed_matrix(Tq, Tk, causal, window)
        for i in range(Tq):
            for j in range(Tk):
                pos = i + Tk - Tq          # bottom-right aligned position
                want = True
                if causal and not j <= pos:
                    want = False
                if window:
                    dist = pos - j if causal else abs(pos - j)
                    if not dist < window:
                        want = False
                assert got[i, j] == want, (Tq, Tk, causal, window, i, j)


def test_window_counts_w_keys_including_diagonal():
    ok = allowed_matrix(10, 10, causal=True, window=3)
    assert ok.sum(1).tolist() == [1, 2, 3, 3, 3, 3, 3, 3, 3, 3]


# ------------------------------------------------------------------ softmax

def test_softmax_matches_scipy():
    from scipy.special import logsumexp, softmax
    rng = np.random.default_rng(1)
    for n in (1, 2, 7, 100):
        z = rng.normal(size=n) * 5
        p, lse = softmax_row(z)
        np.testing.assert_allclose(p, softmax(z), rtol=1e-13)
        assert abs(lse - logsumexp(z)) < 1e-12


def test_softmax1_identity_rows():
    from scipy.special import logsumexp, softmax
    rng = np.random.default_rng(2)
    for n in (1, 3, 50):
        for shift in (-30.0, 0.0, 30.0):
            z = rng.normal(size=n) + shift
            p, lse = softmax1_row(z)
            ext = np.concatenate([z, [0.0]])
            np.testing.assert_allclose(p, softmax(ext)[:n], rtol=1e-12,
                                       atol=1e-300)
            assert abs(lse - logsumexp(ext)) < 1e-12
            s = np.exp(z).sum()
            assert abs(p.sum() - s / (1 + s)) < 1e-12
            assert p.sum() < 1.0


def test_empty_rows():
    e = np.zeros(0)
    assert softmax_row(e)[1] == -math.inf
    assert softmax1_row(e)[1] == 0.0
    assert sparsemax_row(e)[1] == math.inf
    assert entmax15_row(e)[1] == math.inf


# ------------------------------------------------------------------ sparsemax

def _bisect(f, lo, hi, it=200):
    for _ in range(it):
        mid = 0.5 * (lo + hi)
        if f(mid) >= 1.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_sparsemax_two_elements_closed_form():
    for a, b in [(0.0, 0.0), (0.3, 0.1), (1.0, 0.0), (0.0, 2.5), (-1, -1.4)]:
        p, _ = sparsemax_row(np.array([a, b]))
        p1 = min(max((1 + a - b) / 2, 0.0), 1.0)
        np.testing.assert_allclose(p, [p1, 1 - p1], atol=1e-14)


def test_sparsemax_uniform_and_shift():
    rng = np.random.default_rng(3)
    for n in (1, 2, 9):
        p, tau = sparsemax_row(np.full(n, 0.7))
        np.testing.assert_allclose(p, np.full(n, 1.0 / n), atol=1e-14)
        assert abs(tau - (0.7 - 1.0 / n)) < 1e-14
    z = rng.normal(size=30)
    p0, t0 = sparsemax_row(z)
    p1, t1 = sparsemax_row(z + 11.0)
    np.testing.assert_allclose(p0, p1, atol=1e-12)
    assert abs(t1 - t0 - 11.0) < 1e-12


def _brute_support(z, tau_of_set, keep):
    """Unique support S whose closed-form threshold satisfies the KKT
    conditions: every member strictly above tau, every other entry at or
    below it."""
    n = len(z)
    found = []
    for r in range(1, n + 1):
        for S in itertools.combinations(range(n), r):
            tau = tau_of_set(z[list(S)])
            if tau is None:
                continue
            inside = all(keep(z[i], tau) for i in S)
            outside = all(not keep(z[j], tau) for j in range(n) if j not in S)
            if inside and outside:
                found.append((set(S), tau))
    return found


def test_sparsemax_brute_force_support():
    rng = np.random.default_rng(4)
    for _ in range(150):
        n = int(rng.integers(1, 9))
        z = rng.normal(size=n) * rng.choice([0.2, 1.0, 3.0])
        found = _brute_support(z, lambda s: (s.sum() - 1.0) / len(s),
                               lambda x, t: x > t)
        assert len(found) == 1
        S, tau = found[0]
        p, t = sparsemax_row(z)
        assert abs(t - tau) < 1e-12
        assert set(np.nonzero(p > 0)[0].tolist()) == S


def test_sparsemax_is_projection():
    rng = np.random.default_rng(5)
    for _ in range(50):
        n = int(rng.integers(2, 20))
        z = rng.normal(size=n) * 2
        p, _ = sparsemax_row(z)
        assert abs(p.sum() - 1) < 1e-12 and (p >= 0).all()
        best = ((p - z) ** 2).sum()
        for x in rng.dirichlet(np.ones(n) * 0.3, size=200):
            assert best <= ((x - z) ** 2).sum() + 1e-12


def test_sparsemax_bisection():
    rng = np.random.default_rng(6)
    for _ in range(30):
        z = rng.normal(size=int(rng.integers(1, 300))) * 3
        _, tau = sparsemax_row(z)
        f = lambda t: np.maximum(z - t, 0).sum()
        tb = _bisect(f, z.max() - 1.0, z.max())
        assert abs(tau - tb) < 1e-10


# ------------------------------------------------------------------ entmax15

def _entmax_tau_of_set(u):
    k = len(u)
    mu = u.mean()
    delta = (1.0 - k * (np.mean(u * u) - mu * mu)) / k
    if delta < 0:
        return None
    return mu - math.sqrt(delta)


def test_entmax15_two_elements_closed_form():
    for a, b in [(0.0, 0.0), (0.8, 0.1), (2.0, 0.0), (0.3, 1.9), (5, 0)]:
        p, _ = entmax15_row(np.array([a, b]))
        hi, lo = max(a, b), min(a, b)
        delta = (hi - lo) / 2
        if delta >= 1:
            want = (1.0, 0.0)
        else:
            x = (delta + math.sqrt(2 - delta * delta)) / 2
            want = (x * x, (x - delta) ** 2)
        if a < b:
            want = want[::-1]
        np.testing.assert_allclose(p, want, atol=1e-13)


def test_entmax15_uniform():
    for n in (1, 2, 5, 16):
        p, tau = entmax15_row(np.full(n, 0.9))
        np.testing.assert_allclose(p, np.full(n, 1.0 / n), atol=1e-13)
        assert abs(tau - (0.45 - 1 / math.sqrt(n))) < 1e-13


def test_entmax15_brute_force_support():
    rng = np.random.default_rng(7)
    for _ in range(150):
        n = int(rng.integers(1, 9))
        z = rng.normal(size=n) * rng.choice([0.3, 1.0, 4.0])
        u = z / 2
        found = _brute_support(u, _entmax_tau_of_set, lambda x, t: x > t)
        assert len(found) == 1
        S, tau = found[0]
        p, t = entmax15_row(z)
        assert abs(t - tau) < 1e-12
        assert set(np.nonzero(p > 0)[0].tolist()) == S


def test_entmax15_variational():
    """1.5-entmax maximises <p, z> + (4/3) sum(p - p^1.5) over the simplex
    (Tsallis entropy with alpha = 1.5)."""
    rng = np.random.default_rng(8)
    obj = lambda p, z: p @ z + (4.0 / 3.0) * (p - p ** 1.5).sum()
    for _ in range(50):
        n = int(rng.integers(2, 16))
        z = rng.normal(size=n) * 2
        p, _ = entmax15_row(z)
        assert abs(p.sum() - 1) < 1e-12 and (p >= 0).all()
        best = obj(p, z)
        for x in rng.dirichlet(np.ones(n) * 0.5, size=200):
            assert best >= obj(x, z) - 1e-12


def test_entmax15_bisection():
    rng = np.random.default_rng(9)
    for _ in range(30):
        z = rng.normal(size=int(rng.integers(1, 300))) * 3
        _, tau = entmax15_row(z)
        u = z / 2
        f = lambda t: (np.maximum(u - t, 0) ** 2).sum()
        tb = _bisect(f, u.max() - 1.0, u.max())
        assert abs(tau - tb) < 1e-10


# ------------------------------------------------------------------ attention

def _rand(rng, *shape):
    return rng.normal(size=shape)


@pytest.mark.parametrize("causal,window,Tq,Tk", [
    (False, 0, 9, 9), (True, 0, 9, 9), (True, 3, 9, 9), (True, 0, 5, 12),
    (True, 4, 5, 12), (False, 0, 6, 3)])
def test_softmax_attention_matches_torch_sdpa(causal, window, Tq, Tk):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(10)
    B, Hq, Hkv, d, dv = 2, 4, 2, 8, 5
    q, k, v = _rand(rng, B, Hq, Tq, d), _rand(rng, B, Hkv, Tk, d), \
        _rand(rng, B, Hkv, Tk, dv)
    scale = 0.37
    out, lse, _ = attention_fwd(q, k, v, scale, "softmax", causal, window)
    # torch wiring: expand K/V heads, explicit boolean mask
    kt = torch.tensor(k).repeat_interleave(Hq // Hkv, dim=1)
    vt = torch.tensor(v).repeat_interleave(Hq // Hkv, dim=1)
    pos = torch.arange(Tq)[:, None] + (Tk - Tq)
    j = torch.arange(Tk)[None, :]
    m = torch.ones(Tq, Tk, dtype=torch.bool)
    if causal:
        m &= j <= pos
    if window:
        m &= (pos - j) < window if causal else (pos - j).abs() < window
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), kt, vt, attn_mask=m, scale=scale)
    s = torch.tensor(q) @ kt.transpose(-1, -2) * scale
    ref_lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    full = m.any(dim=1)
    np.testing.assert_allclose(out[:, :, full.numpy()],
                               ref[:, :, full].numpy(), atol=1e-12)
    np.testing.assert_allclose(lse[:, :, full.numpy()],
                               ref_lse[:, :, full].numpy(), atol=1e-12)
    # fully masked rows: zero output, -inf LSE
    assert np.all(out[:, :, ~full.numpy()] == 0)
    assert np.all(lse[:, :, ~full.numpy()] == -np.inf)


def test_softmax1_equals_softmax_with_zero_key():
    """softmax1 is softmax with one extra logit 0 whose value row is 0
    ("Important Limitations": the virtual logit-0/value-0 sink).  Prepending
    a zero key and value and aligning the causal mask bottom-right gives each
    query exactly that extra logit."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, T, d = 1, 4, 2, 13, 8
    q, k, v = _rand(rng, B, Hq, T, d), _rand(rng, B, Hkv, T, d), \
        _rand(rng, B, Hkv, T, d)
    for causal in (False, True):
        o1, s1, _ = attention_fwd(q, k, v, 0.5, "softmax1", causal)
        k0 = np.concatenate([np.zeros((B, Hkv, 1, d)), k], axis=2)
        v0 = np.concatenate([np.zeros((B, Hkv, 1, d)), v], axis=2)
        o0, s0, _ = attention_fwd(q, k0, v0, 0.5, "softmax", causal)
        np.testing.assert_allclose(o1, o0, atol=1e-12)
        np.testing.assert_allclose(s1, s0, atol=1e-12)


@pytest.mark.parametrize("normalizer", oracle.NORMALIZERS)
def test_gqa_equals_expanded_heads(normalizer):
    rng = np.random.default_rng(12)
    B, Hq, Hkv, T, d = 2, 6, 2, 10, 4
    q, k, v = _rand(rng, B, Hq, T, d), _rand(rng, B, Hkv, T, d), \
        _rand(rng, B, Hkv, T, d)
    o, s, _ = attention_fwd(q, k, v, 0.9, normalizer, True)
    ke = np.repeat(k, Hq // Hkv, axis=1)
    ve = np.repeat(v, Hq // Hkv, axis=1)
    oe, se, _ = attention_fwd(q, ke, ve, 0.9, normalizer, True)
    np.testing.assert_array_equal(o, oe)
    np.testing.assert_array_equal(s, se)


@pytest.mark.parametrize("normalizer", oracle.NORMALIZERS)
def test_weights_are_distributions_and_masked_zero(normalizer):
    rng = np.random.default_rng(13)
    q, k, v = _rand(rng, 1, 2, 12, 6), _rand(rng, 1, 1, 12, 6), \
        _rand(rng, 1, 1, 12, 6)
    o, s, w = attention_fwd(q, k, v, 1.0, normalizer, True, 5,
                            want_weights=True)
    ok = allowed_matrix(12, 12, True, 5)
    assert np.all(w[..., ~ok] == 0.0)
    assert np.all(w >= 0)
    sums = w.sum(-1)
    if normalizer == "softmax1":
        assert np.all(sums < 1)
    else:
        np.testing.assert_allclose(sums, 1.0, atol=1e-12)
    np.testing.assert_allclose(o, w @ v[0, 0], atol=1e-12)


def test_softcap_transform():
    s = np.linspace(-500, 500, 101)
    z = transform_scores(s, 0.5, 50.0)
    assert np.all(np.abs(z) < 50.0)
    np.testing.assert_allclose(z, 50 * np.tanh(0.5 * s / 50), atol=1e-12)
    np.testing.assert_allclose(transform_scores(s, 0.5, 0.0), 0.5 * s)
    # a huge cap leaves the scores unchanged up to rounding
    np.testing.assert_allclose(transform_scores(s, 0.5, 1e9), 0.5 * s,
                               rtol=1e-9)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(14)
    q, k, v = _rand(rng, 2, 4, 7, 3), _rand(rng, 2, 2, 9, 3), \
        _rand(rng, 2, 2, 9, 5)
    o, s, _ = attention_fwd(q, k, v, 0.7, "entmax15", True, 4)
    rows = np.array([[1, 3, 6], [0, 0, 0], [1, 0, 2]])
    o2, s2, _ = attention_rows(q, k, v, rows, 0.7, "entmax15", True, 4)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(o2[r], o[b, h, i])
        assert s2[r] == s[b, h, i]


@pytest.mark.parametrize("normalizer", oracle.NORMALIZERS)
def test_paged_decode_matches_dense(normalizer):
    """Scatter dense per-sequence K/V into a shuffled page pool by hand and
    check that decoding through the block table equals dense attention."""
    rng = np.random.default_rng(15)
    B, Hq, Hkv, d, page = 3, 4, 2, 8, 4
    lens = [5, 12, 1]
    npages = [-(-L // page) for L in lens]
    P = sum(npages)
    perm = rng.permutation(P)
    table = -np.ones((B, max(npages)), dtype=np.int64)
    kpool = rng.normal(size=(P, Hkv, page, d))
    vpool = rng.normal(size=(P, Hkv, page, d))
    q = rng.normal(size=(B, Hq, 1, d))
    dense_k, dense_v = [], []
    off = 0
    for b, L in enumerate(lens):
        kb = rng.normal(size=(Hkv, L, d))
        vb = rng.normal(size=(Hkv, L, d))
        for p in range(npages[b]):
            table[b, p] = perm[off]
            n = min(page, L - p * page)
            kpool[perm[off], :, :n] = kb[:, p * page:p * page + n]
            vpool[perm[off], :, :n] = vb[:, p * page:p * page + n]
            off += 1
        dense_k.append(kb)
        dense_v.append(vb)
    res = paged_decode(q, kpool, vpool, table, lens, page, 0.5, normalizer)
    for b in range(B):
        o, s, _ = attention_fwd(q[b:b + 1], dense_k[b][None],
                                dense_v[b][None], 0.5, normalizer, True)
        np.testing.assert_allclose(res[b][0], o[0], atol=1e-12)
        np.testing.assert_allclose(res[b][1], s[0], atol=1e-12)


def _rows_ok(fn, kind):
    """Brute-force KKT check of a row function on random rows."""
    rng = np.random.default_rng(16)
    for _ in range(40):
        n = int(rng.integers(1, 7))
        z = rng.normal(size=n) * 1.5
        if kind == "sparsemax":
            found = _brute_support(z, lambda s: (s.sum() - 1.0) / len(s),
                                   lambda x, t: x > t)
        else:
            found = _brute_support(z / 2, _entmax_tau_of_set,
                                   lambda x, t: x > t)
        p, t = fn(z)
        if len(found) != 1 or abs(t - found[0][1]) > 1e-9:
            return False
        if abs(p.sum() - 1) > 1e-9:
            return False
    return True


def _sparsemax_no_minus_one(z):
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    k = np.arange(1, z.size + 1)
    kstar = int(np.nonzero(1 + k * zs > cs)[0].max()) + 1
    tau = cs[kstar - 1] / kstar
    return np.maximum(z - tau, 0), tau


def _entmax_without_half(z):
    p, tau = entmax15_row(2.0 * np.asarray(z))
    return p, tau


def _entmax_larger_root(z):
    u = np.asarray(z) / 2
    us = np.sort(u)[::-1]
    k = np.arange(1, u.size + 1)
    mean = np.cumsum(us) / k
    delta = (1 - k * (np.cumsum(us * us) / k - mean ** 2)) / k
    tau_k = mean + np.sqrt(np.maximum(delta, 0))
    ok = (delta >= 0) & (tau_k < us)
    kstar = int(np.nonzero(ok)[0].max()) + 1 if ok.any() else 1
    tau = tau_k[kstar - 1]
    return np.maximum(u - tau, 0) ** 2, tau


def test_planted_mistakes_are_caught():
    """Plant plausible slips in copies of the row functions (on the CPU) and
    check that the brute-force pins reject every one while accepting the
    oracle."""
    assert _rows_ok(sparsemax_row, "sparsemax")
    assert _rows_ok(entmax15_row, "entmax15")
    assert not _rows_ok(_sparsemax_no_minus_one, "sparsemax")
    assert not _rows_ok(_entmax_without_half, "entmax15")
    assert not _rows_ok(_entmax_larger_root, "entmax15")
    # softmax1 without its sink breaks the S/(1+S) row-sum invariant
    z = np.array([1.0, 0.5, -1.0])
    s = np.exp(z).sum()
    assert abs(softmax_row(z)[0].sum() - s / (1 + s)) > 1e-3
    assert abs(softmax1_row(z)[0].sum() - s / (1 + s)) < 1e-12
    # an off-by-one window (q - k <= W) breaks the worked mask example
    path = os.path.join(GOLDEN, "mask_causal_window4_6x6.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    want = np.array(rows, dtype=int).astype(bool)
    assert not np.array_equal(allowed_matrix(6, 6, True, 5), want)
