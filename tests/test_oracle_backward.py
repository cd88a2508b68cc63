"""Pins for the float64 backward oracle (``oracle.backward``), each
independent of its code:

* central finite differences of the forward oracle's loss
  ``L = sum(dout * O)`` with respect to every entry of q, k and v, for all
  four normalizers and learned sinks, with causal / window / soft-cap masks,
  grouped-query heads and Tq != Tk (the forward is pinned on its own);
* torch's float64 autograd through ``scaled_dot_product_attention`` (math
  backend) for softmax;
* each row's vector-Jacobian product against the explicit Jacobian of the
  row function, built by finite differences;
* planted mistakes (sparsemax without the support-mean term; 1.5-entmax
  weighted by p instead of sqrt(p); softmax without the sum term) are
  rejected by the finite-difference pin.
"""

import numpy as np
import pytest

import oracle
from oracle import attention_fwd
from oracle import backward as bwd

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")


def _problem(seed, B=1, Hq=4, Hkv=2, Tq=5, Tk=7, d=3, dv=2, gain=1.5):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(B, Hq, Tq, d)) * gain, rng.normal(size=(B, Hkv, Tk, d)) * gain,
            rng.normal(size=(B, Hkv, Tk, dv)), rng.normal(size=(B, Hq, Tq, dv)))


def _fd_grads(q, k, v, dout, scale, normalizer, causal, window, softcap, sinks=None,
              eps=1e-6):
    def loss(q_, k_, v_):
        o, _, _ = attention_fwd(q_, k_, v_, scale, normalizer, causal, window, softcap,
                                sinks=sinks)
        return float((o * dout).sum())
    grads = []
    for which in range(3):
        base = [q.copy(), k.copy(), v.copy()]
        x = base[which]
        g = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            x0 = x[idx]
            x[idx] = x0 + eps
            lp = loss(*base)
            x[idx] = x0 - eps
            lm = loss(*base)
            x[idx] = x0
            g[idx] = (lp - lm) / (2 * eps)
        grads.append(g)
    return grads


CONFIGS = [  # causal, window, softcap, Tq, Tk
    (False, 0, 0.0, 5, 7), (True, 0, 0.0, 5, 7), (True, 3, 1.0, 6, 6),
    (False, 2, 0.0, 4, 4)]


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_finite_differences(normalizer, cfg):
    causal, window, cap, Tq, Tk = cfg
    q, k, v, dout = _problem(7 + Tq + 3 * window, Tq=Tq, Tk=Tk)
    scale = 0.8
    got = bwd.attention_bwd(q, k, v, dout, scale, normalizer, causal, window, cap)
    want = _fd_grads(q, k, v, dout, scale, normalizer, causal, window, cap)
    for g, w, name in zip(got, want, "qkv"):
        np.testing.assert_allclose(g, w, atol=2e-7, err_msg=name)


def test_backward_with_sinks_matches_finite_differences():
    q, k, v, dout = _problem(31)
    sinks = np.array([0.5, -1.0, 1.7, float("-inf")])
    got = bwd.attention_bwd(q, k, v, dout, 0.7, "softmax", True, 0, 0.0, sinks=sinks)
    want = _fd_grads(q, k, v, dout, 0.7, "softmax", True, 0, 0.0, sinks=sinks)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, atol=2e-7)


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_backward_matches_torch_autograd(causal):
    torch = pytest.importorskip("torch")
    q, k, v, dout = _problem(41, B=2, Hq=4, Hkv=2, Tq=6, Tk=9, d=5, dv=4)
    scale = 0.45
    dq, dk, dv = bwd.attention_bwd(q, k, v, dout, scale, "softmax", causal)
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    m = torch.tensor(oracle.allowed_matrix(6, 9, causal, 0))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(2, dim=1), vt.repeat_interleave(2, dim=1),
        attn_mask=m, scale=scale)
    (o * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-12)


@pytest.mark.parametrize("normalizer", NORMS)
def test_row_vjp_matches_explicit_jacobian(normalizer):
    rng = np.random.default_rng(5)
    for _ in range(20):
        n = int(rng.integers(1, 9))
        z = rng.normal(0, 1.5, n)
        g = rng.normal(size=n)
        p, _ = oracle.normalize_row(z, normalizer)
        J = np.zeros((n, n))        # J[i, j] = dp_i / dz_j
        eps = 1e-7
        for j in range(n):
            e = np.zeros(n)
            e[j] = eps
            J[:, j] = (oracle.normalize_row(z + e, normalizer)[0] -
                       oracle.normalize_row(z - e, normalizer)[0]) / (2 * eps)
        np.testing.assert_allclose(bwd.row_vjp(p, g, normalizer), J.T @ g, atol=1e-6)


def _vjp_no_mean(p, g, normalizer):
    return (np.asarray(p) > 0) * np.asarray(g)


def _vjp_entmax_by_p(p, g, normalizer):
    s = np.asarray(p)
    return s * (g - np.dot(s, g) / s.sum())


def _vjp_softmax_no_sum(p, g, normalizer):
    return np.asarray(p) * np.asarray(g)


@pytest.mark.parametrize("normalizer,mistake", [
    ("sparsemax", _vjp_no_mean), ("entmax15", _vjp_entmax_by_p),
    ("softmax", _vjp_softmax_no_sum)])
def test_planted_backward_mistakes_are_caught(normalizer, mistake, monkeypatch):
    q, k, v, dout = _problem(19)
    want = _fd_grads(q, k, v, dout, 0.9, normalizer, True, 0, 0.0)
    good = bwd.attention_bwd(q, k, v, dout, 0.9, normalizer, True)
    assert all(np.abs(g - w).max() < 2e-7 for g, w in zip(good, want))
    monkeypatch.setattr(bwd, "row_vjp", mistake)
    bad = bwd.attention_bwd(q, k, v, dout, 0.9, normalizer, True)
    assert max(np.abs(g - w).max() for g, w in zip(bad, want)) > 1e-3


@pytest.mark.parametrize("normalizer", NORMS)
def test_backward_with_block_mask_matches_finite_differences(normalizer):
    """A block mask drops whole 128 x 128 blocks: central differences of the
    forward oracle on a sample of coordinates of q, k and v."""
    rng = np.random.default_rng(23)
    B, Hq, Hkv, T, d = 1, 2, 1, 260, 3
    q = rng.normal(size=(B, Hq, T, d)) * 1.5
    k = rng.normal(size=(B, Hkv, T, d)) * 1.5
    v = rng.normal(size=(B, Hkv, T, d))
    dout = rng.normal(size=(B, Hq, T, d))
    bm = np.array([[[[1, 0, 1], [0, 1, 1], [1, 1, 0]],
                    [[1, 1, 1], [1, 0, 1], [0, 1, 1]]]], dtype=np.uint8)
    got = bwd.attention_bwd(q, k, v, dout, 0.8, normalizer, True, block_mask=bm)

    def loss(q_, k_, v_):
        o, _, _ = attention_fwd(q_, k_, v_, 0.8, normalizer, True, block_mask=bm)
        return float((o * dout).sum())
    eps = 1e-6
    for which, x in enumerate((q, k, v)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in x.shape)
            base = [q.copy(), k.copy(), v.copy()]
            base[which][idx] += eps
            lp = loss(*base)
            base[which][idx] -= 2 * eps
            lm = loss(*base)
            assert abs((lp - lm) / (2 * eps) - got[which][idx]) < 2e-7
