"""The backward pass (nattn_bwd) on the GPU against the float64 oracle's
gradients.

The forward runs on the GPU first (its bf16 output and row statistic are
what the backward is given, as in training); the oracle differentiates the
exact forward of the same bf16 inputs.  Tolerance, from the arithmetic:
the kernels round the weights P and the score gradients dS to bf16 for the
tensor cores (relative 2^-9 each), take delta_i = dO_i . O_i from the bf16
forward output (relative 2^-9), and round the gradients to bf16 on output
(relative 2^-9); a few such relative errors of the gradient's magnitude
(measured: about 5e-3 of the largest and 2.4e-3 of the mean magnitude), so
each gradient tensor must satisfy max |err| <= 1e-2 max |ref| and
mean |err| <= 5e-3 mean |ref|."""

import numpy as np
import pytest

from tests._util import cuda_ok, ensure_built

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")
GRAD_MAX_REL = 1e-2
GRAD_MEAN_REL = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _rand(g, *shape, gain=1.0):
    import torch
    return (torch.randn(*shape, generator=g) * gain).to(torch.bfloat16)


def check_grad(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    err = np.abs(got - want)
    scale_max, scale_mean = np.abs(want).max(), np.abs(want).mean()
    print(f"{what}: max err {err.max():.3e} (ref max {scale_max:.3e}), "
          f"mean err {err.mean():.3e} (ref mean {scale_mean:.3e})")
    assert err.max() <= GRAD_MAX_REL * scale_max + 1e-6, what
    assert err.mean() <= GRAD_MEAN_REL * scale_mean + 1e-7, what


def run_case(B, Hq, Hkv, Tq, Tk, d, causal, window, cap, normalizer, seed,
             q_gain=1.0, sinks=None):
    import torch
    import oracle
    from alternative_normalizers_b200 import (attention, attention_backward,
                                              nattn_get_device_status)
    g = torch.Generator().manual_seed(seed)
    q = _rand(g, B, Hq, Tq, d, gain=q_gain)
    k, v = _rand(g, B, Hkv, Tk, d), _rand(g, B, Hkv, Tk, d)
    do = _rand(g, B, Hq, Tq, d)
    sk = None if sinks is None else sinks.cuda()
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, st, _ = attention(qc, kc, vc, normalizer=normalizer, causal=causal,
                           window=window, softcap=cap, sinks=sk)
    dq, dk, dv = attention_backward(qc, kc, vc, out, st, doc, normalizer=normalizer,
                                    causal=causal, window=window, softcap=cap,
                                    sinks=sk)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    rq, rk, rv = oracle.attention_bwd(q, k, v, do, d ** -0.5, normalizer, causal,
                                      window, cap, sinks=sinks)
    tag = f"{normalizer} {(B, Hq, Hkv, Tq, Tk, d, causal, window, cap)}"
    check_grad(dq.float().cpu().numpy(), rq, "dq " + tag)
    check_grad(dk.float().cpu().numpy(), rk, "dk " + tag)
    check_grad(dv.float().cpu().numpy(), rv, "dv " + tag)


CASES = [
    # B, Hq, Hkv, Tq, Tk, d, causal, window, softcap
    (1, 4, 2, 200, 200, 128, True, 0, 0.0),
    (1, 2, 2, 130, 130, 128, False, 0, 0.0),
    (2, 4, 1, 150, 260, 64, True, 0, 0.0),      # Tq != Tk, group of 4
    (1, 2, 1, 256, 256, 128, True, 100, 0.0),   # sliding window
    (1, 2, 1, 192, 192, 64, True, 0, 5.0),      # soft-cap
    (1, 3, 1, 70, 40, 128, True, 0, 0.0),       # rows with no visible key
]


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_backward(case, normalizer):
    run_case(*case, normalizer, seed=77 + case[3] + case[5])


@pytest.mark.parametrize("normalizer", ("sparsemax", "entmax15"))
def test_backward_sparse_narrow_supports(normalizer):
    """Q x 4: supports of a few keys, where the support-mean term matters most."""
    run_case(1, 2, 1, 256, 256, 128, True, 0, 0.0, normalizer, seed=5, q_gain=4.0)


def test_backward_with_sinks():
    import torch
    sinks = torch.tensor([0.5, -1.5, 2.0, float("-inf")])
    run_case(1, 4, 2, 180, 180, 128, True, 0, 0.0, "softmax", seed=9, sinks=sinks)


def test_backward_unsupported_head_dim():
    import torch
    from alternative_normalizers_b200 import NattnError, attention_backward
    x = torch.zeros(1, 2, 16, 256, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, 2, 16, device="cuda")
    with pytest.raises(NattnError):
        attention_backward(x, x, x, x, st, x, normalizer="softmax")


def _rows_grad(x, w, dout, normalizer, b, h, rows):
    """Oracle dZ rows (and weights) of query head h, composed from the
    oracle's row functions: p from the forward row normalizer, dz from its
    Jacobian; returns {i: (visible key indices, p, dS = dz * scale)}."""
    import oracle
    q = oracle.attention._f64(x["q"][b, h])
    g = h // (w.Hq // w.Hkv)
    k = oracle.attention._f64(x["k"][b, g])
    v = oracle.attention._f64(x["v"][b, g])
    do = oracle.attention._f64(dout[b, h])
    ok_all = oracle.allowed_matrix(w.Tq, w.Tk, w.causal, w.window)
    res = {}
    for i in rows:
        idx = np.nonzero(ok_all[i])[0]
        z = oracle.transform_scores(q[i] @ k[idx].T, w.scale, w.softcap)
        p, _ = oracle.normalize_row(z, normalizer)
        dz = oracle.row_vjp(p, do[i] @ v[idx].T, normalizer)
        res[i] = (idx, p, dz * w.scale)
    return res, q, k, do


@pytest.mark.parametrize("name,normalizer", [("qwen3_8b_prefill", "softmax"),
                                             ("sparse_prefill_t1", "sparsemax"),
                                             ("sparse_prefill_t1", "entmax15")])
def test_backward_fullsize(name, normalizer):
    """Full workload size, in the launch configuration the benchmark times:
    dQ on sampled rows, dK / dV on the last key tile of one key/value head
    (seen, under the causal mask, only by the last 128 query rows of each
    head of its group), and for softmax the column-sum identities
    sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i that hold at any size."""
    import torch
    import oracle
    from alternative_normalizers_b200 import attention, attention_backward
    from alternative_normalizers_b200.workloads import WORKLOADS, make_inputs
    from tests._util import fullsize_rows
    w = WORKLOADS[name]
    x = make_inputs(w)
    gen = torch.Generator().manual_seed(w.seed + 500)
    dout = torch.randn(w.B, w.Hq, w.Tq, w.dv, generator=gen).to(torch.bfloat16)
    qc, kc, vc = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    out, st, _ = attention(qc, kc, vc, normalizer=normalizer, causal=w.causal,
                           scale=w.scale)
    dq, dk, dv = attention_backward(qc, kc, vc, out, st, dout.cuda(),
                                    normalizer=normalizer, causal=w.causal,
                                    scale=w.scale)
    torch.cuda.synchronize()
    dq, dk, dv = (t.float().cpu().numpy() for t in (dq, dk, dv))
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()
    # dQ rows
    rows = fullsize_rows(w, 512)
    got, want = [], []
    for (b, h) in sorted({(int(r[0]), int(r[1])) for r in rows}):
        sel = [int(r[2]) for r in rows if r[0] == b and r[1] == h]
        res, q, k, _ = _rows_grad(x, w, dout, normalizer, b, h, sel)
        for i in sel:
            idx, _, ds = res[i]
            want.append(ds @ k[idx])
            got.append(dq[b, h, i])
    check_grad(np.array(got), np.array(want), f"dq rows {name}/{normalizer}")
    # dK, dV of the last key tile of kv head 0 of batch 0
    b, g = 0, 0
    j0 = w.Tk - 128
    group = w.Hq // w.Hkv
    rk = np.zeros((128, w.d))
    rv = np.zeros((128, w.dv))
    for h in range(g * group, (g + 1) * group):
        sel = list(range(j0 - (w.Tk - w.Tq), w.Tq))
        res, q, _, do = _rows_grad(x, w, dout, normalizer, b, h, sel)
        for i in sel:
            idx, p, ds = res[i]
            m = idx >= j0
            rk[idx[m] - j0] += ds[m, None] * q[i][None, :]
            rv[idx[m] - j0] += p[m, None] * do[i][None, :]
    check_grad(dk[b, g, j0:], rk, f"dk last tile {name}/{normalizer}")
    check_grad(dv[b, g, j0:], rv, f"dv last tile {name}/{normalizer}")
    if normalizer == "softmax":
        for b in range(w.B):
            for g in range(w.Hkv):
                s_k = dk[b, g].sum(0)
                assert np.abs(s_k).max() <= 2 ** -7 * np.abs(dk[b, g]).sum(0).max() + 1e-3
                s_v = dv[b, g].sum(0)
                want_v = dout[b, g * group:(g + 1) * group].float().numpy().sum((0, 1))
                assert np.abs(s_v - want_v).max() <= 2 ** -7 * np.abs(dv[b, g]).sum(0).max() + 1e-3
