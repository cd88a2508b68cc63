"""Learned per-head attention sinks on the GPU against the float64 oracle.

A sink is one extra logit per query head in the softmax's denominator whose
value row is zero ("Attention variants: what to open up, and how far",
TensorCAD, variants table, row "Attention sinks"; section
"Recommendation": sinks as a parameter of the primitive).  Every kernel
family takes it: the two-tile and split-row tcgen05 prefill kernels (d = 64,
128, 256, with and without soft-cap), the row-wise kernel (dense weights,
other head dims), the paged split-KV decode kernels and the row-wise paged
path."""

import numpy as np
import pytest

from tests._util import (check_out, check_stat, cuda_ok, ensure_built,
                         fullsize_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _rand(g, *shape, gain=1.0):
    import torch
    return (torch.randn(*shape, generator=g) * gain).to(torch.bfloat16)


def _sinks(g, Hq, with_neg_inf=False):
    import torch
    s = torch.randn(Hq, generator=g) * 2.0
    if with_neg_inf:
        s[0] = float("-inf")
    return s.float()


CASES = [
    # B, Hq, Hkv, Tq, Tk, d, causal, window, softcap
    (1, 4, 2, 300, 300, 128, True, 0, 0.0),     # two-tile kernel
    (1, 6, 2, 260, 260, 128, True, 0, 0.0),     # odd group: split-row kernel
    (2, 4, 2, 200, 200, 64, False, 0, 0.0),
    (1, 2, 1, 320, 320, 256, True, 128, 30.0),  # d = 256, window, soft-cap
    (1, 4, 2, 256, 256, 128, True, 0, 20.0),    # two-tile kernel, soft-cap
    (1, 4, 2, 300, 120, 128, True, 0, 0.0),     # rows with no visible key
    (1, 4, 2, 70, 90, 40, True, 0, 0.0),        # row-wise kernel
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_sinks_prefill(case):
    import torch
    import oracle
    from alternative_normalizers_b200 import attention, nattn_get_device_status
    B, Hq, Hkv, Tq, Tk, d, causal, window, cap = case
    g = torch.Generator().manual_seed(555 + Tq + d + Hq)
    q, k, v = _rand(g, B, Hq, Tq, d), _rand(g, B, Hkv, Tk, d), _rand(g, B, Hkv, Tk, d)
    sinks = _sinks(g, Hq, with_neg_inf=(Hq == 6))
    out, st, _ = attention(q.cuda(), k.cuda(), v.cuda(), normalizer="softmax",
                           causal=causal, window=window, softcap=cap,
                           sinks=sinks.cuda())
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    o, s, _ = oracle.attention_fwd(q, k, v, d ** -0.5, "softmax", causal,
                                   window, cap, sinks=sinks)
    check_out(out.float().cpu().numpy(), o, str(case))
    check_stat(st.cpu().numpy(), s, str(case))


def test_sinks_dense_weights():
    """Dense weights with sinks: each row sums to 1 - exp(s_h - row_stat)."""
    import torch
    import oracle
    from alternative_normalizers_b200 import attention
    g = torch.Generator().manual_seed(8)
    q, k, v = _rand(g, 1, 2, 64, 32), _rand(g, 1, 1, 64, 32), _rand(g, 1, 1, 64, 32)
    sinks = _sinks(g, 2)
    out, st, w = attention(q.cuda(), k.cuda(), v.cuda(), normalizer="softmax",
                           causal=True, want_weights=True, sinks=sinks.cuda())
    o, s, ww = oracle.attention_fwd(q, k, v, 32 ** -0.5, "softmax", True,
                                    want_weights=True, sinks=sinks)
    w = w.cpu().numpy()
    check_out(out.float().cpu().numpy(), o)
    check_stat(st.cpu().numpy(), s)
    assert np.abs(w - ww).max() < 2e-3
    assert np.all(w[..., ~oracle.allowed_matrix(64, 64, True, 0)] == 0.0)


@pytest.mark.parametrize("Tq,group", [(1, 4), (2, 8), (5, 4)])
def test_sinks_paged(Tq, group):
    import torch
    import oracle
    from alternative_normalizers_b200 import nattn_get_device_status, paged_attention
    B, Hkv, d, page = 4, 2, 128, 64
    Hq = Hkv * group
    g = torch.Generator().manual_seed(91 + Tq * group)
    lens = torch.randint(1, 800, (B,), generator=g)
    npg = (lens + page - 1) // page
    P = int(npg.sum())
    q = _rand(g, B, Hq, Tq, d)
    kp, vp = _rand(g, P, Hkv, page, d), _rand(g, P, Hkv, page, d)
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = torch.full((B, int(npg.max())), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += int(npg[b])
    lens = lens.to(torch.int32)
    sinks = _sinks(g, Hq)
    out, st = paged_attention(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                              lens.cuda(), 800, normalizer="softmax",
                              sinks=sinks.cuda())
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    res = oracle.paged_decode(q, kp, vp, table, lens, page, d ** -0.5,
                              "softmax", sinks=sinks)
    for b in range(B):
        check_out(out[b].float().cpu().numpy(), res[b][0], f"seq {b}")
        check_stat(st[b].cpu().numpy(), res[b][1], f"seq {b}")


def test_sinks_fullsize_qwen3_prefill():
    """The Qwen3-8B-shaped layer (B=2, Hq=32, Hkv=8, T=4096, d=128, causal)
    with a learned sink per query head; 1024 sampled rows."""
    import torch
    import oracle
    from alternative_normalizers_b200 import attention
    from alternative_normalizers_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS["qwen3_8b_prefill"]
    x = make_inputs(w)
    sinks = _sinks(torch.Generator().manual_seed(3), w.Hq)
    out, st, _ = attention(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(),
                           normalizer="softmax", causal=True, scale=w.scale,
                           sinks=sinks.cuda())
    torch.cuda.synchronize()
    rows = fullsize_rows(w, 1024)
    o, s, _ = oracle.attention_rows(x["q"], x["k"], x["v"], rows, w.scale,
                                    "softmax", True, sinks=sinks)
    out, st = out.float().cpu().numpy(), st.cpu().numpy()
    check_out(out[rows[:, 0], rows[:, 1], rows[:, 2]], o, "qwen3 sinks")
    check_stat(st[rows[:, 0], rows[:, 1], rows[:, 2]], s, "qwen3 sinks")
