"""Packed variable-length attention and paged prefill on the GPU against the
float64 oracle.

Packed mode ("HF Attention Normalizers", section "Packed Variable-Length
Attention"): q [total_q, Hq, d], k / v [total_k, Hkv, d] with cumulative
sequence lengths, per-request bottom-right causal alignment, one grid over
the packed batch.  Paged prefill ("Differentiable Paged Attention"): a chunk
of new tokens per sequence against a page pool, on the tensor-core kernels
when there are more rows per key/value head than the decode kernels take."""

import numpy as np
import pytest

from tests._util import check_out, check_stat, compact_pool, cuda_ok, ensure_built

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _rand(g, *shape, gain=1.0):
    import torch
    return (torch.randn(*shape, generator=g) * gain).to(torch.bfloat16)


VARLEN = [
    # lens_q, lens_k, Hq, Hkv, d, causal, window, softcap
    ((300, 1, 130, 0, 700), (300, 257, 130, 40, 900), 4, 2, 128, True, 0, 0.0),
    ((129, 256, 77), (129, 256, 300), 3, 1, 128, True, 0, 0.0),     # odd group
    ((200, 64), (250, 64), 4, 2, 64, False, 0, 0.0),
    ((190, 260), (190, 400), 2, 1, 256, True, 100, 30.0),           # d = 256
]


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("case", VARLEN, ids=lambda c: "x".join(map(str, c[2:])))
def test_varlen(case, normalizer):
    import torch
    import oracle
    from alternative_normalizers_b200 import nattn_get_device_status, varlen_attention
    lq, lk, Hq, Hkv, d, causal, window, cap = case
    g = torch.Generator().manual_seed(sum(lq) + d + Hq)
    tq, tk = sum(lq), sum(lk)
    q, k, v = _rand(g, tq + 3, Hq, d), _rand(g, tk, Hkv, d), _rand(g, tk, Hkv, d)
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    nnz = torch.full((tq + 3, Hq), -1, dtype=torch.int32, device="cuda")
    out, st = varlen_attention(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(),
                               max(lq), max(lk), normalizer=normalizer, causal=causal,
                               window=window, softcap=cap, row_nnz=nnz)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    o, s = oracle.varlen_attention(q[:tq], k, v, cq, ck, d ** -0.5, normalizer, causal,
                                   window, cap)
    check_out(out[:tq].float().cpu().numpy(), o, str(case))
    check_stat(st[:tq].cpu().numpy(), s, str(case))
    if normalizer in ("softmax", "softmax1"):
        got = nnz[:tq].cpu().numpy()
        for b in range(len(lq)):
            ok = oracle.allowed_matrix(lq[b], lk[b], causal, window).sum(1)
            assert np.array_equal(got[cq[b]:cq[b + 1]], ok[:, None].repeat(Hq, 1))


def test_varlen_with_sinks():
    import torch
    import oracle
    from alternative_normalizers_b200 import varlen_attention
    g = torch.Generator().manual_seed(5)
    lq, lk = (150, 40), (150, 300)
    q, k, v = _rand(g, 190, 4, 128), _rand(g, 450, 2, 128), _rand(g, 450, 2, 128)
    cq = torch.tensor([0, 150, 190], dtype=torch.int32)
    ck = torch.tensor([0, 150, 450], dtype=torch.int32)
    sinks = torch.tensor([0.3, -1.0, 2.0, 0.0])
    out, st = varlen_attention(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), 150, 300,
                               normalizer="softmax", sinks=sinks.cuda())
    o, s = oracle.varlen_attention(q, k, v, cq, ck, 128 ** -0.5, "softmax", True,
                                   sinks=sinks)
    check_out(out.float().cpu().numpy(), o)
    check_stat(st.cpu().numpy(), s)


def _pool(g, B, Hkv, d, page, lens):
    import torch
    npg = [(L + page - 1) // page for L in lens]
    P = sum(npg) + 2
    kp, vp = _rand(g, P, Hkv, page, d), _rand(g, P, Hkv, page, d)
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = torch.full((B, max(npg) + 1), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    return kp, vp, table


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("page,d,Hq,Hkv", [(64, 128, 8, 2), (32, 128, 6, 2),
                                           (64, 64, 4, 2), (64, 256, 4, 2)])
def test_paged_prefill(normalizer, page, d, Hq, Hkv):
    """A chunk of 200 new tokens per sequence against cached lengths 200..700
    (group x 200 rows per key/value head: the tensor-core kernels)."""
    import torch
    import oracle
    from alternative_normalizers_b200 import nattn_get_device_status, paged_attention
    g = torch.Generator().manual_seed(page + d + Hq)
    B, Tq = 3, 200
    lens = [200, 700, 451]
    kp, vp, table = _pool(g, B, Hkv, d, page, lens)
    q = _rand(g, B, Hq, Tq, d)
    sl = torch.tensor(lens, dtype=torch.int32)
    out, st = paged_attention(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), sl.cuda(), 768,
                              normalizer=normalizer)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    ck, cv, ct = compact_pool(kp, vp, table, sl, list(range(B)), page)
    res = oracle.paged_decode(q, ck, cv, ct, sl, page, d ** -0.5, normalizer)
    for b in range(B):
        check_out(out[b].float().cpu().numpy(), res[b][0], f"seq {b}")
        check_stat(st[b].cpu().numpy(), res[b][1], f"seq {b}")


def test_paged_prefill_bad_page_is_caught():
    import torch
    from alternative_normalizers_b200 import nattn_get_device_status, paged_attention
    g = torch.Generator().manual_seed(3)
    kp, vp, table = _pool(g, 2, 2, 128, 64, [300, 200])
    table[0, 2] = 10 ** 6
    q = _rand(g, 2, 8, 130, 128)
    paged_attention(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                    torch.tensor([300, 200], dtype=torch.int32).cuda(), 320,
                    normalizer="softmax")
    assert nattn_get_device_status() == -7
    assert nattn_get_device_status() == 0


def test_varlen_fullsize_qwen3_shape():
    """The Qwen3-8B-shaped layer's heads (Hq=32, Hkv=8, d=128) over a packed
    batch of 8192 tokens in four requests (4096, 2048, 1536, 512 tokens),
    causal; sampled rows of every request against the oracle."""
    import torch
    import oracle
    from alternative_normalizers_b200 import varlen_attention
    lens = [4096, 2048, 1536, 512]
    g = torch.Generator().manual_seed(8)
    tot = sum(lens)
    q, k, v = _rand(g, tot, 32, 128), _rand(g, tot, 8, 128), _rand(g, tot, 8, 128)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    out, st = varlen_attention(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), cu.cuda(),
                               max(lens), max(lens), normalizer="softmax", causal=True)
    out, st = out.float().cpu().numpy(), st.cpu().numpy()
    rng = np.random.default_rng(0)
    for b, L in enumerate(lens):
        lo = int(cu[b])
        rows_i = np.unique(np.concatenate([[0, 127, 128, L - 1], rng.integers(0, L, 60)]))
        heads = rng.integers(0, 32, rows_i.size)
        sel = np.stack([np.zeros_like(rows_i), heads, rows_i], 1)
        qs = q[lo:lo + L].transpose(0, 1)[None]
        ks = k[lo:lo + L].transpose(0, 1)[None]
        vs = v[lo:lo + L].transpose(0, 1)[None]
        o, s, _ = oracle.attention_rows(qs, ks, vs, sel, 128 ** -0.5, "softmax", True)
        check_out(out[lo + rows_i, heads], o, f"request {b}")
        check_stat(st[lo + rows_i, heads], s, f"request {b}")
