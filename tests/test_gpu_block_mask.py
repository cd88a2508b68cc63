"""Block masks on the GPU against the float64 oracle.

A block mask keeps or drops whole 128 x 128 blocks of (query, key) pairs on
top of the causal / window rule ("Attention variants", TensorCAD, section "C.
Keep the fused kernel": a mask yields a block mask, and whole blocks that
are masked out are skipped).  Every dense kernel family takes one: the
two-tile and single-tile tcgen05 kernels (d = 64, 128, 256), the threshold
pass and gather of the sparse normalizers with their row-wise overflow
pass, the row-wise kernel (dense weights, other head dims) and the
backward kernels."""

import numpy as np
import pytest

from tests._util import check_out, check_stat, cuda_ok, ensure_built

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _rand(g, *shape):
    import torch
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _mask(g, B, Hq, Tq, Tk, p_keep=0.6):
    import torch
    nq, nk = (Tq + 127) // 128, (Tk + 127) // 128
    return (torch.rand(B, Hq, nq, nk, generator=g) < p_keep).to(torch.uint8)


CASES = [
    # B, Hq, Hkv, Tq, Tk, d, causal, window, softcap
    (1, 4, 2, 520, 520, 128, True, 0, 0.0),     # two-tile kernel
    (1, 3, 1, 400, 400, 128, True, 0, 0.0),     # odd group: split-row kernel
    (2, 2, 1, 300, 460, 64, False, 0, 0.0),
    (1, 2, 1, 384, 384, 256, True, 200, 30.0),  # d = 256, 64-key blocks
    (1, 2, 1, 200, 200, 40, True, 0, 0.0),      # row-wise kernel
]


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_block_mask_prefill(case, normalizer):
    import torch
    import oracle
    from alternative_normalizers_b200 import attention, nattn_get_device_status
    B, Hq, Hkv, Tq, Tk, d, causal, window, cap = case
    g = torch.Generator().manual_seed(300 + Tq + d + Hq)
    q, k, v = _rand(g, B, Hq, Tq, d), _rand(g, B, Hkv, Tk, d), _rand(g, B, Hkv, Tk, d)
    bm = _mask(g, B, Hq, Tq, Tk)
    bm[0, 0, -1, :] = 0        # one query block that keeps nothing
    nnz = torch.full((B, Hq, Tq), -1, dtype=torch.int32, device="cuda")
    out, st, _ = attention(q.cuda(), k.cuda(), v.cuda(), normalizer=normalizer,
                           causal=causal, window=window, softcap=cap,
                           block_mask=bm.cuda(), row_nnz=nnz)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    o, s, w = oracle.attention_fwd(q, k, v, d ** -0.5, normalizer, causal, window,
                                   cap, want_weights=True, block_mask=bm.numpy())
    check_out(out.float().cpu().numpy(), o, str(case))
    check_stat(st.cpu().numpy(), s, str(case))
    got = nnz.cpu().numpy()
    if normalizer in ("softmax", "softmax1"):
        ok = oracle.allowed_matrix(Tq, Tk, causal, window)
        want = np.stack([[(ok & oracle.block_allowed(bm[b, h].numpy(), Tq, Tk)).sum(1)
                          for h in range(Hq)] for b in range(B)])
        assert np.array_equal(got, want)
    else:
        diff = np.abs(got - (w > 0).sum(-1))
        assert diff.max() <= 1 and (diff == 0).mean() >= 0.99


def test_block_mask_dense_weights():
    import torch
    import oracle
    from alternative_normalizers_b200 import attention
    g = torch.Generator().manual_seed(12)
    q, k, v = _rand(g, 1, 2, 200, 32), _rand(g, 1, 1, 200, 32), _rand(g, 1, 1, 200, 32)
    bm = torch.tensor([[[[1, 0], [0, 1]], [[1, 1], [1, 0]]]], dtype=torch.uint8)
    for n in NORMS:
        out, st, w = attention(q.cuda(), k.cuda(), v.cuda(), normalizer=n, causal=True,
                               want_weights=True, block_mask=bm.cuda())
        o, s, ww = oracle.attention_fwd(q, k, v, 32 ** -0.5, n, True, want_weights=True,
                                        block_mask=bm.numpy())
        check_out(out.float().cpu().numpy(), o, n)
        check_stat(st.cpu().numpy(), s, n)
        w = w.cpu().numpy()
        assert np.abs(w - ww).max() < 2e-3
        dropped = ~oracle.block_allowed(bm[0, 0].numpy(), 200, 200)
        assert np.all(w[0, 0][dropped] == 0)


@pytest.mark.parametrize("normalizer", NORMS)
def test_document_mask(normalizer):
    """Three documents of 256, 256 and 128 tokens packed in one sequence with
    a block-diagonal block mask: each document's rows match the oracle run on
    that document alone."""
    import torch
    import oracle
    from alternative_normalizers_b200 import attention
    g = torch.Generator().manual_seed(44)
    T = 640
    q, k, v = _rand(g, 1, 4, T, 128), _rand(g, 1, 2, T, 128), _rand(g, 1, 2, T, 128)
    bm = torch.zeros(1, 4, 5, 5, dtype=torch.uint8)
    for lo, hi in ((0, 2), (2, 4), (4, 5)):
        bm[..., lo:hi, lo:hi] = 1
    out, st, _ = attention(q.cuda(), k.cuda(), v.cuda(), normalizer=normalizer,
                           causal=True, block_mask=bm.cuda())
    out, st = out.float().cpu().numpy(), st.cpu().numpy()
    for lo, hi in ((0, 256), (256, 512), (512, 640)):
        o, s, _ = oracle.attention_fwd(q[:, :, lo:hi], k[:, :, lo:hi], v[:, :, lo:hi],
                                       128 ** -0.5, normalizer, True)
        check_out(out[:, :, lo:hi], o, f"doc {lo}")
        check_stat(st[:, :, lo:hi], s, f"doc {lo}")


@pytest.mark.parametrize("normalizer", ("softmax", "sparsemax"))
def test_block_mask_backward(normalizer):
    import torch
    import oracle
    from alternative_normalizers_b200 import attention, attention_backward
    from tests.test_gpu_backward import check_grad
    g = torch.Generator().manual_seed(61)
    B, Hq, Hkv, T, d = 1, 4, 2, 384, 128
    q, k, v = _rand(g, B, Hq, T, d), _rand(g, B, Hkv, T, d), _rand(g, B, Hkv, T, d)
    do = _rand(g, B, Hq, T, d)
    bm = _mask(g, B, Hq, T, T, 0.7)
    bm[..., :, 0] = 1
    qc, kc, vc, bmc = q.cuda(), k.cuda(), v.cuda(), bm.cuda()
    out, st, _ = attention(qc, kc, vc, normalizer=normalizer, causal=True, block_mask=bmc)
    dq, dk, dv = attention_backward(qc, kc, vc, out, st, do.cuda(), normalizer=normalizer,
                                    causal=True, block_mask=bmc)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd(q, k, v, do, d ** -0.5, normalizer, True,
                                      block_mask=bm.numpy())
    check_grad(dq.float().cpu().numpy(), rq, "dq")
    check_grad(dk.float().cpu().numpy(), rk, "dk")
    check_grad(dv.float().cpu().numpy(), rv, "dv")
