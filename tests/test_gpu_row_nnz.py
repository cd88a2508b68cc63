"""row_nnz: the per-row count of keys with a nonzero weight, written by every
kernel path, against the float64 oracle's weights.

For sparsemax / 1.5-entmax the count is the support size; a key whose
weight is within rounding of zero may fall on either side, so the counts
must agree on almost every row and differ by at most one elsewhere.  For
softmax / softmax1 it is the number of visible keys, which is exact."""

import numpy as np
import pytest

from tests._util import cuda_ok, ensure_built

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _rand(gen, *shape):
    import torch
    return torch.randn(*shape, generator=gen).to(torch.bfloat16)


def _check(got, want_nnz, normalizer):
    got = np.asarray(got).ravel()
    want = np.asarray(want_nnz).ravel()
    if normalizer in ("softmax", "softmax1"):
        assert np.array_equal(got, want)
    else:
        diff = np.abs(got.astype(np.int64) - want.astype(np.int64))
        assert diff.max() <= 1, diff.max()
        assert (diff == 0).mean() >= 0.99


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("Hkv", [2, 4])  # head-pair kernel, split-row kernel
def test_row_nnz_prefill(normalizer, Hkv):
    import torch
    import oracle
    from alternative_normalizers_b200 import attention
    g = torch.Generator().manual_seed(31 + Hkv)
    q, k, v = _rand(g, 1, 4, 260, 128), _rand(g, 1, Hkv, 260, 128), _rand(g, 1, Hkv, 260, 128)
    nnz = torch.full((1, 4, 260), -1, dtype=torch.int32, device="cuda")
    attention(q.cuda(), k.cuda(), v.cuda(), normalizer=normalizer, causal=True, row_nnz=nnz)
    torch.cuda.synchronize()
    _, _, w = oracle.attention_fwd(q, k, v, 128 ** -0.5, normalizer, True, want_weights=True)
    if normalizer in ("softmax", "softmax1"):
        want = oracle.allowed_matrix(260, 260, True, 0).sum(axis=1)[None, None, :].repeat(4, 1)
    else:
        want = (w > 0).sum(axis=-1)
    _check(nnz.cpu().numpy(), want, normalizer)


@pytest.mark.parametrize("normalizer", NORMS)
def test_row_nnz_rowwise_with_weights(normalizer):
    import torch
    import oracle
    from alternative_normalizers_b200 import attention
    g = torch.Generator().manual_seed(37)
    q, k, v = _rand(g, 1, 2, 40, 32), _rand(g, 1, 1, 40, 32), _rand(g, 1, 1, 40, 32)
    nnz = torch.full((1, 2, 40), -1, dtype=torch.int32, device="cuda")
    _, _, w = attention(q.cuda(), k.cuda(), v.cuda(), normalizer=normalizer, causal=True,
                        want_weights=True, row_nnz=nnz)
    torch.cuda.synchronize()
    got = nnz.cpu().numpy()
    if normalizer in ("softmax", "softmax1"):
        _check(got, oracle.allowed_matrix(40, 40, True, 0).sum(axis=1)[None, None, :].repeat(2, 1),
               normalizer)
    else:
        # the kernel's own weights: the count is exactly their nonzeros
        assert np.array_equal(got, (w.cpu().numpy() > 0).sum(axis=-1))


@pytest.mark.parametrize("normalizer", NORMS)
def test_row_nnz_paged_decode(normalizer):
    import torch
    import oracle
    from alternative_normalizers_b200 import paged_attention
    g = torch.Generator().manual_seed(41)
    B, Hq, Hkv, d, page = 3, 8, 2, 128, 64
    lens = torch.tensor([70, 300, 129], dtype=torch.int32)
    npg = [(int(L) + page - 1) // page for L in lens]
    P = sum(npg)
    kp, vp = _rand(g, P, Hkv, page, d), _rand(g, P, Hkv, page, d)
    qd = _rand(g, B, Hq, 1, d)
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = torch.full((B, max(npg)), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    nnz = torch.full((B, Hq, 1), -1, dtype=torch.int32, device="cuda")
    paged_attention(qd.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lens.cuda(), 320,
                    normalizer=normalizer, row_nnz=nnz)
    torch.cuda.synchronize()
    got = nnz.cpu().numpy()
    want = np.zeros((B, Hq, 1), dtype=np.int64)
    for b in range(B):
        L = int(lens[b])
        if normalizer in ("softmax", "softmax1"):
            want[b] = L
            continue
        k, _ = oracle.paged_gather(kp, vp, table, L, b, page)
        q = qd[b, :, 0].double().numpy()
        for h in range(Hq):
            z = q[h] @ k[h // (Hq // Hkv)].T * d ** -0.5
            p, _ = (oracle.sparsemax_row(z) if normalizer == "sparsemax"
                    else oracle.entmax15_row(z))
            want[b, h, 0] = int((p > 0).sum())
    _check(got, want, normalizer)
