"""GPU parity on small and ragged problems, every path against the float64
oracle: the row-wise kernel (dense weights), the tcgen05 prefill kernels
(online softmax/softmax1, two-phase sparsemax/entmax15) and the paged
split-KV decode kernels.  Sizes span several 128-row tiles and a ragged
tail so the oracle still finishes in seconds."""

import numpy as np
import pytest

from tests._util import (check_out, check_stat, cuda_ok, ensure_built,
                         sample_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

NORMS = ("softmax", "softmax1", "sparsemax", "entmax15")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _rand(gen, *shape, gain=1.0):
    import torch
    return (torch.randn(*shape, generator=gen) * gain).to(torch.bfloat16)


def _inputs(seed, B, Hq, Hkv, Tq, Tk, d, dv=None, gain=1.0):
    import torch
    g = torch.Generator().manual_seed(seed)
    dv = d if dv is None else dv
    return (_rand(g, B, Hq, Tq, d, gain=gain), _rand(g, B, Hkv, Tk, d, gain=gain),
            _rand(g, B, Hkv, Tk, dv, gain=gain))


def _gpu(q, k, v, **kw):
    import torch
    from alternative_normalizers_b200 import attention, nattn_get_device_status
    out, st, w = attention(q.cuda(), k.cuda(), v.cuda(), **kw)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    return (out.float().cpu().numpy(), st.cpu().numpy(),
            None if w is None else w.cpu().numpy())


# ----------------------------------------------------------------- row-wise

@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_with_weights(normalizer, causal):
    """B=1, Hq=2, Hkv=1, T=64, d=32: the tiny correctness case, dense weights
    returned; masked weights must be exactly zero."""
    from alternative_normalizers_b200.workloads import WORKLOADS, make_dense
    import oracle
    w = WORKLOADS["tiny_causal" if causal else "tiny"]
    x = make_dense(w)
    out, st, wt = _gpu(x["q"], x["k"], x["v"], normalizer=normalizer,
                       causal=causal, want_weights=True)
    o, s, ww = oracle.attention_fwd(x["q"], x["k"], x["v"], w.scale,
                                    normalizer, causal, want_weights=True)
    check_out(out, o, normalizer)
    check_stat(st, s, normalizer)
    assert np.abs(wt - ww).max() < 2e-3
    ok = oracle.allowed_matrix(w.Tq, w.Tk, causal, 0)
    assert np.all(wt[..., ~ok] == 0.0)
    if normalizer in ("sparsemax", "entmax15"):
        # exact zeros of the sparse normalizers are reproduced
        agree = (wt == 0) == (ww == 0)
        assert agree.mean() > 0.995


@pytest.mark.parametrize("normalizer", NORMS)
def test_rowwise_odd_head_dim(normalizer):
    """d=40, dv=24 are outside the tensor-core shapes: row-wise kernel."""
    import oracle
    q, k, v = _inputs(7, 1, 4, 2, 37, 53, 40, 24)
    out, st, _ = _gpu(q, k, v, normalizer=normalizer, causal=True, window=9)
    o, s, _ = oracle.attention_fwd(q, k, v, 40 ** -0.5, normalizer, True, 9)
    check_out(out, o)
    check_stat(st, s)


# ----------------------------------------------------------------- tcgen05

TC_CASES = [
    # B, Hq, Hkv, Tq, Tk, d, causal, window, softcap
    (1, 4, 2, 320, 320, 128, True, 0, 0.0),
    (1, 4, 2, 320, 320, 128, False, 0, 0.0),
    (2, 2, 1, 256, 256, 64, True, 0, 0.0),
    (1, 2, 1, 200, 333, 128, True, 0, 0.0),      # Tq != Tk, bottom-right
    (1, 2, 2, 300, 100, 128, True, 0, 0.0),      # Tq > Tk: masked rows
    (1, 2, 1, 384, 384, 256, True, 0, 50.0),     # Gemma-like soft-cap
    # cap 4: most 64-score chunks lie within the cap (polynomial tanh), a
    # few hold a score past it (hardware tanh) in the same launch
    (1, 2, 1, 384, 384, 256, True, 0, 4.0),
    (1, 4, 2, 320, 320, 128, True, 0, 4.0),
    (1, 4, 2, 320, 320, 128, True, 0, 50.0),     # soft-cap on the pair kernel
    (1, 2, 1, 600, 600, 128, True, 256, 0.0),    # sliding window
    (1, 2, 1, 300, 300, 128, True, 1000, 1.0),   # window >= T, heavy cap
    (1, 2, 1, 130, 130, 128, False, 50, 0.0),    # two-sided window
    (2, 4, 2, 1, 500, 128, True, 0, 0.0),        # one query row over 500 keys
    (1, 4, 4, 17, 1, 64, False, 0, 0.0),         # a single key
]


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "x".join(map(str, c)))
def test_tc_prefill(case, normalizer):
    import oracle
    B, Hq, Hkv, Tq, Tk, d, causal, window, cap = case
    q, k, v = _inputs(11 + Tq + d, B, Hq, Hkv, Tq, Tk, d)
    out, st, _ = _gpu(q, k, v, normalizer=normalizer, causal=causal,
                      window=window, softcap=cap)
    o, s, _ = oracle.attention_fwd(q, k, v, d ** -0.5, normalizer, causal,
                                   window, cap)
    check_out(out, o, str(case))
    check_stat(st, s, str(case))


@pytest.mark.parametrize("normalizer", ("sparsemax", "entmax15"))
def test_tc_sparse_temperature(normalizer):
    """Q x 4 gives narrow supports (often a single key): tau and the zeros
    must still be exact."""
    import oracle
    q, k, v = _inputs(5, 1, 2, 1, 512, 512, 128)
    q = (q.float() * 4).to(q.dtype)
    out, st, _ = _gpu(q, k, v, normalizer=normalizer, causal=True)
    o, s, _ = oracle.attention_fwd(q, k, v, 128 ** -0.5, normalizer, True)
    check_out(out, o)
    check_stat(st, s)


@pytest.mark.parametrize("normalizer", ("sparsemax", "entmax15"))
def test_tc_sparse_overflow_rows(normalizer):
    """Identical keys make every score equal: each row's support is its whole
    visible range, which overflows the phase-1 candidate buffer and sends the
    rows to the row-wise kernel."""
    import torch
    import oracle
    q, k, v = _inputs(9, 1, 2, 1, 384, 384, 128)
    k = k[:, :, :1].expand(-1, -1, 384, -1).contiguous()
    out, st, _ = _gpu(q, k, v, normalizer=normalizer, causal=True)
    o, s, _ = oracle.attention_fwd(q, k, v, 128 ** -0.5, normalizer, True)
    check_out(out, o)
    check_stat(st, s)


@pytest.mark.parametrize("normalizer,qscale", [("sparsemax", 1 / 128), ("entmax15", 1 / 8)])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_tc_sparse_wide_supports(normalizer, qscale, d):
    """Flat score rows (queries scaled down): supports of up to a few
    hundred keys, wider than the threshold pass's candidate buffers on most
    rows past the first tile.  Those rows take the wide kernel (Newton
    passes over their full score rows, weights multiplied on the tensor
    cores); the first rows of the causal band stay within the buffers, so
    tiles hold both kinds.  Output, threshold and support size (row_nnz)
    against the oracle, on a ragged 1000-row causal problem."""
    import torch
    import oracle
    from alternative_normalizers_b200 import attention, nattn_get_device_status
    T = 1000
    q, k, v = _inputs(41 + d, 1, 4, 2, T, T, d)
    q = (q.float() * qscale).to(q.dtype)
    nnz = torch.full((1, 4, T), -1, dtype=torch.int32, device="cuda")
    out, st, _ = attention(q.cuda(), k.cuda(), v.cuda(), normalizer=normalizer,
                           causal=True, row_nnz=nnz)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    o, s, w = oracle.attention_fwd(q, k, v, d ** -0.5, normalizer, True,
                                   want_weights=True)
    want_nnz = (w > 0).sum(axis=-1)
    # the case exercises what it is meant to: supports beyond the buffers
    assert want_nnz.max() > 200
    check_out(out.float().cpu().numpy(), o)
    check_stat(st.cpu().numpy(), s)
    diff = np.abs(nnz.cpu().numpy().astype(np.int64) - want_nnz)
    assert diff.max() <= 1 and (diff == 0).mean() >= 0.99


@pytest.mark.parametrize("normalizer", ("softmax", "softmax1"))
@pytest.mark.parametrize("d,Hq", [(256, 2), (128, 3)])
def test_online_rescale_every_block(normalizer, d, Hq):
    """Scores that rise by about 9 (log2 units) from one 64-key block to the
    next: the running maximum moves past the lazy-rescale margin of 8 on
    every block, so the single-tile kernel (d = 256, and odd GQA groups)
    rescales O on every block while the previous block's PV may still be in
    flight.  Each block's keys tie, so the weights of earlier blocks stay
    visible in O (about 2^-9 per block back)."""
    import torch
    import oracle
    T = 1024
    g = torch.Generator().manual_seed(77 + d)
    q = torch.zeros(1, Hq, T, d)
    q[..., 0] = 4.0
    k = torch.randn(1, 1, T, d, generator=g) * 0.01
    # x = q.k * scale * log2(e) rises by ~9 per 64 keys
    step = 9.0 / (4.0 * d ** -0.5 * 1.4426950408889634)
    k[0, 0, :, 0] = step * (torch.arange(T) // 64).float()
    v = torch.randn(1, 1, T, d, generator=g)
    q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    out, st, _ = _gpu(q, k, v, normalizer=normalizer, causal=True)
    o, s, _ = oracle.attention_fwd(q, k, v, d ** -0.5, normalizer, True)
    check_out(out, o)
    check_stat(st, s)


def test_softmax1_is_softmax_with_zero_key_on_gpu():
    """GPU softmax1 equals GPU softmax on the input with a zero key and zero
    value prepended (bottom-right causal), which also exercises Tk' = T + 1."""
    import torch
    q, k, v = _inputs(13, 1, 4, 2, 257, 257, 128)
    o1, s1, _ = _gpu(q, k, v, normalizer="softmax1", causal=True)
    z = torch.zeros(1, 2, 1, 128, dtype=torch.bfloat16)
    o0, s0, _ = _gpu(q, torch.cat([z, k], 2), torch.cat([z, v], 2),
                     normalizer="softmax", causal=True)
    assert np.abs(o1 - o0).max() <= 2e-2
    assert np.abs(s1 - s0).max() <= 1e-3


# ----------------------------------------------------------------- decode

def _paged_case(seed, B, Hq, Hkv, d, page, lo, hi, Tq=1):
    import torch
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(lo, hi + 1, (B,), generator=g)
    npg = (lens + page - 1) // page
    P = int(npg.sum())
    q = _rand(g, B, Hq, Tq, d)
    kp = _rand(g, P, Hkv, page, d)
    vp = _rand(g, P, Hkv, page, d)
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = torch.full((B, int(npg.max())), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += int(npg[b])
    return q, kp, vp, table, lens.to(torch.int32)


@pytest.mark.parametrize("normalizer", NORMS)
@pytest.mark.parametrize("page,d,Tq", [(64, 128, 1), (32, 128, 1), (64, 64, 2),
                                       (64, 256, 1)])
def test_paged_decode(normalizer, page, d, Tq):
    import torch
    import oracle
    from alternative_normalizers_b200 import paged_attention
    from alternative_normalizers_b200 import nattn_get_device_status
    B, Hq, Hkv = 5, 8, 2
    q, kp, vp, table, lens = _paged_case(21 + page + d, B, Hq, Hkv, d, page, 1,
                                         700, Tq)
    maxlen = 704
    out, st = paged_attention(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                              lens.cuda(), maxlen, normalizer=normalizer)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    res = oracle.paged_decode(q, kp, vp, table, lens, page, d ** -0.5,
                              normalizer)
    for b in range(B):
        check_out(out[b].float().cpu().numpy(), res[b][0], f"seq {b}")
        check_stat(st[b].cpu().numpy(), res[b][1], f"seq {b}")


@pytest.mark.parametrize("normalizer", ["sparsemax", "entmax15"])
@pytest.mark.parametrize("page,gain", [(64, 0.02), (64, 0.3), (32, 0.1)])
def test_paged_decode_long_and_flat(normalizer, page, gain):
    """Sequences of several splits and queries scaled down so that scores
    crowd near their maximum: thousands of threshold candidates per row (more
    than the threshold kernel keeps in shared memory at the smallest gain)
    and supports longer than the apply pass's per-split list."""
    import torch
    import oracle
    from alternative_normalizers_b200 import paged_attention
    from alternative_normalizers_b200 import nattn_get_device_status
    B, Hq, Hkv, d = 3, 8, 2, 128
    q, kp, vp, table, lens = _paged_case(77 + page, B, Hq, Hkv, d, page, 2100,
                                         5000)
    q = (q.float() * gain).to(torch.bfloat16)
    out, st = paged_attention(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                              lens.cuda(), 5000, normalizer=normalizer)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    res = oracle.paged_decode(q, kp, vp, table, lens, page, d ** -0.5,
                              normalizer)
    for b in range(B):
        check_out(out[b].float().cpu().numpy(), res[b][0], f"seq {b}")
        check_stat(st[b].cpu().numpy(), res[b][1], f"seq {b}")


def test_paged_decode_bad_block_table_reports_bounds():
    """An out-of-range page id is caught on the device: the status word says
    NATTN_EBOUNDS and nothing faults."""
    import torch
    from alternative_normalizers_b200 import paged_attention
    from alternative_normalizers_b200 import nattn_get_device_status
    q, kp, vp, table, lens = _paged_case(3, 2, 8, 2, 128, 64, 100, 300)
    table[1, 0] = 10 ** 6
    paged_attention(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lens.cuda(),
                    320, normalizer="softmax")
    assert nattn_get_device_status() == -7
    assert nattn_get_device_status() == 0


def test_dense_weights_sum_and_zeros():
    """Weights from the weights path: rows sum to one (softmax1 below one)."""
    q, k, v = _inputs(17, 1, 2, 1, 50, 70, 64)
    for n in NORMS:
        _, _, w = _gpu(q, k, v, normalizer=n, causal=True, want_weights=True)
        s = w.sum(-1)
        if n == "softmax1":
            assert (s < 1).all()
        else:
            assert np.abs(s - 1).max() < 1e-4
