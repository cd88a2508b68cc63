"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times.  The oracle recomputes at least 1024 seeded query rows per
workload one by one (tile-edge rows, every head of one KV group, rows at the
window edge, uniform picks; the same rows on every run); the kernels run on
the whole problem.  For the sparse normalizers the GPU's support of every
sampled row (its count of nonzero weights) is checked against the oracle's
set of keys with p > 0, and the exact-zero fraction is reported."""

import numpy as np
import pytest

from tests._util import (check_out, check_stat, compact_pool, cuda_ok,
                         ensure_built, fullsize_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


_cache = {}


def _inputs(name):
    from alternative_normalizers_b200.workloads import WORKLOADS, make_inputs
    if name not in _cache:
        _cache.clear()
        w = WORKLOADS[name]
        _cache[name] = (w, make_inputs(w))
    return _cache[name]


def _run(w, x, normalizer, want_nnz=False):
    import torch
    from alternative_normalizers_b200 import (attention, nattn_get_device_status,
                                              paged_attention)
    nnz = None
    if want_nnz:
        nnz = torch.full((w.B, w.Hq, w.Tq), -1, dtype=torch.int32, device="cuda")
    if w.paged:
        out, st = paged_attention(
            x["q"].cuda(), x["k_pool"].cuda(), x["v_pool"].cuda(),
            x["block_table"].cuda(), x["seqlens"].cuda(), w.len_range[1],
            normalizer=normalizer, causal=w.causal, row_nnz=nnz)
    else:
        out, st, _ = attention(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(),
                               normalizer=normalizer, causal=w.causal,
                               window=w.window, softcap=w.softcap,
                               scale=w.scale, row_nnz=nnz)
    torch.cuda.synchronize()
    assert nattn_get_device_status() == 0
    return (out.float().cpu().numpy(), st.cpu().numpy(),
            None if nnz is None else nnz.cpu().numpy())


def support_check(w, x, rows, normalizer, tau_o, nnz_gpu):
    """Compare the GPU's support size of each sampled row with the oracle's
    set {j : p_j > 0}.  Membership is decided by u_j > tau (u = z for
    sparsemax, z / 2 for 1.5-entmax); a key within a rounding band of tau
    may fall on either side, so the GPU count must lie between the oracle's
    counts at tau + band and tau - band, and equal the oracle's count on
    every row with no key in the band.  Returns the exact-zero fractions
    (GPU, oracle) over the visible keys of the sampled rows."""
    import oracle
    q = oracle.attention._f64(x["q"])
    k = oracle.attention._f64(x["k"])
    group = w.Hq // w.Hkv
    ok_all = oracle.allowed_matrix(w.Tq, w.Tk, w.causal, w.window)
    half = 0.5 if normalizer == "entmax15" else 1.0
    vis = sup_o = sup_g = 0
    banded = 0
    for r, (b, h, i) in enumerate(rows):
        ok = ok_all[i]
        z = oracle.transform_scores(q[b, h, i] @ k[b, h // group].T, w.scale,
                                    w.softcap)[ok]
        u = z * half
        t = tau_o[r]
        band = 1e-4 * max(1.0, abs(t))
        exact = int((u > t).sum())
        lo, hi = int((u > t + band).sum()), int((u > t - band).sum())
        g = int(nnz_gpu[r])
        assert lo <= g <= hi, f"row {(b, h, i)}: gpu {g} oracle [{lo}, {hi}]"
        if lo == hi:
            assert g == exact, f"row {(b, h, i)}: gpu {g} oracle {exact}"
        else:
            banded += 1
        vis += ok.sum()
        sup_o += exact
        sup_g += g
    # keys within the band of tau are rare: at most a few percent of rows
    assert banded <= max(2, len(rows) // 20)
    return 1.0 - sup_g / vis, 1.0 - sup_o / vis


DENSE = [("qwen3_8b_prefill", "softmax"), ("qwen3_8b_prefill", "softmax1"),
         ("sparse_prefill_t1", "sparsemax"), ("sparse_prefill_t1", "entmax15"),
         ("sparse_prefill_t4", "sparsemax"), ("sparse_prefill_t4", "entmax15"),
         ("gemma2_9b_local", "softmax"), ("gemma2_9b_local", "softmax1"),
         ("gemma2_9b_global", "softmax"), ("gemma2_9b_global", "softmax1")]


@pytest.mark.parametrize("name,normalizer", DENSE)
def test_fullsize_dense(name, normalizer):
    import oracle
    w, x = _inputs(name)
    sparse = normalizer in ("sparsemax", "entmax15")
    out, st, nnz = _run(w, x, normalizer, want_nnz=sparse)
    rows = fullsize_rows(w, 1024)
    assert len(rows) >= 1024
    o, s, _ = oracle.attention_rows(x["q"], x["k"], x["v"], rows, w.scale,
                                    normalizer, w.causal, w.window, w.softcap)
    got_o = out[rows[:, 0], rows[:, 1], rows[:, 2]]
    got_s = st[rows[:, 0], rows[:, 1], rows[:, 2]]
    check_out(got_o, o, f"{name}/{normalizer}")
    check_stat(got_s, s, f"{name}/{normalizer}")
    assert np.isfinite(out).all()
    if sparse:
        zg, zo = support_check(w, x, rows, normalizer, s,
                               nnz[rows[:, 0], rows[:, 1], rows[:, 2]])
        print(f"{name}/{normalizer}: exact-zero fraction gpu {zg:.6f} "
              f"oracle {zo:.6f} over {len(rows)} rows")
        assert zg > 0.98 and abs(zg - zo) <= 1e-4


def test_fullsize_softmax1_zero_logit_identity():
    """Qwen3-8B-shaped layer: softmax1 equals softmax with one zero key and
    zero value prepended (bottom-right causal), both on the GPU at full
    size."""
    import torch
    w, x = _inputs("qwen3_8b_prefill")
    from alternative_normalizers_b200 import attention
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    o1, s1, _ = attention(q, k, v, normalizer="softmax1", causal=True)
    z = torch.zeros(w.B, w.Hkv, 1, w.d, dtype=torch.bfloat16, device="cuda")
    o0, s0, _ = attention(q, torch.cat([z, k], 2), torch.cat([z, v], 2),
                          normalizer="softmax", causal=True, scale=w.scale)
    torch.cuda.synchronize()
    d = (o1.float() - o0.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3
    assert (s1 - s0).abs().max().item() <= 1e-3


@pytest.mark.parametrize("normalizer", ["softmax", "softmax1", "sparsemax",
                                        "entmax15"])
def test_fullsize_paged_decode(normalizer):
    import oracle
    from tests._util import workload_seed
    w, x = _inputs("paged_decode")
    out, st, nnz = _run(w, x, normalizer, want_nnz=True)
    rng = np.random.default_rng(workload_seed(w.name))
    lens = x["seqlens"].numpy()
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens))} |
                  set(rng.choice(w.B, 6, replace=False).tolist()))
    ck, cv, ct = compact_pool(x["k_pool"], x["v_pool"], x["block_table"],
                              lens, seqs, w.page_size)
    res = oracle.paged_decode(x["q"], ck, cv, ct, lens, w.page_size, w.scale,
                              normalizer, seqs=seqs)
    for b in seqs:
        check_out(out[b], res[b][0], f"seq {b}")
        check_stat(st[b], res[b][1], f"seq {b}")
        if normalizer in ("softmax", "softmax1"):
            assert (nnz[b] == lens[b]).all()
    assert np.isfinite(out).all()
