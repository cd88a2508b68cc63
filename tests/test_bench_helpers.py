"""Host logic of bench.py's sparse measurements, checked on the CPU.

``sparse_prefill_stats`` and ``sparse_decode_bytes`` read the row
thresholds the kernel wrote and recount supports and touched V pages from
float32 scores.  Here a stand-in runner supplies the float64 oracle's
thresholds instead of the kernel's, and the counts are compared with the
oracle's own weights (a weight is nonzero exactly on the support)."""

import os
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from alternative_normalizers_b200.workloads import (WORKLOADS, make_dense,  # noqa: E402
                                                    make_paged, shrink)


def _runner(w, x, stat):
    return SimpleNamespace(w=w, x=x, host=x, stat=stat, call=lambda n: None)


@pytest.mark.parametrize("normalizer", ["sparsemax", "entmax15"])
def test_sparse_prefill_stats_match_oracle_supports(normalizer):
    w = shrink(WORKLOADS["sparse_prefill_t1"], B=1, Hq=2, Hkv=1, Tq=48, Tk=48,
               d=32, dv=32)
    x = make_dense(w)
    _, stat, wts = oracle.attention_fwd(x["q"], x["k"], x["v"], w.scale,
                                        normalizer, causal=True,
                                        want_weights=True)
    r = _runner(w, x, torch.from_numpy(stat).float())
    got = bench.sparse_prefill_stats(r, normalizer)
    sup = (wts > 0).sum(axis=-1).ravel()
    visible = w.B * w.Hq * w.Tq * (w.Tq + 1) // 2
    # float32 scores against float64 thresholds: a key exactly at the
    # threshold could flip, which the seeded case does not contain
    assert got["support_max"] == int(sup.max())
    assert abs(got["support_mean"] - sup.mean()) < 0.01
    assert abs(got["exact_zero_fraction"] - (1 - sup.sum() / visible)) < 1e-6
    assert abs(got["tau_mean"] - stat.mean()) < 1e-3


@pytest.mark.parametrize("normalizer", ["sparsemax", "entmax15"])
def test_sparse_decode_bytes_count_touched_v_pages(normalizer):
    w = shrink(WORKLOADS["paged_decode"], B=3, Hq=4, Hkv=2, d=32, dv=32,
               page_size=16, len_range=(20, 90))
    x = make_paged(w)
    res = oracle.paged_decode(x["q"], x["k_pool"], x["v_pool"],
                              x["block_table"], x["seqlens"], w.page_size,
                              w.scale, normalizer)
    stat = torch.stack([torch.from_numpy(res[b][1]) for b in range(w.B)]).float()
    r = _runner(w, x, stat)
    got = bench.sparse_decode_bytes(r, normalizer)

    # brute force: a (sequence, kv head, page) is touched when some query
    # head of the group gives one of the page's keys a nonzero weight
    grp = w.Hq // w.Hkv
    ps = w.page_size
    touched = 0
    kb = sb = 0
    for b in range(w.B):
        L = int(x["seqlens"][b])
        k, v = oracle.paged_gather(x["k_pool"], x["v_pool"], x["block_table"],
                                   L, b, ps)
        q = x["q"][b, :, 0].double().numpy()
        for g in range(w.Hkv):
            z = q[g * grp:(g + 1) * grp] @ k[g].T * w.scale
            u = z / 2 if normalizer == "entmax15" else z
            tau = res[b][1][g * grp:(g + 1) * grp, 0][:, None]
            nz = (u > tau).any(axis=0)
            for p in range(-(-L // ps)):
                touched += bool(nz[p * ps:(p + 1) * ps].any())
        kb += -(-L // ps) * ps * w.Hkv * w.d * 2
        sb += 3 * w.Hq * L * 4
    assert got["v_pages"] == touched
    assert got["v_bytes"] == touched * ps * w.dv * 2
    assert got["k_bytes"] == kb
    assert got["score_bytes"] == sb
    assert got["total"] == kb + got["v_bytes"] + sb + got["qo_bytes"]
    # supports are small, so some V pages are never read
    assert 0 < touched < sum(-(-int(L) // ps) for L in x["seqlens"]) * w.Hkv


@pytest.mark.parametrize("B,Hq,Hkv", [(2, 32, 8), (1, 16, 8), (3, 6, 3), (1, 4, 1)])
def test_e2e_chunks_cover_heads_once_and_are_contiguous(B, Hq, Hkv):
    """The end-to-end loop's chunks cover every (batch entry, KV head) exactly
    once, and each chunk's slices of q [B, Hq, T, d] and k [B, Hkv, T, d] are
    contiguous views (what a single copy per tensor and chunk relies on)."""
    chunks = bench.e2e_chunks(B, Hkv)
    seen = [(b, g) for b, g0, g1 in chunks for g in range(g0, g1)]
    assert sorted(seen) == [(b, g) for b in range(B) for g in range(Hkv)]
    grp = Hq // Hkv
    q = torch.zeros(B, Hq, 5, 4)
    k = torch.zeros(B, Hkv, 7, 4)
    for b, g0, g1 in chunks:
        assert q[b:b + 1, g0 * grp:g1 * grp].is_contiguous()
        assert k[b:b + 1, g0:g1].is_contiguous()
