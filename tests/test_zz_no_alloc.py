"""The allocation-free decode entry point, nattn_decode_noalloc.

It exists for callers that must not allocate device memory where they run
attention (memory owned by another allocator, no allocator handed to a
plugin, or a decode step that cannot afford cudaMalloc's implicit
synchronisation).  It keeps its split partials in a fixed array inside the
library instead of a caller workspace.  Here it is called through the C ABI
on two calls in a row and checked against the float64 oracle and against
the workspace-based entry point (nattn_fwd_ex), within the parity
tolerances.  One case has more partials than the array holds at the usual
split count, so the entry point must use fewer, longer splits.  A batch
whose partials cannot fit even with one split per sequence is refused.

This file is collected last so that a failure here does not hide any other
result of a stop-at-first-failure run.
"""

import numpy as np
import pytest

from tests._util import (OUT_MAX_ABS, OUT_MEAN_ABS, STAT_ABS, check_out,
                         check_stat, compact_pool, cuda_ok, ensure_built)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

SCRATCH_BYTES = 8 << 20   # NATTN_NOALLOC_SCRATCH_BYTES


def _paged(seed, B, Hq, Hkv, d, page, lo, hi):
    import torch
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(lo, hi + 1, (B,), generator=g)
    npg = (lens + page - 1) // page
    P = int(npg.sum())
    q = torch.randn(B, Hq, 1, d, generator=g).to(torch.bfloat16)
    kp = torch.randn(P, Hkv, page, d, generator=g).to(torch.bfloat16)
    vp = torch.randn(P, Hkv, page, d, generator=g).to(torch.bfloat16)
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = torch.full((B, int(npg.max())), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += int(npg[b])
    return q, kp, vp, table, lens.to(torch.int32)


def _splits_that_fit(B, Hq, dv):
    """Splits whose partials fit the array (the header's rule)."""
    up = lambda x: (x + 255) // 256 * 256
    rows = B * Hq
    return SCRATCH_BYTES // (up(rows * dv * 4) + up(rows * 8))


# (seed, B, Hq, Hkv, d, lo, hi): the second case needs 4 splits of 32
# pages at its longest sequence but only 3 fit the array
CASES = [(77, 48, 32, 8, 128, 1, 6000), (78, 32, 64, 4, 256, 6200, 8192)]


@pytest.mark.parametrize("normalizer", ["softmax", "softmax1"])
@pytest.mark.parametrize("case", CASES, ids=["fits", "refit"])
def test_noalloc_decode_matches_oracle_and_workspace_entry_point(normalizer, case):
    import torch
    import oracle
    ensure_built()
    from alternative_normalizers_b200 import binding
    seed, B, Hq, Hkv, d, lo, hi = case
    maxlen = (hi + 63) // 64 * 64
    if seed == 78:
        assert _splits_that_fit(B, Hq, d) < (maxlen // 64 + 31) // 32
    q, kp, vp, table, lens = _paged(seed, B, Hq, Hkv, d, 64, lo, hi)
    seqs = sorted({int(np.argmax(lens.numpy())), int(np.argmin(lens.numpy())),
                   3, B - 1})
    ck, cv, ct = compact_pool(kp, vp, table, lens, seqs, 64)
    res = oracle.paged_decode(q, ck, cv, ct, lens, 64, d ** -0.5,
                              normalizer, seqs=seqs)
    q, kp, vp, table, lens = (t.cuda() for t in (q, kp, vp, table, lens))
    # existing entry point, caller-provided workspace
    ref_o, ref_s = binding.paged_attention(q, kp, vp, table, lens, maxlen,
                                           normalizer=normalizer)
    torch.cuda.synchronize()
    ref_o, ref_s = ref_o.float().cpu().numpy(), ref_s.cpu().numpy()
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        st = torch.full((q.shape[0], q.shape[1], 1), float("nan"), device="cuda")
        a = binding.build_args(q, kp, vp, out, st, None, normalizer=normalizer,
                               causal=True, block_table=table, seqlens=lens,
                               page_size=64, max_seqlen=maxlen)
        a.workspace, a.workspace_bytes = None, 0
        rc = binding.nattn_decode_noalloc(a)
        assert rc == 0, binding.nattn_strerror(rc)
        torch.cuda.synchronize()
        assert binding.nattn_get_device_status() == 0
        got_o, got_s = out.float().cpu().numpy(), st.cpu().numpy()
        assert np.isfinite(got_o).all(), f"call {call}"
        for b in seqs:
            check_out(got_o[b], res[b][0], f"call {call} seq {b}")
            check_stat(got_s[b], res[b][1], f"call {call} seq {b}")
        err = np.abs(got_o - ref_o)
        assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, \
            f"call {call}: max {err.max():.3e} mean {err.mean():.3e}"
        assert np.abs(got_s - ref_s).max() <= STAT_ABS, f"call {call}"


def test_noalloc_decode_rejects_oversized_batch():
    ensure_built()
    from alternative_normalizers_b200 import binding
    a = binding.NattnArgs()
    # partials for one split: 8192 seqs * 32 heads * (256 + 2) * 4 bytes =
    # 270 MB, far beyond the fixed array
    a.B, a.Hq, a.Hkv, a.Tq, a.Tk, a.d, a.dv = 8192, 32, 8, 1, 4096, 256, 256
    a.scale, a.normalizer, a.causal = 0.06, 0, 1
    a.q = a.k = a.v = a.out = 4096
    a.block_table = a.seqlens = 4096
    a.page_size, a.block_table_stride, a.num_pages = 64, 64, 1000
    assert binding.nattn_decode_noalloc(a) == -3     # NATTN_ETOOLARGE
    # just past the rule: one split needs one byte block more than the array
    a.B, a.Hq, a.Hkv, a.d, a.dv = 64, 128, 8, 256, 256  # 8192 rows: 8 MiB + 64 KiB
    assert _splits_that_fit(64, 128, 256) == 0
    assert binding.nattn_decode_noalloc(a) == -3
    a.normalizer = 2                                   # sparse: not this path
    assert binding.nattn_decode_noalloc(a) == -2
    a.normalizer = 0
    a.block_table = None                               # dense: not this path
    assert binding.nattn_decode_noalloc(a) == -2
