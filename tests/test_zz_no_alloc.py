"""The allocation-free decode entry point, nattn_decode_noalloc.

It exists for callers that must not allocate device memory where they run
attention (memory owned by another allocator, no allocator handed to a
plugin, or a decode step that cannot afford cudaMalloc's implicit
synchronisation).  It keeps its split partials in a fixed array inside the
library instead of a caller workspace.  Here it is called through the C ABI
and must give the same result as the workspace-based entry point
(nattn_fwd_ex) within the parity tolerances, on two calls in a row, and it
must refuse a batch whose partials cannot fit its array.

This file is collected last so that a failure here does not hide any other
result of a stop-at-first-failure run.
"""

import numpy as np
import pytest

from tests._util import OUT_MAX_ABS, OUT_MEAN_ABS, STAT_ABS, cuda_ok, ensure_built

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]


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


@pytest.mark.parametrize("normalizer", ["softmax", "softmax1"])
def test_noalloc_decode_matches_workspace_entry_point(normalizer):
    import torch
    ensure_built()
    from alternative_normalizers_b200 import binding
    q, kp, vp, table, lens = _paged(77, 48, 32, 8, 128, 64, 1, 6000)
    q, kp, vp, table, lens = (t.cuda() for t in (q, kp, vp, table, lens))
    maxlen = 6016
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
        err = np.abs(got_o - ref_o)
        assert np.isfinite(got_o).all(), f"call {call}"
        assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, \
            f"call {call}: max {err.max():.3e} mean {err.mean():.3e}"
        assert np.abs(got_s - ref_s).max() <= STAT_ABS, f"call {call}"


def test_noalloc_decode_rejects_oversized_batch():
    ensure_built()
    from alternative_normalizers_b200 import binding
    a = binding.NattnArgs()
    # partials for one split: 8192 seqs * 8 kv heads * 4 rows * (256 + 2) * 4
    # bytes = 270 MB, far beyond the fixed array
    a.B, a.Hq, a.Hkv, a.Tq, a.Tk, a.d, a.dv = 8192, 32, 8, 1, 4096, 256, 256
    a.scale, a.normalizer, a.causal = 0.06, 0, 1
    a.q = a.k = a.v = a.out = 4096
    a.block_table = a.seqlens = 4096
    a.page_size, a.block_table_stride, a.num_pages = 64, 64, 1000
    assert binding.nattn_decode_noalloc(a) == -3     # NATTN_ETOOLARGE
    a.normalizer = 2                                   # sparse: not this path
    assert binding.nattn_decode_noalloc(a) == -2
    a.normalizer = 0
    a.block_table = None                               # dense: not this path
    assert binding.nattn_decode_noalloc(a) == -2
