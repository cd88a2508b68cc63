"""Failure paths on the GPU that fault, trap or hang nothing.

* The bounded-wait path: a self-test kernel waits, through the same bounded
  mbarrier wait the attention kernels use, on a phase that nothing
  completes.  The wait gives up after its budget and records
  NATTN_ETIMEOUT; the host reads the status and the context stays usable
  (a normal call afterwards matches the oracle).
* Poisoned scratch: the caller-owned workspace is filled with NaN bit
  patterns before each call.  Every value a kernel reads from scratch must
  have been written by an earlier kernel of the same call, so the outputs
  still match the oracle."""

import numpy as np
import pytest

from tests._util import check_out, check_stat, cuda_ok, ensure_built

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _rand(gen, *shape):
    import torch
    return torch.randn(*shape, generator=gen).to(torch.bfloat16)


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    import oracle
    from alternative_normalizers_b200 import binding
    assert binding.nattn_get_device_status() == binding.NATTN_OK
    assert binding.nattn_selftest_wait_timeout(None) == binding.NATTN_OK
    assert binding.nattn_get_device_status() == -6  # NATTN_ETIMEOUT
    assert binding.nattn_get_device_status() == binding.NATTN_OK  # cleared
    g = torch.Generator().manual_seed(3)
    q, k, v = _rand(g, 1, 2, 96, 64), _rand(g, 1, 1, 96, 64), _rand(g, 1, 1, 96, 64)
    out, st, _ = binding.attention(q.cuda(), k.cuda(), v.cuda(), normalizer="softmax",
                                   causal=True)
    torch.cuda.synchronize()
    assert binding.nattn_get_device_status() == binding.NATTN_OK
    o, s, _ = oracle.attention_fwd(q, k, v, 64 ** -0.5, "softmax", True)
    check_out(out.float().cpu().numpy(), o)
    check_stat(st.cpu().numpy(), s)


def _run_poisoned(args_fn, out, stat):
    import torch
    from alternative_normalizers_b200 import binding
    a = args_fn()
    need = binding.nattn_workspace_size(a)
    assert need > 0
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")  # NaN words
    a.workspace, a.workspace_bytes = ws.data_ptr(), need
    rc = binding.nattn_fwd_ex(a)
    torch.cuda.synchronize()
    assert rc == binding.NATTN_OK
    assert binding.nattn_get_device_status() == binding.NATTN_OK
    return out.float().cpu().numpy(), stat.cpu().numpy()


@pytest.mark.parametrize("normalizer", ["sparsemax", "entmax15"])
def test_poisoned_workspace_sparse_prefill(normalizer):
    import torch
    import oracle
    from alternative_normalizers_b200 import binding
    g = torch.Generator().manual_seed(17)
    q, k, v = _rand(g, 1, 4, 300, 128), _rand(g, 1, 2, 300, 128), _rand(g, 1, 2, 300, 128)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty(1, 4, 300, 128, dtype=torch.bfloat16, device="cuda")
    st = torch.empty(1, 4, 300, dtype=torch.float32, device="cuda")
    got, gst = _run_poisoned(
        lambda: binding.build_args(qd, kd, vd, out, st, None, normalizer=normalizer,
                                   causal=True),
        out, st)
    o, s, _ = oracle.attention_fwd(q, k, v, 128 ** -0.5, normalizer, True)
    check_out(got, o)
    check_stat(gst, s)


@pytest.mark.parametrize("normalizer", ["softmax", "sparsemax", "entmax15"])
def test_poisoned_workspace_paged_decode(normalizer):
    import torch
    import oracle
    from alternative_normalizers_b200 import binding
    g = torch.Generator().manual_seed(23)
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
    out = torch.empty(B, Hq, 1, d, dtype=torch.bfloat16, device="cuda")
    st = torch.empty(B, Hq, 1, dtype=torch.float32, device="cuda")
    dev = [x.cuda() for x in (qd, kp, vp, table, lens)]
    got, gst = _run_poisoned(
        lambda: binding.build_args(dev[0], dev[1], dev[2], out, st, None,
                                   normalizer=normalizer, block_table=dev[3],
                                   seqlens=dev[4], page_size=page, max_seqlen=320),
        out, st)
    res = oracle.paged_decode(qd, kp, vp, table, lens, page, d ** -0.5, normalizer)
    for b in range(B):
        check_out(got[b], res[b][0])
        check_stat(gst[b], res[b][1])
