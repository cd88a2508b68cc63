"""ctypes binding of libnattn (include/nattn.h).

Argument marshalling only: every step of the attention forward runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream; nothing here computes attention.  If the shared library is missing
the first call raises, there is no other implementation to fall back on.
"""

import ctypes
import os

from .workloads import NORMALIZER_IDS

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("NATTN_LIB") or os.path.join(_HERE, "lib", "libnattn.so")

NATTN_OK = 0
ERRORS = {
    -1: "NATTN_EINVAL", -2: "NATTN_EUNSUPPORTED", -3: "NATTN_ETOOLARGE",
    -4: "NATTN_EWORKSPACE", -5: "NATTN_ECUDA", -6: "NATTN_ETIMEOUT",
    -7: "NATTN_EBOUNDS", -8: "NATTN_EALIGN",
}


class NattnArgs(ctypes.Structure):
    """Mirror of ``nattn_args``."""

    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("row_stat", ctypes.c_void_p),
        ("weights", ctypes.c_void_p), ("row_nnz", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("Tq", ctypes.c_int), ("Tk", ctypes.c_int), ("d", ctypes.c_int),
        ("dv", ctypes.c_int),
        ("scale", ctypes.c_float), ("normalizer", ctypes.c_int),
        ("causal", ctypes.c_int), ("window", ctypes.c_int),
        ("softcap", ctypes.c_float),
        ("block_table", ctypes.c_void_p), ("seqlens", ctypes.c_void_p),
        ("page_size", ctypes.c_int), ("block_table_stride", ctypes.c_int),
        ("num_pages", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("stream", ctypes.c_void_p), ("sinks", ctypes.c_void_p),
        ("block_mask", ctypes.c_void_p),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("total_q", ctypes.c_int), ("total_k", ctypes.c_int),
    ]


class NattnBwdArgs(ctypes.Structure):
    """Mirror of ``nattn_bwd_args``."""

    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("grad_out", ctypes.c_void_p),
        ("row_stat", ctypes.c_void_p),
        ("grad_q", ctypes.c_void_p), ("grad_k", ctypes.c_void_p),
        ("grad_v", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("Tq", ctypes.c_int), ("Tk", ctypes.c_int), ("d", ctypes.c_int),
        ("dv", ctypes.c_int),
        ("scale", ctypes.c_float), ("normalizer", ctypes.c_int),
        ("causal", ctypes.c_int), ("window", ctypes.c_int),
        ("softcap", ctypes.c_float), ("sinks", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("stream", ctypes.c_void_p), ("block_mask", ctypes.c_void_p),
    ]


class NattnError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {ERRORS.get(code, code)} "
                         f"({nattn_strerror(code)})")


_lib = None


def lib():
    """Load libnattn.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libnattn.so not found at {LIB_PATH}; build it with "
                "`python -m alternative_normalizers_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(NattnArgs)
        L.nattn_fwd_ex.argtypes = [P]
        L.nattn_fwd_ex.restype = ctypes.c_int
        L.nattn_workspace_size.argtypes = [P]
        L.nattn_workspace_size.restype = ctypes.c_size_t
        L.nattn_fwd.argtypes = (
            [ctypes.c_void_p] * 4 + [ctypes.c_void_p]
            + [ctypes.c_int] * 7 + [ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_float]
            + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p])
        L.nattn_fwd.restype = ctypes.c_int
        L.nattn_get_device_status.argtypes = [ctypes.c_void_p]
        L.nattn_get_device_status.restype = ctypes.c_int
        L.nattn_strerror.argtypes = [ctypes.c_int]
        L.nattn_strerror.restype = ctypes.c_char_p
        L.nattn_version.argtypes = []
        L.nattn_version.restype = ctypes.c_int
        L.nattn_decode_noalloc.argtypes = [P]
        L.nattn_decode_noalloc.restype = ctypes.c_int
        PB = ctypes.POINTER(NattnBwdArgs)
        L.nattn_bwd.argtypes = [PB]
        L.nattn_bwd.restype = ctypes.c_int
        L.nattn_bwd_workspace_size.argtypes = [PB]
        L.nattn_bwd_workspace_size.restype = ctypes.c_size_t
        L.nattn_selftest_wait_timeout.argtypes = [ctypes.c_void_p]
        L.nattn_selftest_wait_timeout.restype = ctypes.c_int
        _lib = L
    return _lib


# --------------------------------------------------------------------------
# The C entry points under their own names
# --------------------------------------------------------------------------

def nattn_fwd(q, k, v, out, row_stat, B, Hq, Hkv, Tq, Tk, d, dv, scale,
              normalizer, causal, window, softcap, block_table, seqlens,
              stream):
    """``nattn_fwd`` with raw device pointers (ints) and sizes."""
    return lib().nattn_fwd(q, k, v, out, row_stat, B, Hq, Hkv, Tq, Tk, d, dv,
                           scale, normalizer, causal, window, softcap,
                           block_table, seqlens, stream)


def nattn_fwd_ex(args: NattnArgs):
    return lib().nattn_fwd_ex(ctypes.byref(args))


def nattn_workspace_size(args: NattnArgs):
    return lib().nattn_workspace_size(ctypes.byref(args))


def nattn_bwd(args: NattnBwdArgs):
    return lib().nattn_bwd(ctypes.byref(args))


def nattn_bwd_workspace_size(args: NattnBwdArgs):
    return lib().nattn_bwd_workspace_size(ctypes.byref(args))


def nattn_get_device_status(stream=None):
    return lib().nattn_get_device_status(stream)


def nattn_strerror(code):
    return lib().nattn_strerror(code).decode()


def nattn_version():
    return lib().nattn_version()


def nattn_selftest_wait_timeout(stream=None):
    """Launch the bounded-wait self-test: one wait that nothing completes,
    which gives up after about two seconds and records NATTN_ETIMEOUT."""
    return lib().nattn_selftest_wait_timeout(stream)


def nattn_decode_noalloc(args: NattnArgs):
    """Paged softmax/softmax1 decode with the library's fixed scratch array:
    no workspace, no allocation (``args.workspace`` is ignored)."""
    return lib().nattn_decode_noalloc(ctypes.byref(args))


# --------------------------------------------------------------------------
# torch-tensor front ends (allocation + marshalling)
# --------------------------------------------------------------------------

def _ptr(t):
    return None if t is None else t.data_ptr()


def _norm_id(normalizer):
    if isinstance(normalizer, str):
        return NORMALIZER_IDS[normalizer]
    return int(normalizer)


def build_args(q, k, v, out, row_stat=None, weights=None, *, normalizer,
               causal=False, window=0, softcap=0.0, scale=None,
               block_table=None, seqlens=None, page_size=0, max_seqlen=None,
               stream=None, row_nnz=None, sinks=None, block_mask=None):
    """Fill an ``NattnArgs`` from torch tensors (no device work).
    ``row_nnz`` (int32 [B, Hq, Tq] or None) receives the number of keys with
    a nonzero weight in each row; ``sinks`` (float32 [Hq] or None) are the
    learned per-head sink logits (softmax only); ``block_mask`` (uint8
    [B, Hq, ceil(Tq/128), ceil(Tk/128)] or None) drops whole 128 x 128
    blocks of (query, key) pairs."""
    import torch
    B, Hq, Tq, d = q.shape
    a = NattnArgs()
    a.q, a.k, a.v, a.out = _ptr(q), _ptr(k), _ptr(v), _ptr(out)
    a.row_stat, a.weights = _ptr(row_stat), _ptr(weights)
    a.row_nnz = _ptr(row_nnz)
    a.sinks = _ptr(sinks)
    a.block_mask = _ptr(block_mask)
    a.B, a.Hq, a.Tq, a.d = B, Hq, Tq, d
    a.Hkv = k.shape[1]
    a.dv = v.shape[3]
    a.scale = (1.0 / d ** 0.5) if scale is None else scale
    a.normalizer = _norm_id(normalizer)
    a.causal, a.window, a.softcap = int(bool(causal)), int(window), float(softcap)
    if block_table is not None:
        a.block_table, a.seqlens = _ptr(block_table), _ptr(seqlens)
        a.page_size = page_size or k.shape[2]
        a.block_table_stride = block_table.shape[1]
        a.num_pages = k.shape[0]
        a.Tk = int(max_seqlen)
    else:
        a.Tk = k.shape[2]
    if stream is None and q.is_cuda:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    a.stream = stream
    return a


def _run(a, workspace_holder):
    import torch
    need = nattn_workspace_size(a)
    ws = None
    if need:
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        a.workspace, a.workspace_bytes = ws.data_ptr(), need
    workspace_holder.append(ws)
    rc = nattn_fwd_ex(a)
    if rc != NATTN_OK:
        raise NattnError(rc, "nattn_fwd_ex")


def attention(q, k, v, normalizer="softmax", causal=False, window=0,
              softcap=0.0, scale=None, want_weights=False, out=None,
              row_stat=None, row_nnz=None, sinks=None, block_mask=None):
    """Dense attention forward.  q [B,Hq,Tq,d], k [B,Hkv,Tk,d], v
    [B,Hkv,Tk,dv] (bf16, CUDA, contiguous).  Returns (out, row_stat,
    weights|None); fills ``row_nnz`` (int32 [B,Hq,Tq]) when given.
    ``sinks`` (float32 [Hq], softmax only): learned per-head sink logits.
    ``block_mask`` (uint8 [B, Hq, ceil(Tq/128), ceil(Tk/128)]): 0 drops the
    128 x 128 block of (query, key) pairs."""
    import torch
    B, Hq, Tq, _ = q.shape
    Tk, dv = k.shape[2], v.shape[3]
    out = torch.empty(B, Hq, Tq, dv, dtype=torch.bfloat16, device=q.device) \
        if out is None else out
    row_stat = torch.empty(B, Hq, Tq, dtype=torch.float32, device=q.device) \
        if row_stat is None else row_stat
    weights = torch.empty(B, Hq, Tq, Tk, dtype=torch.float32,
                          device=q.device) if want_weights else None
    a = build_args(q, k, v, out, row_stat, weights, normalizer=normalizer,
                   causal=causal, window=window, softcap=softcap, scale=scale,
                   row_nnz=row_nnz, sinks=sinks, block_mask=block_mask)
    keep = []
    _run(a, keep)
    return out, row_stat, weights


def varlen_attention(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                     max_seqlen_k, normalizer="softmax", causal=True, window=0,
                     softcap=0.0, scale=None, sinks=None, out=None,
                     row_stat=None, row_nnz=None):
    """Packed variable-length attention: q [total_q, Hq, d], k [total_k,
    Hkv, d], v [total_k, Hkv, dv] (bf16, CUDA, contiguous), cumulative
    lengths int32 [B + 1] on the device.  Returns (out [total_q, Hq, dv],
    row_stat [total_q, Hq]); fills ``row_nnz`` ([total_q, Hq]) when given."""
    import torch
    total_q, Hq, d = q.shape
    total_k, Hkv, _ = k.shape
    dv = v.shape[2]
    out = torch.empty(total_q, Hq, dv, dtype=torch.bfloat16, device=q.device) \
        if out is None else out
    row_stat = torch.empty(total_q, Hq, dtype=torch.float32, device=q.device) \
        if row_stat is None else row_stat
    a = NattnArgs()
    a.q, a.k, a.v, a.out = _ptr(q), _ptr(k), _ptr(v), _ptr(out)
    a.row_stat, a.row_nnz, a.sinks = _ptr(row_stat), _ptr(row_nnz), _ptr(sinks)
    a.B = cu_seqlens_q.numel() - 1
    a.Hq, a.Hkv, a.d, a.dv = Hq, Hkv, d, dv
    a.Tq, a.Tk = int(max_seqlen_q), int(max_seqlen_k)
    a.scale = (1.0 / d ** 0.5) if scale is None else scale
    a.normalizer = _norm_id(normalizer)
    a.causal, a.window, a.softcap = int(bool(causal)), int(window), float(softcap)
    a.cu_seqlens_q, a.cu_seqlens_k = _ptr(cu_seqlens_q), _ptr(cu_seqlens_k)
    a.total_q, a.total_k = total_q, total_k
    a.stream = torch.cuda.current_stream(q.device).cuda_stream
    keep = []
    _run(a, keep)
    return out, row_stat


def paged_attention(q, k_pool, v_pool, block_table, seqlens, max_seqlen,
                    normalizer="softmax", causal=True, window=0, softcap=0.0,
                    scale=None, out=None, row_stat=None, row_nnz=None,
                    sinks=None):
    """Attention of q [B,Hq,Tq,d] over a paged cache: k_pool/v_pool
    [num_pages, Hkv, page, d], block_table int32 [B, max_pages], seqlens
    int32 [B] (each <= max_seqlen).  Fills ``row_nnz`` when given."""
    import torch
    B, Hq, Tq, _ = q.shape
    dv = v_pool.shape[3]
    out = torch.empty(B, Hq, Tq, dv, dtype=torch.bfloat16, device=q.device) \
        if out is None else out
    row_stat = torch.empty(B, Hq, Tq, dtype=torch.float32, device=q.device) \
        if row_stat is None else row_stat
    a = build_args(q, k_pool, v_pool, out, row_stat, None,
                   normalizer=normalizer, causal=causal, window=window,
                   softcap=softcap, scale=scale, block_table=block_table,
                   seqlens=seqlens, page_size=k_pool.shape[2],
                   max_seqlen=max_seqlen, row_nnz=row_nnz, sinks=sinks)
    keep = []
    _run(a, keep)
    return out, row_stat


def build_bwd_args(q, k, v, out, row_stat, grad_out, grad_q, grad_k, grad_v, *,
                   normalizer, causal=False, window=0, softcap=0.0,
                   scale=None, sinks=None, stream=None, block_mask=None):
    """Fill an ``NattnBwdArgs`` from torch tensors (no device work)."""
    import torch
    B, Hq, Tq, d = q.shape
    a = NattnBwdArgs()
    a.q, a.k, a.v, a.out = _ptr(q), _ptr(k), _ptr(v), _ptr(out)
    a.grad_out, a.row_stat = _ptr(grad_out), _ptr(row_stat)
    a.grad_q, a.grad_k, a.grad_v = _ptr(grad_q), _ptr(grad_k), _ptr(grad_v)
    a.B, a.Hq, a.Tq, a.d = B, Hq, Tq, d
    a.Hkv, a.Tk, a.dv = k.shape[1], k.shape[2], v.shape[3]
    a.scale = (1.0 / d ** 0.5) if scale is None else scale
    a.normalizer = _norm_id(normalizer)
    a.causal, a.window, a.softcap = int(bool(causal)), int(window), float(softcap)
    a.sinks = _ptr(sinks)
    a.block_mask = _ptr(block_mask)
    if stream is None and q.is_cuda:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    a.stream = stream
    return a


def attention_backward(q, k, v, out, row_stat, grad_out, normalizer="softmax",
                       causal=False, window=0, softcap=0.0, scale=None,
                       sinks=None, block_mask=None):
    """Gradients (dq, dk, dv) of sum(grad_out * O) for the dense forward
    that produced ``out`` and ``row_stat`` with the same arguments (bf16,
    CUDA, contiguous; d == dv in {64, 128})."""
    import torch
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    a = build_bwd_args(q, k, v, out, row_stat, grad_out, dq, dk, dv,
                       normalizer=normalizer, causal=causal, window=window,
                       softcap=softcap, scale=scale, sinks=sinks,
                       block_mask=block_mask)
    need = nattn_bwd_workspace_size(a)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    a.workspace, a.workspace_bytes = ws.data_ptr(), need
    rc = nattn_bwd(a)
    if rc != NATTN_OK:
        raise NattnError(rc, "nattn_bwd")
    return dq, dk, dv
