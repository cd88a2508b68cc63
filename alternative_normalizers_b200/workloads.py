"""Seeded synthetic workloads shared by the tests, the bench and the smoke run.

This module only draws random inputs and lays them out; it holds none of the
attention arithmetic (no scores, masks or normalizers), so it may serve both
the CUDA path and the float64 oracle.  Every tensor is drawn in float32 from
a CPU ``torch.Generator`` and rounded to bfloat16 (round-to-nearest-even);
both sides then read the same bf16 values.

The shapes follow the model families the source pages name (Qwen3 in "HF
Attention Normalizers", section "Qwen3 Surgery Path"; Gemma 2's soft-cap and
local/global layers in "Attention variants", TensorCAD, sections "What the
engine does today" and "Two places it is already wrong"); no weights or
datasets are involved.
"""

from dataclasses import dataclass, field, replace

import torch

NORMALIZER_IDS = {"softmax": 0, "softmax1": 1, "sparsemax": 2, "entmax15": 3}


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, mask switches and input recipe."""

    name: str
    B: int
    Hq: int
    Hkv: int
    Tq: int
    Tk: int
    d: int
    dv: int
    causal: bool = True
    window: int = 0
    softcap: float = 0.0
    normalizers: tuple = ("softmax", "softmax1", "sparsemax", "entmax15")
    seed: int = 1000
    q_gain: float = 1.0          # multiplies Q after drawing (temperature)
    kv_gain: float = 1.0         # multiplies Q, K and V (value spread)
    rms_qk: bool = False         # RMS-normalise Q/K rows (QK-norm-like)
    paged: bool = False
    page_size: int = 64
    len_range: tuple = (0, 0)    # paged: inclusive range of key lengths
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def scale(self):
        return 1.0 / (self.d ** 0.5)

    def useful_flops(self):
        """Useful forward FLOPs by the accounting rule of "Attention
        variants" (TensorCAD), section "What the engine does today":
        ``4 * T_eff * head_dim`` per query row and head, halved when causal,
        with ``T_eff`` the window when there is one."""
        t_eff = self.window if self.window > 0 else self.Tk
        f = 4.0 * self.B * self.Hq * self.Tq * t_eff * self.d
        return f / 2 if self.causal else f


WORKLOADS = {
    # tiny correctness case, all four normalizers, dense weights returned
    "tiny": Workload("tiny", 1, 2, 1, 64, 64, 32, 32, causal=False,
                     seed=1001),
    "tiny_causal": Workload("tiny_causal", 1, 2, 1, 64, 64, 32, 32,
                            causal=True, seed=1001),
    # Qwen3-8B-shaped prefill layer, GQA 4:1, QK-norm-like inputs
    "qwen3_8b_prefill": Workload("qwen3_8b_prefill", 2, 32, 8, 4096, 4096,
                                 128, 128, causal=True, seed=1002,
                                 rms_qk=True,
                                 normalizers=("softmax", "softmax1")),
    # sparse normalizers at two query temperatures
    "sparse_prefill_t1": Workload("sparse_prefill_t1", 1, 16, 8, 8192, 8192,
                                  128, 128, causal=True, seed=1003,
                                  normalizers=("sparsemax", "entmax15")),
    "sparse_prefill_t4": Workload("sparse_prefill_t4", 1, 16, 8, 8192, 8192,
                                  128, 128, causal=True, seed=1003,
                                  q_gain=4.0,
                                  normalizers=("sparsemax", "entmax15")),
    # the same at a quarter of the query scale: flat score rows and wide
    # supports (about 200 keys per row for 1.5-entmax, against about 23 at
    # Q x1), beyond the threshold pass's candidate buffers
    "sparse_prefill_wide": Workload("sparse_prefill_wide", 1, 16, 8, 8192, 8192,
                                    128, 128, causal=True, seed=1003,
                                    q_gain=0.25,
                                    normalizers=("sparsemax", "entmax15")),
    # Gemma-2-9B-shaped local (window 4096) and global layers, soft-cap 50
    "gemma2_9b_local": Workload("gemma2_9b_local", 1, 16, 8, 8192, 8192, 256,
                                256, causal=True, window=4096, softcap=50.0,
                                seed=1004, kv_gain=0.5,
                                normalizers=("softmax", "softmax1")),
    "gemma2_9b_global": Workload("gemma2_9b_global", 1, 16, 8, 8192, 8192,
                                 256, 256, causal=True, softcap=50.0,
                                 seed=1004, kv_gain=0.5,
                                 normalizers=("softmax", "softmax1")),
    # paged decode batch: 64 sequences, lengths uniform in [1024, 32768]
    "paged_decode": Workload("paged_decode", 64, 32, 8, 1, 0, 128, 128,
                             causal=True, seed=1005, paged=True,
                             page_size=64, len_range=(1024, 32768)),
}


def _bf16(x):
    return x.to(torch.bfloat16)


def _draw(gen, shape, gain=1.0):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if gain != 1.0:
        x = x * gain
    return x


def _rms(x):
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True))


def make_dense(w: Workload, seed=None):
    """Dense bf16 CPU tensors q [B,Hq,Tq,d], k/v [B,Hkv,Tk,d|dv].

    Draw order: q, k, v.  Q/K rows are RMS-normalised in float32 when
    ``rms_qk``; ``kv_gain`` scales all three, ``q_gain`` scales q (both
    powers of two or exact halves in the configured workloads, so the bf16
    rounding is the same as drawing at that scale)."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    q = _draw(gen, (w.B, w.Hq, w.Tq, w.d), w.kv_gain)
    k = _draw(gen, (w.B, w.Hkv, w.Tk, w.d), w.kv_gain)
    v = _draw(gen, (w.B, w.Hkv, w.Tk, w.dv), w.kv_gain)
    if w.rms_qk:
        q, k = _rms(q), _rms(k)
    q = _bf16(q)
    if w.q_gain != 1.0:
        q = _bf16(q.float() * w.q_gain)
    return {"q": q, "k": _bf16(k), "v": _bf16(v)}


def make_paged(w: Workload, seed=None):
    """Paged decode inputs.

    Draw order: sequence lengths (uniform integers in ``len_range``,
    inclusive), q, then the K/V pool, then the page permutation.  The pool
    holds exactly ``sum ceil(len / page)`` pages, laid out
    [num_pages, Hkv, page, d]; the block table [B, max_pages] assigns a
    random permutation of the pool to the sequences in order and pads with
    -1."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    lo, hi = w.len_range
    lens = torch.randint(lo, hi + 1, (w.B,), generator=gen, dtype=torch.int64)
    npages = (lens + w.page_size - 1) // w.page_size
    P = int(npages.sum())
    q = _bf16(_draw(gen, (w.B, w.Hq, w.Tq, w.d), w.kv_gain))
    k_pool = torch.empty((P, w.Hkv, w.page_size, w.d), dtype=torch.bfloat16)
    v_pool = torch.empty((P, w.Hkv, w.page_size, w.dv), dtype=torch.bfloat16)
    chunk = 1024
    for pool in (k_pool, v_pool):
        for s in range(0, P, chunk):
            e = min(P, s + chunk)
            pool[s:e] = _bf16(_draw(gen, (e - s,) + tuple(pool.shape[1:]),
                                    w.kv_gain))
    perm = torch.randperm(P, generator=gen).to(torch.int32)
    maxp = int(npages.max())
    table = torch.full((w.B, maxp), -1, dtype=torch.int32)
    off = 0
    for b in range(w.B):
        n = int(npages[b])
        table[b, :n] = perm[off:off + n]
        off += n
    return {"q": q, "k_pool": k_pool, "v_pool": v_pool, "block_table": table,
            "seqlens": lens.to(torch.int32)}


def make_inputs(w: Workload, seed=None):
    return make_paged(w, seed) if w.paged else make_dense(w, seed)


def shrink(w: Workload, **kw):
    """A smaller copy of a workload with the same recipe (for parity runs
    the oracle finishes in seconds)."""
    return replace(w, **kw)
