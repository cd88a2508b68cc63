"""Float64 CPU oracle for attention with a selectable row normalizer.

TEST INFRASTRUCTURE ONLY.  This package is the slow, obviously correct
definition that the CUDA kernels are checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The product path
(``alternative_normalizers_b200``) never imports, calls or links anything
here, and nothing here imports the product package: the two share no code.

Every function cites the passage of the source pages it restates:

* "HF Attention Normalizers" (PyPI project page), section "Supported
  Normalizers" (the table defining softmax1, sparsemax, entmax15 and vanilla
  softmax) and section "Important Limitations" (softmax1 as a virtual
  logit-0 / value-0 sink; one threshold per query row for the sparse
  normalizers).
* "attention interface" (transformers-v5 wiki), section "common
  flexattention patterns" (the sliding-window rule ``(q >= k) and
  (q - k < window_size)``).
* "Attention variants: what to open up, and how far" (TensorCAD docs),
  section "What the engine does today" (the parameter table: heads/kv_heads,
  head_dim/v_head_dim, causal, window, logit_softcap ``cap*tanh(score/cap)``).
* "Attention" (factory.ai transformers wiki), section "What every backend
  must support" (query/key/value after grouped-query expansion, scaling,
  is_causal; output plus optional weights).
* "HF Attention Normalizers", section "Packed Variable-Length Attention"
  (bottom-right causal alignment when query and key lengths differ).
* "HF Attention Normalizers", section "Important Limitations" for the
  backward pass (saved row statistics, probabilities recomputed; gradients
  in ``backward.py``).
* "Attention variants: what to open up, and how far" (TensorCAD docs),
  variants table, row "Attention sinks" (a learned per-head term in the
  softmax's denominator).

Readings where the pages are silent:
sparsemax is the Euclidean projection onto the probability simplex;
1.5-entmax is ``p_i = relu(z_i/2 - tau)^2`` with ``sum p = 1`` and its
threshold is reported in units of ``z/2``; scores are scaled, then soft-capped,
then masked; query head ``h`` reads key/value head ``h // (Hq // Hkv)``.
"""

from .attention import (  # noqa: F401
    NORMALIZERS,
    allowed_matrix,
    block_allowed,
    transform_scores,
    softmax_row,
    softmax1_row,
    softmax_sink_row,
    sparsemax_row,
    entmax15_row,
    normalize_row,
    attention_fwd,
    attention_rows,
    paged_gather,
    paged_decode,
    varlen_attention,
)
from .backward import attention_bwd, row_vjp  # noqa: F401
