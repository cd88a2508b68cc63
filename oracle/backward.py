"""Plain float64 gradients of ``O = N(scale * Q K^T + mask) V``.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA path never
imports this module.

The backward pass the pages describe keeps only the forward's per-row
statistic (the log-sum-exp for softmax / softmax1, the threshold for the
sparse normalizers) and recomputes the probabilities to accumulate the
query, key and value gradients ("HF Attention Normalizers", section
"Important Limitations": softmax1 saves row max / denominator statistics and
recomputes probabilities during the fused backward; the sparse kernels save
one threshold per query row and recompute tiles during the fused backward).
This module states what those gradients are, with nothing blocked or fused:
each row's probabilities come from the forward row functions, and each row's
vector-Jacobian product is the normalizer's own Jacobian applied to
``g = dL/dp``:

* softmax, softmax1, softmax with a learned sink: ``dp_i/dz_j = p_i (delta_ij
  - p_j)`` (the sink is one more logit with a zero value row; its own weight
  takes no gradient), so ``dz = p * (g - sum_j p_j g_j)``;
* sparsemax: on the support S the map is ``z -> z - tau`` with tau the mean
  shift, so ``dz = s * (g - mean_S(g))``, ``s = 1[p > 0]`` (Martins and
  Astudillo, 2016, the sparsemax Jacobian);
* 1.5-entmax: with ``s = sqrt(p) = relu(z/2 - tau)`` the Jacobian is
  ``diag(s) - s s^T / sum(s)`` (Peters, Niculae and Martins, 2019, the
  alpha-entmax Jacobian at alpha = 1.5; the factor 1/2 of ``u = z/2`` and the
  2 of ``p = s^2`` cancel), so ``dz = s * (g - sum(s g) / sum(s))``.

Then the score transform's chain rule (``z = cap * tanh(scale * s / cap)``
gives ``dz/ds = scale * (1 - tanh^2)``; no cap: ``scale``) and the two
matrix products, with grouped-query heads summed into their key/value head.
"""

import numpy as np

from .attention import (_f64, allowed_matrix, block_allowed, normalize_row,
                        softmax_sink_row, transform_scores)


def row_vjp(p, g, normalizer):
    """``dL/dz`` of one row from its weights ``p`` (visible keys only) and
    ``g = dL/dp``, by the Jacobian of the row's normalizer."""
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    if p.size == 0:
        return p.copy()
    if normalizer in ("softmax", "softmax1"):
        return p * (g - np.dot(p, g))
    if normalizer == "sparsemax":
        s = (p > 0).astype(np.float64)
        return s * (g - np.dot(s, g) / s.sum())
    if normalizer == "entmax15":
        s = np.sqrt(p)
        return s * (g - np.dot(s, g) / s.sum())
    raise ValueError(normalizer)


def attention_bwd(q, k, v, dout, scale, normalizer, causal=False, window=0,
                  softcap=0.0, sinks=None, block_mask=None):
    """Gradients ``(dq, dk, dv)`` of ``L = sum(dout * O)`` for the forward of
    ``attention_fwd`` with the same arguments.  Shapes as in the forward:
    ``q`` [B, Hq, Tq, d], ``k`` [B, Hkv, Tk, d], ``v`` [B, Hkv, Tk, dv],
    ``dout`` [B, Hq, Tq, dv]; query head ``h`` reads key/value head
    ``h // (Hq // Hkv)``, so ``dk`` and ``dv`` sum over the heads of a group.
    ``sinks`` (length Hq) only with softmax; ``block_mask`` as in the
    forward.  Returns float64 arrays."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Tq, d = q.shape
    _, Hkv, Tk, _ = k.shape
    group = Hq // Hkv
    if sinks is not None:
        assert normalizer == "softmax", "sinks go with softmax"
        sinks = np.asarray(_f64(sinks), dtype=np.float64).reshape(-1)
    ok = allowed_matrix(Tq, Tk, causal, window)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = h // group
            s = q[b, h] @ k[b, g].T                      # raw dot products
            z = transform_scores(s, scale, softcap)
            if softcap > 0:
                dzds = scale * (1.0 - np.tanh(scale * s / softcap) ** 2)
            else:
                dzds = np.full_like(s, scale)
            ok_bh = ok if block_mask is None else \
                ok & block_allowed(block_mask[b, h], Tq, Tk)
            P = np.zeros((Tq, Tk))
            dZ = np.zeros((Tq, Tk))
            dP = dout[b, h] @ v[b, g].T                  # dL/dp
            for i in range(Tq):
                m = ok_bh[i]
                if sinks is None:
                    p, _ = normalize_row(z[i][m], normalizer)
                else:
                    p, _ = softmax_sink_row(z[i][m], sinks[h])
                P[i, m] = p
                dZ[i, m] = row_vjp(p, dP[i][m], normalizer)
            dS = dZ * dzds
            dq[b, h] = dS @ k[b, g]
            dk[b, g] += dS.T @ q[b, h]
            dv[b, g] += P.T @ dout[b, h]
    return dq, dk, dv
