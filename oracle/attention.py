"""Plain float64 restatement of ``O = N(scale * Q K^T + mask) V``.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA path never
imports this module.

Nothing here is blocked, fused or reordered: scores are materialised with a
float64 matrix product, the mask is applied by exclusion, and each row goes
through its normalizer on its own, exactly in the order the definitions give.
"""

import math

import numpy as np

NORMALIZERS = ("softmax", "softmax1", "sparsemax", "entmax15")


# --------------------------------------------------------------------------
# Masking and score transform
# --------------------------------------------------------------------------

def allowed_matrix(Tq, Tk, causal, window):
    """Boolean [Tq, Tk]: may query ``i`` attend to key ``j``?

    Causal masking hides future positions ("Attention variants", TensorCAD,
    parameter table, row ``causal``).  When query and key lengths differ the
    causal diagonal is aligned bottom-right, so query ``i`` sits at key
    position ``i + (Tk - Tq)`` ("HF Attention Normalizers", section "Packed
    Variable-Length Attention").  The sliding window keeps
    ``(q >= k) and (q - k < window)`` ("attention interface", section "common
    flexattention patterns", sliding window; the same rule as the
    ``and_masks(causal, window)`` example on the tensorplay ``nn.attention``
    page).  ``window == 0`` means no window.  Without ``causal`` a window is
    read as two-sided, ``|q - k| < window`` (a reading: the pages only show
    the causal window).
    """
    pos = np.arange(Tq)[:, None] + (Tk - Tq)
    j = np.arange(Tk)[None, :]
    ok = np.ones((Tq, Tk), dtype=bool)
    if causal:
        ok &= j <= pos
    if window > 0:
        if causal:
            ok &= (pos - j) < window
        else:
            ok &= np.abs(pos - j) < window
    return ok


BLOCK = 128  # side of one block of a block mask


def block_allowed(block_mask_bh, Tq, Tk):
    """Boolean [Tq, Tk] of one (batch, head) block mask: a block mask keeps or
    drops whole 128 x 128 blocks of (query, key) pairs ("Attention variants",
    TensorCAD, section "C. Keep the fused kernel": a mask also yields a block
    mask, and whole blocks that are masked out are skipped).
    ``block_mask_bh`` is [ceil(Tq/128), ceil(Tk/128)], nonzero = keep."""
    bm = np.asarray(block_mask_bh) != 0
    return bm[np.arange(Tq)[:, None] // BLOCK, np.arange(Tk)[None, :] // BLOCK]


def transform_scores(s, scale, softcap):
    """Scale the raw dot products, then apply the logit soft-cap.

    ``cap * tanh(score / cap)`` is the ``logit_softcap`` switch of the
    "Attention variants" (TensorCAD) parameter table, as used by Gemma 2;
    ``softcap == 0`` disables it.  Order: scale, then cap, then mask.
    """
    z = scale * np.asarray(s, dtype=np.float64)
    if softcap > 0:
        z = softcap * np.tanh(z / softcap)
    return z


# --------------------------------------------------------------------------
# Row normalizers.  Each takes the allowed scores of one query row
# (1-D float64) and returns (p, row_stat).
# --------------------------------------------------------------------------

def softmax_row(z):
    """Vanilla softmax ``exp(z_i) / sum_j exp(z_j)`` ("HF Attention
    Normalizers", "Supported Normalizers" table, row ``vanilla / softmax``).

    row_stat is the natural-log log-sum-exp.  An empty row (every key
    masked) gives no weights and ``-inf``.
    """
    z = np.asarray(z, dtype=np.float64)
    if z.size == 0:
        return z.copy(), -math.inf
    m = z.max()
    e = np.exp(z - m)
    s = e.sum()
    return e / s, m + math.log(s)


def softmax1_row(z):
    """softmax1 ``exp(z_i) / (1 + sum_j exp(z_j))`` ("HF Attention
    Normalizers", "Supported Normalizers" table, row ``softmax1``, Softmax-N
    with n = 1).  The ``1`` is the virtual logit-0 sink of section
    "Important Limitations", so the largest logit used for stability is
    ``max(0, max z)``.  row_stat is ``log(1 + sum exp z)``; an empty row
    gives no weights and ``0``.
    """
    z = np.asarray(z, dtype=np.float64)
    m = max(0.0, float(z.max())) if z.size else 0.0
    e = np.exp(z - m)
    s = math.exp(-m) + e.sum()
    return e / s, m + math.log(s)


def softmax_sink_row(z, sink):
    """softmax with a learned attention sink: ``exp(z_i) / (exp(s) +
    sum_j exp(z_j))`` for the row's sink logit ``s`` ("Attention variants:
    what to open up, and how far", TensorCAD, variants table, row "Attention
    sinks": gpt-oss adds a learned per-head term to the softmax's
    denominator).  The sink is one more logit whose value row is zero, so
    this is softmax over ``[z, s]`` with the sink's own weight dropped.
    ``s = 0`` is softmax1; ``s = -inf`` is plain softmax.  row_stat is
    ``log(exp(s) + sum exp z)``; an empty row gives no weights and ``s``.
    """
    z = np.asarray(z, dtype=np.float64)
    s = float(sink)
    m = max(s, float(z.max())) if z.size else s
    if m == -math.inf:          # no sink and no visible key
        return z.copy(), -math.inf
    e = np.exp(z - m)
    tot = math.exp(s - m) + e.sum()
    return e / tot, m + math.log(tot)


def sparsemax_row(z):
    """sparsemax: Euclidean projection of ``z`` onto the probability simplex
    ("HF Attention Normalizers", "Supported Normalizers": a sparse probability
    transform with exact zeros; the projection reading follows Martins and
    Astudillo, 2016).

    Exact sort-based threshold: with ``z`` sorted in decreasing order the
    support size is the largest ``k`` with ``1 + k z_(k) > sum_{r<=k} z_(r)``
    and ``tau = (sum_{r<=k} z_(r) - 1) / k``; ``p = max(z - tau, 0)``.
    row_stat is ``tau`` (``+inf`` for an empty row).
    """
    z = np.asarray(z, dtype=np.float64)
    if z.size == 0:
        return z.copy(), math.inf
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    k = np.arange(1, z.size + 1, dtype=np.float64)
    ok = 1.0 + k * zs > cs
    kstar = int(np.nonzero(ok)[0].max()) + 1
    tau = (cs[kstar - 1] - 1.0) / kstar
    return np.maximum(z - tau, 0.0), tau


def entmax15_row(z):
    """1.5-entmax ("HF Attention Normalizers", "Supported Normalizers": between
    softmax and sparsemax, also sparse).  Reading: alpha-entmax with
    alpha = 1.5 (Peters, Niculae and Martins, 2019), ``p_i = relu(z_i/2 -
    tau)^2`` with ``sum p = 1``.

    Exact sort-based threshold in ``u = z / 2``: with ``u`` sorted in
    decreasing order, a support of the top ``k`` entries needs
    ``sum_{r<=k} (u_(r) - tau)^2 = 1``, whose smaller root is
    ``tau_k = mean_k - sqrt(delta_k)`` with
    ``delta_k = (1 - k * var_k) / k`` (``var_k`` the population variance of
    the top ``k``).  The support size is the largest ``k`` with
    ``delta_k >= 0`` and ``tau_k < u_(k)``.  row_stat is ``tau`` in units of
    ``z / 2`` (``+inf`` for an empty row).
    """
    z = np.asarray(z, dtype=np.float64)
    if z.size == 0:
        return z.copy(), math.inf
    u = z / 2.0
    us = np.sort(u)[::-1]
    k = np.arange(1, u.size + 1, dtype=np.float64)
    mean = np.cumsum(us) / k
    meansq = np.cumsum(us * us) / k
    var = meansq - mean * mean
    delta = (1.0 - k * var) / k
    tau_k = mean - np.sqrt(np.maximum(delta, 0.0))
    ok = (delta >= 0.0) & (tau_k < us)
    kstar = int(np.nonzero(ok)[0].max()) + 1
    tau = float(tau_k[kstar - 1])
    return np.maximum(u - tau, 0.0) ** 2, tau


_ROW_FN = {
    "softmax": softmax_row,
    "softmax1": softmax1_row,
    "sparsemax": sparsemax_row,
    "entmax15": entmax15_row,
}


def normalize_row(z, normalizer):
    """Dispatch to one of the four row normalizers by name."""
    return _ROW_FN[normalizer](z)


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _f64(x):
    """Upcast a tensor or array exactly to a float64 numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def attention_rows(q, k, v, rows, scale, normalizer, causal=False, window=0,
                   softcap=0.0, want_weights=False, sinks=None, block_mask=None):
    """Attention output for selected query rows.

    ``q`` [B, Hq, Tq, d], ``k`` [B, Hkv, Tk, d], ``v`` [B, Hkv, Tk, dv]
    (anything numpy can upcast; bf16 tensors are upcast exactly).  ``rows``
    is an int array [n, 3] of (b, h, i).  Query head ``h`` reads key/value
    head ``h // (Hq // Hkv)``: the backend receives query/key/value after
    grouped-query expansion ("Attention", factory.ai wiki, "What every
    backend must support"), and the reading here is the contiguous grouping
    of that expansion.

    ``sinks`` (length Hq, natural-log logits) turns softmax into softmax
    with a learned per-head sink (``softmax_sink_row``); only with
    ``normalizer == "softmax"``.  ``block_mask`` ([B, Hq, ceil(Tq/128),
    ceil(Tk/128)], nonzero = keep) removes whole 128 x 128 blocks on top of
    the causal / window rule (``block_allowed``).

    Returns ``out`` [n, dv], ``row_stat`` [n] and, if asked, dense weights
    [n, Tk] with exact zeros on masked keys.
    """
    if sinks is not None:
        assert normalizer == "softmax", "sinks go with softmax"
        sinks = np.asarray(_f64(sinks), dtype=np.float64).reshape(-1)
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Tq, d = q.shape
    _, Hkv, Tk, _ = k.shape
    dv = v.shape[3]
    group = Hq // Hkv
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    n = rows.shape[0]
    out = np.zeros((n, dv))
    stat = np.zeros(n)
    weights = np.zeros((n, Tk)) if want_weights else None
    ok_all = allowed_matrix(Tq, Tk, causal, window)
    # group the requested rows by (b, h) so each head is one matrix product
    keys = rows[:, 0] * Hq + rows[:, 1]
    for key in np.unique(keys):
        sel = np.nonzero(keys == key)[0]
        b, h = int(key // Hq), int(key % Hq)
        g = h // group
        qi = rows[sel, 2]
        s = q[b, h, qi, :] @ k[b, g].T            # [len(sel), Tk]
        z = transform_scores(s, scale, softcap)
        ok_bh = ok_all if block_mask is None else \
            ok_all & block_allowed(block_mask[b, h], Tq, Tk)
        for t, (r, i) in enumerate(zip(sel, qi)):
            ok = ok_bh[i]
            if sinks is None:
                p, st = normalize_row(z[t][ok], normalizer)
            else:
                p, st = softmax_sink_row(z[t][ok], sinks[h])
            stat[r] = st
            if p.size:
                out[r] = p @ v[b, g][ok]
            if want_weights:
                weights[r, ok] = p
    return out, stat, weights


def attention_fwd(q, k, v, scale, normalizer, causal=False, window=0,
                  softcap=0.0, want_weights=False, sinks=None, block_mask=None):
    """Full attention forward: ``out`` [B, Hq, Tq, dv], ``row_stat``
    [B, Hq, Tq] and optionally ``weights`` [B, Hq, Tq, Tk] (float64)."""
    qa = _f64(q)
    B, Hq, Tq, _ = qa.shape
    Tk = _f64(k).shape[2]
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(Tq),
                             indexing="ij")
    rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    out, stat, w = attention_rows(qa, k, v, rows, scale, normalizer, causal,
                                  window, softcap, want_weights, sinks,
                                  block_mask)
    dv = out.shape[1]
    out = out.reshape(B, Hq, Tq, dv)
    stat = stat.reshape(B, Hq, Tq)
    if want_weights:
        w = w.reshape(B, Hq, Tq, Tk)
    return out, stat, w


# --------------------------------------------------------------------------
# Packed variable-length sequences
# --------------------------------------------------------------------------

def varlen_attention(q, k, v, cu_q, cu_k, scale, normalizer, causal=False,
                     window=0, softcap=0.0, sinks=None):
    """Packed variable-length attention ("HF Attention Normalizers", section
    "Packed Variable-Length Attention": FlashAttention-style packed layouts
    with cumulative sequence lengths, per-request bottom-right causal
    alignment, GQA, different query and key lengths).

    ``q`` [total_q, Hq, d], ``k`` [total_k, Hkv, d], ``v`` [total_k, Hkv, dv];
    sequence ``b`` owns query tokens ``[cu_q[b], cu_q[b+1])`` and key tokens
    ``[cu_k[b], cu_k[b+1])`` and is an attention problem of its own.  Returns
    ``out`` [total_q, Hq, dv] and ``row_stat`` [total_q, Hq]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    total_q, Hq, _ = q.shape
    dv = v.shape[2]
    out = np.zeros((total_q, Hq, dv))
    stat = np.zeros((total_q, Hq))
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 == q0:
            continue
        qs = q[q0:q1].transpose(1, 0, 2)[None]
        ks = k[k0:k1].transpose(1, 0, 2)[None]
        vs = v[k0:k1].transpose(1, 0, 2)[None]
        o, st, _ = attention_fwd(qs, ks, vs, scale, normalizer, causal, window,
                                 softcap, sinks=sinks)
        out[q0:q1] = o[0].transpose(1, 0, 2)
        stat[q0:q1] = st[0].T
    return out, stat


# --------------------------------------------------------------------------
# Paged KV cache
# --------------------------------------------------------------------------

def paged_gather(k_pool, v_pool, block_table, seqlen, b, page_size):
    """Logical K/V of sequence ``b`` read through its block table.

    The cache is a pool of fixed-size pages; ``block_table[b, p]`` names the
    physical page holding logical positions ``[p*page, (p+1)*page)`` ("HF
    Attention Normalizers", section "Differentiable Paged Attention":
    ``key_cache, value_cache, block_table, sequence_lengths, block_size``).
    Pool layout (a reading; the pages give none): [num_pages, Hkv, page, d].
    Returns k [Hkv, seqlen, d], v [Hkv, seqlen, dv].
    """
    k_pool, v_pool = _f64(k_pool), _f64(v_pool)
    bt = np.asarray(block_table)
    npages = -(-int(seqlen) // page_size)
    ks, vs = [], []
    for p in range(npages):
        page = int(bt[b, p])
        ks.append(k_pool[page])
        vs.append(v_pool[page])
    kk = np.concatenate(ks, axis=1)[:, :seqlen]
    vv = np.concatenate(vs, axis=1)[:, :seqlen]
    return kk, vv


def paged_decode(q, k_pool, v_pool, block_table, seqlens, page_size, scale,
                 normalizer, causal=True, window=0, softcap=0.0, seqs=None,
                 sinks=None):
    """Attention of ``q`` [B, Hq, Tq, d] over each sequence's paged K/V.

    Each sequence has its own key length ``seqlens[b]``; the query rows are
    aligned bottom-right against it (so with ``Tq == 1`` the single query
    sees every key).  ``seqs`` restricts the work to some sequences.
    Returns ``{b: (out [Hq, Tq, dv], row_stat [Hq, Tq])}``.
    """
    qa = _f64(q)
    B, Hq, Tq, _ = qa.shape
    lens = np.asarray(seqlens)
    res = {}
    for b in (range(B) if seqs is None else seqs):
        kk, vv = paged_gather(k_pool, v_pool, block_table, int(lens[b]), b,
                              page_size)
        o, st, _ = attention_fwd(qa[b:b + 1], kk[None], vv[None], scale,
                                 normalizer, causal, window, softcap,
                                 sinks=sinks)
        res[int(b)] = (o[0], st[0])
    return res
