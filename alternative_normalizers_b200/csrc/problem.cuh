// The attention problem as the kernels see it, plus the two index rules
// every kernel shares: which keys a query row may see, and where a key row
// lives (dense tensor or paged pool).
#pragma once

#include "common.cuh"

namespace nattn {

struct Problem {
  const bf16* q;
  const bf16* k;
  const bf16* v;
  bf16* out;
  float* row_stat;
  float* weights;
  int32_t* row_nnz;  // keys with a nonzero weight per row, or null
  int B, Hq, Hkv, Tq, Tk, d, dv;
  float scale;
  int norm;
  int causal;
  int window;
  float softcap;
  // learned per-head attention sinks: logit of a value-0 sink in the
  // softmax denominator of query head h (natural-log units), or null
  const float* sinks;
  // block mask [B, Hq, bm_nq, bm_nk] (nonzero = keep the 128 x 128 block of
  // (query, key) pairs) or null; bm_nq = ceil(Tq / 128), bm_nk = ceil(Tk / 128)
  const uint8_t* block_mask;
  int bm_nq, bm_nk;
  // paged mode (block_table != nullptr)
  const int32_t* block_table;
  const int32_t* seqlens;
  int page_size, bt_stride, num_pages;
  // packed variable-length mode (cu_q != nullptr): q [total_q, Hq, d],
  // k / v [total_k, Hkv, d | dv], out [total_q, Hq, dv], row_stat and
  // row_nnz [total_q, Hq]; sequence b owns query tokens [cu_q[b], cu_q[b+1])
  // and key tokens [cu_k[b], cu_k[b+1]); Tq / Tk are the largest lengths
  const int32_t* cu_q;
  const int32_t* cu_k;
  int total_q, total_k;
};

// One sequence's lengths and, in packed mode, its first query / key token.
// Lengths outside the declared bounds are recorded as NATTN_EBOUNDS and the
// sequence is treated as empty.
struct SeqInfo {
  int Lq, Lk, q0, k0;
};

__device__ __forceinline__ SeqInfo seq_info(const Problem& P, int b) {
  SeqInfo s{P.Tq, P.Tk, 0, 0};
  if (P.cu_q != nullptr) {
    s.q0 = P.cu_q[b];
    s.k0 = P.cu_k[b];
    s.Lq = P.cu_q[b + 1] - s.q0;
    s.Lk = P.cu_k[b + 1] - s.k0;
    if (s.q0 < 0 || s.k0 < 0 || s.Lq < 0 || s.Lk < 0 || s.Lq > P.Tq || s.Lk > P.Tk ||
        s.q0 + s.Lq > P.total_q || s.k0 + s.Lk > P.total_k) {
      set_status(NATTN_EBOUNDS);
      s.Lq = s.Lk = 0;
      s.q0 = s.k0 = 0;
    }
  } else if (P.block_table != nullptr) {
    s.Lk = P.seqlens[b];
    if (s.Lk < 0 || s.Lk > P.Tk || s.Lk > P.bt_stride * P.page_size) {
      set_status(NATTN_EBOUNDS);
      s.Lk = 0;
    }
  }
  return s;
}

// Flat index of query row i of head h of sequence b: the row of out,
// row_stat and row_nnz (and of every per-row scratch array).
__device__ __forceinline__ size_t row_index(const Problem& P, int b, int h, int i,
                                            const SeqInfo& s) {
  return P.cu_q != nullptr ? (size_t)(s.q0 + i) * P.Hq + h
                           : ((size_t)b * P.Hq + h) * P.Tq + i;
}

// Inclusive key range [lo, hi] visible to query row i when the row's key
// length is L.  The query sits at key position pos = i + L - Tq (causal
// diagonal aligned bottom-right, "HF Attention Normalizers", section "Packed
// Variable-Length Attention").  Causal keeps j <= pos; a window W keeps
// pos - j < W ("attention interface" wiki, "common flexattention patterns",
// sliding window), and without causal also j - pos < W.  The visible set is
// always one contiguous range (possibly empty: hi < lo).
struct RowRange {
  int lo, hi;
};

__host__ __device__ __forceinline__ RowRange row_range(int Tq, int causal, int window,
                                                       int i, int L) {
  const int pos = i + L - Tq;
  int lo = 0, hi = L - 1;
  if (causal && pos < hi) hi = pos;
  if (window > 0) {
    if (pos - window + 1 > lo) lo = pos - window + 1;
    if (!causal && pos + window - 1 < hi) hi = pos + window - 1;
  }
  return RowRange{lo, hi};
}

__device__ __forceinline__ RowRange row_range(const Problem& P, int i, int L) {
  return row_range(P.Tq, P.causal, P.window, i, L);
}

// Logit of the value-0 sink in the denominator of query head h, natural-log
// units: the learned per-head sink when given ("Attention variants",
// TensorCAD, variants table, row "Attention sinks": a learned per-head term
// in the softmax's denominator), 0 for softmax1 (its virtual logit-0 sink,
// "HF Attention Normalizers", section "Important Limitations"), else -inf
// (no sink).
__device__ __forceinline__ float sink_logit(const Problem& P, int h) {
  if (P.sinks != nullptr) return P.sinks[h];
  return P.norm == NATTN_SOFTMAX1 ? 0.f : -INFINITY;
}

// Block mask: is the 128 x 128 block (query block qb, key block kb) of query
// head h of batch b kept?  Whole blocks that a mask drops are skipped
// ("Attention variants", TensorCAD, section "C. Keep the fused kernel": a
// mask yields a block mask, and masked-out blocks are skipped).  Always true
// without a block mask.
__device__ __forceinline__ bool block_kept(const Problem& P, int b, int h, int qb, int kb) {
  if (P.block_mask == nullptr) return true;
  return P.block_mask[(((size_t)b * P.Hq + h) * P.bm_nq + qb) * P.bm_nk + kb] != 0;
}

// Key blocks of BN keys (BN = 64 or 128) in [kb, kend) that heads h0 or h1
// keep for query block qb: the next one at or after kb, and how many there
// are.  Every role of a kernel walks the same sequence.
template <int BN>
__device__ __forceinline__ int next_kept(const Problem& P, int b, int h0, int h1, int qb, int kb,
                                         int kend) {
  if (P.block_mask == nullptr) return kb;
  while (kb < kend && !block_kept(P, b, h0, qb, (kb * BN) >> 7) &&
         !block_kept(P, b, h1, qb, (kb * BN) >> 7))
    ++kb;
  return kb;
}
template <int BN>
__device__ __forceinline__ int count_kept(const Problem& P, int b, int h0, int h1, int qb, int kb,
                                          int kend) {
  if (P.block_mask == nullptr) return kend - kb;
  int n = 0;
  for (; kb < kend; ++kb)
    n += (block_kept(P, b, h0, qb, (kb * BN) >> 7) || block_kept(P, b, h1, qb, (kb * BN) >> 7))
             ? 1
             : 0;
  return n;
}

// Address of key (or value) row j of sequence b, kv head g.  Dense layout
// [B, Hkv, Tk, dim]; packed layout [total_k, Hkv, dim]; paged pool
// [num_pages, Hkv, page_size, dim] through the block table.  An
// out-of-range page id sets `bad` and returns nullptr.
__device__ __forceinline__ const bf16* key_row(const Problem& P, const bf16* base, int dim,
                                               int b, int g, int j, bool& bad) {
  if (P.cu_q != nullptr) return base + ((size_t)(P.cu_k[b] + j) * P.Hkv + g) * dim;
  if (P.block_table == nullptr)
    return base + (((size_t)b * P.Hkv + g) * P.Tk + j) * dim;
  const int page = P.block_table[(size_t)b * P.bt_stride + j / P.page_size];
  if (page < 0 || page >= P.num_pages) {
    bad = true;
    return nullptr;
  }
  return base + (((size_t)page * P.Hkv + g) * P.page_size + (j % P.page_size)) * dim;
}

// One step of the threshold iteration.  With w the scores in threshold units
// less the row maximum, g(t) = sum relu(w - t)^k - 1 (k = 1 for sparsemax,
// 2 for 1.5-entmax) is convex and decreasing and its root is tau.  From the
// count, sum, sum of squares and minimum of the w above the iterate t, the
// closed-form threshold of that set is accepted once it satisfies the
// optimality conditions (every member of the set above it; the set holds
// everything above t, and t stays at or below the root); otherwise Newton's
// method moves t right, never past the root, so {w > t} always contains the
// support.  For sparsemax this is Michelot's projection algorithm.  Returns
// 1 when t is now the threshold, 0 when t moved and another step is needed,
// -1 when no progress is possible (t stays a lower bound of the threshold).
__device__ __forceinline__ int tau_step(float cnt, float s1, float s2, float wmin, bool entmax,
                                        float& t) {
  float ts, tn;
  bool valid = true;
  if (!entmax) {
    ts = (s1 - 1.f) / cnt;
    tn = ts;
  } else {
    const float mu = s1 / cnt;
    const float delta = (1.f - (s2 - s1 * mu)) / cnt;
    valid = delta >= 0.f;
    ts = valid ? mu - sqrtf(delta) : -INFINITY;
    const float g = s2 - 2.f * t * s1 + t * t * cnt;
    const float gp = 2.f * (s1 - t * cnt);
    tn = t + (g - 1.f) / gp;
  }
  if (valid && ts >= t && wmin > ts) {
    t = ts;
    return 1;
  }
  if (!(tn > t)) return -1;
  t = tn;
  return 0;
}

}  // namespace nattn
