/*
 * libnattn: fused attention forward with a selectable row normalizer, for
 * NVIDIA B200 (sm_100a).
 *
 *     O = N(scale * Q K^T + mask) V
 *
 * The backend contract follows "Attention" (factory.ai transformers wiki),
 * section "What every backend must support": query, key and value after
 * grouped-query expansion, a mask, the scaling factor and is_causal in; the
 * attention output and, on request, the attention weights out.  Here the
 * grouped-query expansion is done inside the kernels (key/value heads are
 * passed unexpanded, query head h reads key/value head h / (Hq / Hkv)).
 *
 * The normalizers are those of "HF Attention Normalizers" (PyPI project
 * page), section "Supported Normalizers":
 *   NATTN_SOFTMAX    exp(z_i) / sum_j exp(z_j)
 *   NATTN_SOFTMAX1   exp(z_i) / (1 + sum_j exp(z_j))   (Softmax-N, n = 1)
 *   NATTN_SPARSEMAX  Euclidean projection onto the probability simplex,
 *                    p_i = max(z_i - tau, 0)
 *   NATTN_ENTMAX15   1.5-entmax, p_i = max(z_i / 2 - tau, 0)^2
 *
 * The mask switches are those of the "sdpa" primitive in "Attention variants:
 * what to open up, and how far" (TensorCAD), section "What the engine does
 * today": causal, sliding window, and the Gemma-2 logit soft-cap
 * cap * tanh(score / cap).  Scores are scaled, then capped, then masked.
 *
 * Conventions for every entry point:
 *   - All tensors are contiguous, row-major, in device memory, and start on a
 *     16-byte boundary.  Q/K/V/O are bfloat16; row_stat and weights float32;
 *     block tables and sequence lengths int32.
 *   - The caller owns every buffer.  nattn_fwd_ex allocates nothing; nattn_fwd
 *     allocates stream-ordered scratch (cudaMallocAsync / cudaFreeAsync on
 *     the given stream) only when the chosen path needs it.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and return after launching.  Errors found on the host
 *     are returned before anything is launched; errors found on the device
 *     (a bad block-table entry, a bounded wait that gave up) are recorded in a
 *     per-device status word read by nattn_get_device_status().
 *   - There is no fallback: an unsupported request returns an error code and
 *     computes nothing ("HF Attention Normalizers", section "Strict vs
 *     Fallback Mode": strict mode raises a clear error).
 */
#ifndef NATTN_H
#define NATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NATTN_SOFTMAX = 0,
  NATTN_SOFTMAX1 = 1,
  NATTN_SPARSEMAX = 2,
  NATTN_ENTMAX15 = 3
} nattn_normalizer;

enum {
  NATTN_OK = 0,
  NATTN_EINVAL = -1,        /* bad argument: NULL pointer, negative size,
                               Hq % Hkv != 0, non-finite scale, ...        */
  NATTN_EUNSUPPORTED = -2,  /* well-formed but outside what the kernels do:
                               d or dv not a multiple of 8 in [8, 256],
                               paged mode with dense weights, ...            */
  NATTN_ETOOLARGE = -3,     /* dense weights asked for more than 2^26 entries,
                               or a size beyond the int32 index range       */
  NATTN_EWORKSPACE = -4,    /* workspace NULL or smaller than
                               nattn_workspace_size()                        */
  NATTN_ECUDA = -5,         /* a CUDA runtime call or kernel launch failed  */
  NATTN_ETIMEOUT = -6,      /* device: a bounded wait gave up               */
  NATTN_EBOUNDS = -7,       /* device: a block-table entry or a sequence
                               length was out of range; the offending work
                               item wrote zeros and was skipped             */
  NATTN_EALIGN = -8         /* q, k, v, out or workspace not 16-byte
                               aligned, or row_stat, weights or row_nnz not
                               4-byte aligned                                */
};

/*
 * Full argument block.
 *
 * Dense mode (block_table == NULL):
 *   q        bf16 [B, Hq, Tq, d]
 *   k        bf16 [B, Hkv, Tk, d]
 *   v        bf16 [B, Hkv, Tk, dv]
 *   Query row i sits at key position i + (Tk - Tq) (causal mask aligned
 *   bottom-right, "HF Attention Normalizers", section "Packed Variable-Length
 *   Attention").
 *
 * Paged mode (block_table != NULL), the paged KV cache of "HF Attention
 * Normalizers", section "Differentiable Paged Attention" (key_cache,
 * value_cache, block_table, sequence_lengths, block_size):
 *   q        bf16 [B, Hq, Tq, d]   (Tq new tokens per sequence; decode: 1)
 *   k        bf16 [num_pages, Hkv, page_size, d]   physical page pool
 *   v        bf16 [num_pages, Hkv, page_size, dv]
 *   block_table  int32 [B, block_table_stride]: logical page p of sequence b
 *                lives in physical page block_table[b * stride + p]
 *   seqlens  int32 [B]: key length of each sequence, 1 <= seqlens[b] <= Tk
 *   Tk       the largest key length any sequence may have (sizes scratch)
 *   Query row i of sequence b sits at key position i + seqlens[b] - Tq.
 *
 * Outputs (both modes):
 *   out      bf16 [B, Hq, Tq, dv]  (rows with no visible key are all zero)
 *   row_stat float32 [B, Hq, Tq] or NULL.  softmax: natural-log
 *            log-sum-exp (-inf for a row with no visible key); softmax1:
 *            log(1 + sum exp z) (0 for such a row); sparsemax: tau; entmax15:
 *            tau in units of z/2 (+inf for such a row).
 *   weights  float32 [B, Hq, Tq, Tk] dense attention weights or NULL (dense
 *            mode only, at most 2^26 entries; masked entries are exactly 0).
 *   row_nnz  int32 [B, Hq, Tq] or NULL: keys with a nonzero weight in each
 *            row.  sparsemax / entmax15: the support size (every other
 *            visible key has a weight of exactly 0); softmax / softmax1: the
 *            number of visible keys.  0 for a row with no visible key.
 *
 * Learned per-head attention sinks ("Attention variants: what to open up,
 * and how far", TensorCAD, variants table, row "Attention sinks": a learned
 * per-head term in the softmax's denominator; section "Recommendation":
 * sinks as a parameter of the primitive):
 *   sinks    float32 [Hq] or NULL, device memory, finite values (-inf: that
 *            head has no sink).  With NATTN_SOFTMAX, query head h normalizes
 *            over its visible scores plus one extra logit sinks[h] whose
 *            value row is zero:
 *                p_j = exp(z_j) / (exp(sinks[h]) + sum_k exp(z_k)),
 *            row_stat = log(exp(sinks[h]) + sum_k exp(z_k)), and a row with
 *            no visible key gets output 0 and row_stat sinks[h].  softmax1 is
 *            the special case sinks[h] = 0.  Any other normalizer with sinks:
 *            NATTN_EUNSUPPORTED.  4-byte aligned (NATTN_EALIGN).
 *
 * Packed variable-length mode (cu_seqlens_q != NULL; "HF Attention
 * Normalizers", section "Packed Variable-Length Attention": FlashAttention-
 * style packed layouts with cumulative sequence lengths, GQA, different
 * query and key lengths, per-request bottom-right causal alignment, one grid
 * over the packed batch with no padded staging):
 *   q        bf16 [total_q, Hq, d]
 *   k        bf16 [total_k, Hkv, d]
 *   v        bf16 [total_k, Hkv, dv]
 *   out      bf16 [total_q, Hq, dv]; row_stat, row_nnz [total_q, Hq]
 *   cu_seqlens_q, cu_seqlens_k  int32 [B + 1], device memory, nondecreasing
 *            from 0: sequence b owns query tokens [cu_seqlens_q[b],
 *            cu_seqlens_q[b+1]) and key tokens [cu_seqlens_k[b],
 *            cu_seqlens_k[b+1]); its query row i sits at key position
 *            i + Lk_b - Lq_b.
 *   Tq, Tk   the largest query and key length of any sequence (they size the
 *            grid; a longer sequence is recorded as NATTN_EBOUNDS on the
 *            device and computed as empty).
 *   total_q, total_k  rows of q and of k / v (>= the last cumulative length).
 * Not with a block table, dense weights or a block mask
 * (NATTN_EUNSUPPORTED).
 *
 * Paged prefill: in paged mode a chunk of Tq new tokens per sequence against
 * a page pool with 32- or 64-token pages runs on the same tensor-core
 * kernels as dense prefill whenever (Hq / Hkv) * Tq > 16 (fewer rows per
 * key/value head go to the split-KV decode kernels).
 *
 * Block mask ("Attention variants: what to open up, and how far",
 * TensorCAD, section "C. Keep the fused kernel": a mask yields a block mask,
 * and whole blocks that are masked out are skipped):
 *   block_mask  uint8 [B, Hq, ceil(Tq/128), ceil(Tk/128)] or NULL, device
 *            memory.  Entry [b, h, qb, kb] == 0 drops every (query, key)
 *            pair of query rows [128 qb, 128 qb + 128) and keys
 *            [128 kb, 128 kb + 128) of query head h, on top of the causal /
 *            window rule; dropped blocks are neither loaded nor multiplied.
 *            Document masks (block-aligned documents), block-level prefix-LM
 *            and block-sparse patterns are block masks.  A row whose visible
 *            keys are all dropped is a row with no visible key.  Dense mode
 *            only (paged mode with a block mask: NATTN_EUNSUPPORTED).
 *
 * window == 0 disables the sliding window; with causal it keeps keys with
 * 0 <= pos - j < window ("attention interface" wiki, section "common
 * flexattention patterns"); without causal it keeps |pos - j| < window.
 * softcap == 0 disables the soft-cap.
 */
typedef struct nattn_args {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* row_stat;
  float* weights;
  int32_t* row_nnz;
  int B, Hq, Hkv, Tq, Tk, d, dv;
  float scale;
  int normalizer;
  int causal;
  int window;
  float softcap;
  const int32_t* block_table;
  const int32_t* seqlens;
  int page_size;
  int block_table_stride;
  int num_pages;
  void* workspace;          /* device scratch, >= nattn_workspace_size(args) */
  size_t workspace_bytes;
  void* stream;             /* cudaStream_t */
  const float* sinks;       /* learned per-head attention sinks, or NULL (see
                               below); NATTN_SOFTMAX only                   */
  const uint8_t* block_mask;/* 128 x 128 block mask, or NULL (see below);
                               dense mode only                              */
  const int32_t* cu_seqlens_q; /* packed variable-length mode (see below),  */
  const int32_t* cu_seqlens_k; /* or NULL                                   */
  int total_q;              /* packed mode: rows of q / out                 */
  int total_k;              /* packed mode: rows of k / v                   */
} nattn_args;

/*
 * Attention forward with the argument list of the backend contract
 * ("Attention", factory.ai transformers wiki, section "What every backend
 * must support"; paged arguments as in "HF Attention Normalizers", section
 * "Differentiable Paged Attention").
 *
 * Dense mode when block_table == NULL.  In paged mode this short form fixes
 * page_size = 64 and block_table_stride = ceil(Tk / 64), and takes the pool
 * size from the device allocations that hold k and v: the pool has as many
 * whole pages [Hkv, 64, d] (and [Hkv, 64, dv]) as fit between k (and v) and
 * the end of the allocation containing it (cuMemGetAddressRange).  A page id
 * at or past that bound is caught on the device (NATTN_EBOUNDS; that row's
 * work is skipped), so a bad table never reads memory the process does not
 * own; with a sub-allocating allocator the bound is the enclosing segment,
 * not the tensor.  k or v outside any device allocation of this process:
 * NATTN_EINVAL.  Use nattn_fwd_ex for other page sizes, strides or an exact
 * page count.  Scratch the chosen path needs is allocated and freed
 * stream-ordered (cudaMallocAsync / cudaFreeAsync) on `stream`.
 * Returns NATTN_OK or a negative error code.
 */
int nattn_fwd(const void* q, const void* k, const void* v, void* out,
              float* row_stat, int B, int Hq, int Hkv, int Tq, int Tk, int d,
              int dv, float scale, int normalizer, int causal, int window,
              float softcap, const int32_t* block_table,
              const int32_t* seqlens, void* stream);

/* Attention forward from a full argument block; allocates nothing.  The
 * caller passes scratch of at least nattn_workspace_size(a) bytes (NULL is
 * fine when that size is 0).  Returns NATTN_OK or a negative error code. */
int nattn_fwd_ex(const nattn_args* a);

/* Bytes of device scratch nattn_fwd_ex needs for these arguments (pointers
 * are not read).  Returns 0 for an invalid argument block. */
size_t nattn_workspace_size(const nattn_args* a);

/*
 * Backward pass: gradients of L = sum(grad_out * O) with respect to q, k and
 * v, recomputing the weights from the forward's saved row statistic ("HF
 * Attention Normalizers", section "Important Limitations": softmax1 saves
 * row max / denominator statistics and recomputes probabilities during the
 * fused backward; the sparse kernels save one threshold per query row and
 * recompute tiles during the fused backward).  Per row, the normalizer's
 * Jacobian: softmax / softmax1 / sinks dz = p (g - sum p g); sparsemax
 * dz = s (g - mean over the support of g), s = 1[p > 0]; 1.5-entmax
 * dz = s (g - sum s g / sum s), s = sqrt(p); g = grad_out V^T.
 *
 * Dense mode only.  Layouts as in the forward:
 *   q, k, v      bf16 [B,Hq,Tq,d], [B,Hkv,Tk,d], [B,Hkv,Tk,dv]: the forward's
 *                inputs
 *   out          bf16 [B,Hq,Tq,dv]: the forward's output
 *   grad_out     bf16 [B,Hq,Tq,dv]: dL/dO
 *   row_stat     float32 [B,Hq,Tq]: the forward's row_stat (log-sum-exp or
 *                tau) for the same arguments
 *   grad_q, grad_k, grad_v  bf16, shaped like q, k, v (outputs; grad_k and
 *                grad_v sum over the query heads of each group)
 * The mask, soft-cap, scale, normalizer and sinks must be the forward's.
 * Supported: d == dv in {64, 128}; anything else NATTN_EUNSUPPORTED.  The
 * caller passes scratch of nattn_bwd_workspace_size(a) bytes (one float per
 * query row).  Asynchronous on `stream`; allocates nothing.  Returns NATTN_OK
 * or a negative error code.
 */
typedef struct nattn_bwd_args {
  const void* q;
  const void* k;
  const void* v;
  const void* out;
  const void* grad_out;
  const float* row_stat;
  void* grad_q;
  void* grad_k;
  void* grad_v;
  int B, Hq, Hkv, Tq, Tk, d, dv;
  float scale;
  int normalizer;
  int causal;
  int window;
  float softcap;
  const float* sinks;       /* as in nattn_args (NATTN_SOFTMAX only)         */
  void* workspace;
  size_t workspace_bytes;
  void* stream;             /* cudaStream_t */
  const uint8_t* block_mask;/* as in nattn_args                             */
} nattn_bwd_args;

int nattn_bwd(const nattn_bwd_args* a);

/* Bytes of device scratch nattn_bwd needs (pointers are not read); 0 for an
 * invalid or unsupported argument block. */
size_t nattn_bwd_workspace_size(const nattn_bwd_args* a);

/* Synchronises `stream`, returns the device status word of the current device
 * (NATTN_OK, NATTN_ETIMEOUT or NATTN_EBOUNDS; the first error recorded since
 * the last call wins) and clears it.  NATTN_ECUDA if the sync itself fails. */
int nattn_get_device_status(void* stream);

/* Static description of an error code. */
const char* nattn_strerror(int code);

/*
 * Paged decode that allocates nothing (no paper counterpart; a deployment
 * convenience of this library).
 *
 * Some callers cannot allocate device memory at the point where they run
 * attention: a serving loop whose memory is owned by another allocator, a
 * plugin that is handed pointers but no allocator, or a latency-critical
 * decode step that must not risk the implicit synchronisation of
 * cudaMalloc.  This entry point takes the same argument block as
 * nattn_fwd_ex in paged mode but ignores `workspace`: its split-KV partial
 * results live in a fixed device array inside the library, of
 * NATTN_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the library
 * holds until the process exits.
 *
 *   - Supported: paged mode, NATTN_SOFTMAX or NATTN_SOFTMAX1, d == dv in
 *     {64, 128, 256}, page_size 32 or 64, (Hq / Hkv) * Tq <= 16.  Anything
 *     else returns NATTN_EUNSUPPORTED.
 *   - The split count is chosen so the partials fit the array.  With
 *     rows = B * Hq * Tq, one split needs
 *         up256(rows * dv * 4) + up256(rows * 8)
 *     bytes, where up256 rounds up to a multiple of 256; a batch for which
 *     that exceeds NATTN_NOALLOC_SCRATCH_BYTES returns NATTN_ETOOLARGE and
 *     launches nothing.  Fewer splits than nattn_fwd_ex would use means
 *     longer runs of pages per CTA: same result, less parallelism.
 *   - The first call on a device looks up that device's address of the
 *     array (cudaGetSymbolAddress, with the device current) and keeps it
 *     with the id of the device's current context; a call that finds a
 *     different context current (after cudaDeviceReset, say) looks it up
 *     again.  Make the first call, and the first after such a change,
 *     outside any stream capture.
 *   - Every call shares the one array and leaves its contents behind.  The
 *     kernels overwrite every partial they later read, so nothing has to
 *     start at zero, but calls that overlap on the GPU (other streams, other
 *     host threads) race on the array: order them on one stream.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 * Returns NATTN_OK or a negative error code; asynchronous on a->stream.
 */
#define NATTN_NOALLOC_SCRATCH_BYTES (8u << 20)
int nattn_decode_noalloc(const nattn_args* a);

/*
 * Self-test of the bounded-wait failure path (no paper counterpart; a test
 * hook of this library).
 *
 * Every wait of the kernels above on an mbarrier phase is bounded: after
 * about two seconds it records NATTN_ETIMEOUT in the device status word, lets
 * the other roles of its CTA stop, and returns, so the CUDA context stays
 * usable.  This entry point launches one CTA whose thread waits, with that
 * same bounded wait, on an mbarrier that nothing ever completes, and so
 * exercises the path without faulting, trapping or hanging the GPU.
 *
 * Asynchronous on `stream` (NULL: the default stream); the kernel runs for
 * about two seconds.  Returns NATTN_OK if the launch succeeded, else
 * NATTN_ECUDA.  Afterwards nattn_get_device_status(stream) returns
 * NATTN_ETIMEOUT (and clears it).
 */
int nattn_selftest_wait_timeout(void* stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int nattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NATTN_H */
