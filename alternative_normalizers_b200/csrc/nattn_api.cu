// libnattn host side: argument validation, scratch layout, TMA descriptors and
// kernel dispatch behind the C ABI declared in include/nattn.h.
//
// Dispatch (no fallback between backends; each request has one path):
//   dense weights requested              -> row-wise kernel
//   paged KV, supported shape            -> split-KV decode kernels
//   dense, head dims 64/128/256 (d == dv)-> tcgen05 prefill kernels
//   anything else that validates         -> row-wise kernel
#include <math.h>
#include <mutex>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "backward.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_pair.cuh"
#include "prefill_tc.cuh"
#include "prefill_wide.cuh"
#include "problem.cuh"
#include "rowwise.cuh"

using namespace nattn;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kRowSmemCap = 48 * 1024;  // scores kept in shared memory per row
constexpr long long kMaxWeights = 1ll << 26;

// ---------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point (no -lcuda needed)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 tensor viewed as [outer][rows][inner] with a (64 x box_rows) box and
// the 128-byte swizzle.  Rows past `rows` read as zero.
bool make_map_3d(CUtensorMap* m, const void* base, int inner, int rows, long long outer,
                 int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * 2 * rows};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor in the packed layout [rows][planes][inner] (token-major) with a
// (64 x 1 x box_rows) box: box_rows rows of one plane, 128-byte swizzle.
bool make_map_packed(CUtensorMap* m, const void* base, int inner, int planes, long long rows,
                     int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)planes, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * 2 * planes};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap* m, const void* base, int inner, long long rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Driver entry points looked up by name through the runtime (no -lcuda).
template <class F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<F>(p);
  return nullptr;
}

typedef CUresult (*AddrRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
typedef CUresult (*CtxCurrentFn)(CUcontext*);
typedef CUresult (*CtxIdFn)(CUcontext, unsigned long long*);

// Bytes from `p` to the end of the device allocation that contains it, or 0
// when `p` is not inside a device allocation of this process.
size_t bytes_to_alloc_end(const void* p) {
  static AddrRangeFn fn = driver_fn<AddrRangeFn>("cuMemGetAddressRange");
  if (!fn) return 0;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return 0;
  const CUdeviceptr at = reinterpret_cast<CUdeviceptr>(p);
  return (at >= base && at < base + size) ? (size_t)(base + size - at) : 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Streaming multiprocessors of the current device.
int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 148;
  return n;
}

// Per-device one-time kernel attribute set-up (dynamic shared memory opt-in).
template <class K>
cudaError_t allow_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// ---------------------------------------------------------------------------
// Path selection and scratch sizing
// ---------------------------------------------------------------------------
enum Path { PATH_NONE, PATH_ROWWISE, PATH_TC, PATH_DECODE };

struct Plan {
  Path path = PATH_NONE;
  bool sparse = false;
  // decode
  int R = 0, nsplit = 0, pps = 0;
  // scratch offsets (bytes)
  size_t off_tau = 0, off_ovfc = 0, off_ovfr = 0, off_slots = 0;
  size_t off_supc = 0, off_supl = 0, off_rlb = 0, off_wide = 0;
  int sup_cap = 0;
  size_t off_opart = 0, off_ml = 0, off_scores = 0, off_pmask = 0;
  int pm_words = 0;
  size_t total = 0;
  int row_grid = 0, row_cap = 0;
  bool row_slots = false;
};

bool is_paged(const nattn_args* a) { return a->block_table != nullptr; }
bool is_packed(const nattn_args* a) { return a->cu_seqlens_q != nullptr; }

// Query rows of the problem: B * Hq * Tq, or total_q * Hq when packed.
long long num_rows(const nattn_args* a) {
  return is_packed(a) ? (long long)a->total_q * a->Hq : (long long)a->B * a->Hq * a->Tq;
}

// 128-row query tiles of the single-head tensor-core kernels' grid.
long long ntiles_tc(const nattn_args* a) {
  return (long long)a->B * a->Hq * ((a->Tq + TC_BM - 1) / TC_BM);
}

int validate(const nattn_args* a) {
  if (a == nullptr) return NATTN_EINVAL;
  if (a->B < 0 || a->Hq < 0 || a->Tq < 0 || a->Tk < 0) return NATTN_EINVAL;
  if (a->B == 0 || a->Hq == 0 || a->Tq == 0) return NATTN_OK;  // nothing to compute
  if (a->Hkv < 1 || a->Hq % a->Hkv != 0) return NATTN_EINVAL;
  if (a->d < 8 || a->d > 256 || a->d % 8 || a->dv < 8 || a->dv > 256 || a->dv % 8)
    return NATTN_EUNSUPPORTED;
  if (!(a->scale == a->scale) || isinf(a->scale)) return NATTN_EINVAL;
  if (!(a->softcap >= 0.f) || isinf(a->softcap)) return NATTN_EINVAL;
  if (a->window < 0) return NATTN_EINVAL;
  if (a->normalizer < 0 || a->normalizer > 3) return NATTN_EINVAL;
  if (a->causal != 0 && a->causal != 1) return NATTN_EINVAL;
  if (!a->q || !a->k || !a->v || !a->out) return NATTN_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out))
    return NATTN_EALIGN;
  if ((a->row_stat && (reinterpret_cast<uintptr_t>(a->row_stat) & 3)) ||
      (a->weights && (reinterpret_cast<uintptr_t>(a->weights) & 3)) ||
      (a->row_nnz && (reinterpret_cast<uintptr_t>(a->row_nnz) & 3)) ||
      (a->sinks && (reinterpret_cast<uintptr_t>(a->sinks) & 3)))
    return NATTN_EALIGN;
  if (a->sinks && a->normalizer != NATTN_SOFTMAX) return NATTN_EUNSUPPORTED;
  if (is_packed(a)) {
    if (!a->cu_seqlens_k || a->total_q < 1 || a->total_k < 1 || a->Tk < 1) return NATTN_EINVAL;
    if (is_paged(a)) return NATTN_EINVAL;
    if (a->weights || a->block_mask) return NATTN_EUNSUPPORTED;
    if ((long long)a->total_k * a->Hkv >= (1ll << 31)) return NATTN_ETOOLARGE;
  } else if (a->cu_seqlens_k) {
    return NATTN_EINVAL;
  }
  const long long rows = num_rows(a);
  if (rows >= (1ll << 31) || rows * (long long)(a->d > a->dv ? a->d : a->dv) >= (1ll << 40))
    return NATTN_ETOOLARGE;
  if (is_paged(a)) {
    if (!a->seqlens || a->page_size < 1 || a->block_table_stride < 1 || a->num_pages < 1 ||
        a->Tk < 1)
      return NATTN_EINVAL;
    if (a->weights || a->block_mask) return NATTN_EUNSUPPORTED;
    if ((long long)a->num_pages * a->Hkv * a->page_size >= (1ll << 31))
      return NATTN_ETOOLARGE;
  } else if (!is_packed(a)) {
    if ((long long)a->B * a->Hkv * a->Tk >= (1ll << 31)) return NATTN_ETOOLARGE;
    if (a->weights && rows * (long long)a->Tk > kMaxWeights) return NATTN_ETOOLARGE;
  }
  return NATTN_OK;
}

// Pages per decode split: 32 pages (2048 keys at 64-token pages) give every
// CTA a long run of pages to stream while the (sequence, kv head, split) grid
// of the decode workload still fills the three to five CTAs each SM holds
// many times over.
constexpr int kDecodePagesPerSplit = 32;

Plan make_plan(const nattn_args* a) {
  Plan pl;
  const bool sparse = a->normalizer == NATTN_SPARSEMAX || a->normalizer == NATTN_ENTMAX15;
  pl.sparse = sparse;
  const size_t rows = (size_t)num_rows(a);
  const int group = a->Hq / a->Hkv;
  const bool tc_dims = a->d == a->dv && (a->d == 64 || a->d == 128 || a->d == 256);
  const bool ps_ok = a->page_size == 32 || a->page_size == 64;
  if (is_paged(a)) {
    if (tc_dims && ps_ok && group * a->Tq <= 16) {
      pl.path = PATH_DECODE;
      pl.R = group * a->Tq;
      const int maxp = (a->Tk + a->page_size - 1) / a->page_size;
      pl.pps = kDecodePagesPerSplit;
      if (pl.pps > maxp) pl.pps = maxp;
      pl.nsplit = (maxp + pl.pps - 1) / pl.pps;
      const size_t parts = (size_t)a->B * a->Hkv * pl.nsplit * pl.R;
      size_t off = 0;
      pl.off_opart = off;
      off = up256(off + parts * a->dv * 4);
      pl.off_ml = off;
      off = up256(off + parts * 2 * 4);
      if (sparse) {
        pl.off_scores = off;
        off = up256(off + rows * (size_t)a->Tk * 4);
        pl.off_tau = off;
        off = up256(off + rows * 4);
        pl.pm_words = (maxp + 31) / 32;
        pl.off_pmask = off;
        off = up256(off + rows * (size_t)pl.pm_words * 4);
      }
      pl.total = off;
      return pl;
    }
  }
  // dense, packed, and paged chunks too big for the decode kernels: tcgen05
  if (!a->weights && tc_dims && a->Tk >= 1 && (!is_paged(a) || ps_ok)) {
    pl.path = PATH_TC;
    if (sparse) {
      size_t off = 0;
      pl.off_tau = off;
      off = up256(off + rows * 4);
      pl.off_ovfc = off;
      off = up256(off + 4);
      pl.off_ovfr = off;
      off = up256(off + rows * 4);
      pl.sup_cap = (a->d >= 256) ? TauCap<256>::value : TauCap<128>::value;
      pl.off_supc = off;  // one count per row half
      off = up256(off + rows * 2 * 4);
      pl.off_rlb = off;
      off = up256(off + rows * 4);
      // wide-kernel tile list: its count, then one entry per tile
      pl.off_wide = off;
      off = up256(off + 4 + (size_t)ntiles_tc(a) * 4);
      pl.off_supl = off;
      off = up256(off + rows * (size_t)pl.sup_cap * 8);
      pl.row_grid = 2 * 148;
      pl.row_cap = a->Tk < kRowSmemCap ? (a->Tk < 256 ? 256 : a->Tk) : kRowSmemCap;
      if (a->Tk > kRowSmemCap) {
        pl.row_slots = true;
        pl.off_slots = off;
        off = up256(off + (size_t)pl.row_grid * a->Tk * 4);
      }
      pl.total = off;
    }
    return pl;
  }
  // row-wise
  pl.path = PATH_ROWWISE;
  pl.row_grid = (int)(rows < 148 * 16 ? rows : 148 * 16);
  if (pl.row_grid < 1) pl.row_grid = 1;
  const int tk = a->Tk;
  pl.row_cap = tk < kRowSmemCap ? (tk < 256 ? 256 : tk) : kRowSmemCap;
  if (tk > kRowSmemCap) {
    pl.row_slots = true;
    pl.off_slots = 0;
    pl.total = up256((size_t)pl.row_grid * tk * 4);
  }
  return pl;
}

Problem to_problem(const nattn_args* a) {
  Problem P;
  P.q = static_cast<const bf16*>(a->q);
  P.k = static_cast<const bf16*>(a->k);
  P.v = static_cast<const bf16*>(a->v);
  P.out = static_cast<bf16*>(a->out);
  P.row_stat = a->row_stat;
  P.weights = a->weights;
  P.row_nnz = a->row_nnz;
  P.B = a->B;
  P.Hq = a->Hq;
  P.Hkv = a->Hkv;
  P.Tq = a->Tq;
  P.Tk = a->Tk;
  P.d = a->d;
  P.dv = a->dv;
  P.scale = a->scale;
  P.norm = a->normalizer;
  P.causal = a->causal;
  P.window = a->window;
  P.softcap = a->softcap;
  P.sinks = a->sinks;
  P.block_mask = a->block_mask;
  P.bm_nq = (a->Tq + 127) / 128;
  P.bm_nk = (a->Tk + 127) / 128;
  P.block_table = a->block_table;
  P.seqlens = a->seqlens;
  P.page_size = a->page_size;
  P.bt_stride = a->block_table_stride;
  P.num_pages = a->num_pages;
  P.cu_q = a->cu_seqlens_q;
  P.cu_k = a->cu_seqlens_k;
  P.total_q = a->total_q;
  P.total_k = a->total_k;
  return P;
}

int check_launch() {
  return cudaGetLastError() == cudaSuccess ? NATTN_OK : NATTN_ECUDA;
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
int launch_rowwise(const Problem& P, const Plan& pl, const int* row_list,
                   const int* row_count, int nrows, float* slots, int grid,
                   cudaStream_t st) {
  const int bytes = (256 + 64 + ROW_WARPS * 256 + pl.row_cap) * 4;
  if (allow_smem(rowwise_kernel, bytes) != cudaSuccess) return NATTN_ECUDA;
  rowwise_kernel<<<grid, ROW_THREADS, bytes, st>>>(P, row_list, row_count, nrows,
                                                   pl.row_cap, slots);
  return check_launch();
}

template <int D>
int launch_tc(const nattn_args* a, const Problem& P, const Plan& pl, uint8_t* ws,
              cudaStream_t st) {
  constexpr int BN = (D == 256) ? 64 : 128;
  constexpr int KST = 2, VST = 2;
  CUtensorMap mq, mk, mv;
  bool maps;
  if (is_packed(a)) {
    maps = make_map_packed(&mq, a->q, D, a->Hq, a->total_q, TC_BM) &&
           make_map_packed(&mk, a->k, D, a->Hkv, a->total_k, BN) &&
           make_map_packed(&mv, a->v, D, a->Hkv, a->total_k, BN);
  } else {
    maps = make_map_3d(&mq, a->q, D, a->Tq, (long long)a->B * a->Hq, TC_BM);
    if (is_paged(a)) {  // the pool as rows, one box per page
      const long long prow = (long long)a->num_pages * a->Hkv * a->page_size;
      maps = maps && make_map_2d(&mk, a->k, D, prow, a->page_size) &&
             make_map_2d(&mv, a->v, D, prow, a->page_size);
    } else {
      maps = maps && make_map_3d(&mk, a->k, D, a->Tk, (long long)a->B * a->Hkv, BN) &&
             make_map_3d(&mv, a->v, D, a->Tk, (long long)a->B * a->Hkv, BN);
    }
  }
  if (!maps) return NATTN_ECUDA;
  TcArgs A;
  A.P = P;
  const float log2e = 1.4426950408889634f;
  const int ntq = (a->Tq + TC_BM - 1) / TC_BM;
  const unsigned grid = (unsigned)((long long)a->B * a->Hq * ntq);
  if (!pl.sparse) {
    A.zscale = a->scale * log2e;
    A.capscale = a->softcap * log2e;
    A.tau = nullptr;
    A.ovf_rows = nullptr;
    A.ovf_count = nullptr;
    A.sup_count = nullptr;
    A.sup_list = nullptr;
    A.sup_cap = 0;
    A.rlb = nullptr;
    A.wide_tiles = A.wide_count = nullptr;
    // two query heads of one KV group per CTA, each with its own S and O
    if constexpr (D <= 128) {
      if ((a->Hq / a->Hkv) % 2 == 0) {
        using PL = PairLayout<D, KST, VST>;
        const bool cap = a->softcap > 0.f || !(A.zscale > 0.f);
        const bool bm = a->block_mask != nullptr;  // dense mode only
        decltype(&prefill_pair_kernel<D, KST, VST, true, true, PAIR_DENSE>) kp;
        if (is_packed(a))
          kp = cap ? prefill_pair_kernel<D, KST, VST, true, false, PAIR_PACKED>
                   : prefill_pair_kernel<D, KST, VST, false, false, PAIR_PACKED>;
        else if (is_paged(a))
          kp = cap ? prefill_pair_kernel<D, KST, VST, true, false, PAIR_PAGED>
                   : prefill_pair_kernel<D, KST, VST, false, false, PAIR_PAGED>;
        else
          kp = cap ? (bm ? prefill_pair_kernel<D, KST, VST, true, true, PAIR_DENSE>
                         : prefill_pair_kernel<D, KST, VST, true, false, PAIR_DENSE>)
                   : (bm ? prefill_pair_kernel<D, KST, VST, false, true, PAIR_DENSE>
                         : prefill_pair_kernel<D, KST, VST, false, false, PAIR_DENSE>);
        // persistent: one CTA per SM (shared memory and TMEM allow one), each
        // walking its share of the tiles
        const long long ntiles = (long long)a->B * (a->Hq / 2) * ntq;
        const unsigned pgrid = (unsigned)(ntiles < num_sms() ? ntiles : num_sms());
        if (allow_smem(kp, PL::ALLOC) != cudaSuccess) return NATTN_ECUDA;
        kp<<<pgrid, PAIR_THREADS, PL::ALLOC, st>>>(mq, mk, mv, A);
        return check_launch();
      }
    }
    // each S row split between two warps: two O halves where TMEM holds
    // them, else one O the halves share (d = 256)
    constexpr int NH = 2;
    using LY = TcLayout<D, D, BN, KST, VST, TC_ONLINE, NH>;
    auto k = prefill_tc_kernel<D, D, BN, KST, VST, TC_ONLINE, NH>;
    if (allow_smem(k, LY::ALLOC) != cudaSuccess) return NATTN_ECUDA;
    k<<<grid, LY::THREADS, LY::ALLOC, st>>>(mq, mk, mv, A);
    return check_launch();
  }
  const float us = (a->normalizer == NATTN_ENTMAX15) ? 0.5f : 1.0f;
  A.zscale = a->scale * us;
  A.capscale = a->softcap * us;
  A.tau = reinterpret_cast<float*>(ws + pl.off_tau);
  A.ovf_count = reinterpret_cast<int*>(ws + pl.off_ovfc);
  A.ovf_rows = reinterpret_cast<int*>(ws + pl.off_ovfr);
  A.sup_count = reinterpret_cast<int*>(ws + pl.off_supc);
  A.sup_list = reinterpret_cast<int2*>(ws + pl.off_supl);
  A.rlb = reinterpret_cast<float*>(ws + pl.off_rlb);
  A.wide_count = reinterpret_cast<int*>(ws + pl.off_wide);
  A.wide_tiles = A.wide_count + 1;
  A.sup_cap = pl.sup_cap;
  if (cudaMemsetAsync(A.ovf_count, 0, sizeof(int), st) != cudaSuccess) return NATTN_ECUDA;
  if (cudaMemsetAsync(A.wide_count, 0, sizeof(int), st) != cudaSuccess) return NATTN_ECUDA;
  // d <= 128: each S row split between two warps (eight normalizer warps
  // hide each other's latency); d = 256 keeps whole rows (64-key blocks
  // leave 32 columns per half)
  constexpr int NHT = (D <= 128) ? 2 : 1;
  using LY = TcLayout<D, D, BN, 2, 1, TC_TAU, NHT>;
  static_assert(LY::CAP == TauCap<(D >= 256 ? 256 : 128)>::value, "workspace plan capacity");
  // candidate counts start at zero: the apply kernel reads every row, and
  // rows that no sequence owns (packed padding, a sequence rejected on the
  // device) are never written by the threshold pass
  if (cudaMemsetAsync(A.sup_count, 0, (size_t)num_rows(a) * NHT * sizeof(int), st) !=
      cudaSuccess)
    return NATTN_ECUDA;
  {
    auto k = prefill_tc_kernel<D, D, BN, 2, 1, TC_TAU, NHT>;
    if (allow_smem(k, LY::ALLOC) != cudaSuccess) return NATTN_ECUDA;
    k<<<grid, LY::THREADS, LY::ALLOC, st>>>(mq, mk, mv, A);
    if (check_launch() != NATTN_OK) return NATTN_ECUDA;
  }
  {
    // phase 2: exact threshold and fp32 gather; sparsemax's short supports
    // are bound by the dependent steps (two rows per warp), 1.5-entmax's by
    // the value-row loads in flight (one row per warp)
    const size_t rows = (size_t)num_rows(a);
    if (a->normalizer == NATTN_SPARSEMAX) {
      const unsigned g2 = (unsigned)((rows + 2 * APPLY_WARPS - 1) / (2 * APPLY_WARPS));
      sparse_apply_kernel<D, NHT, LY::CAPR, 2><<<g2, APPLY_WARPS * 32, 0, st>>>(
          P, A.sup_count, A.sup_list, A.tau, A.rlb);
    } else {
      const unsigned g2 = (unsigned)((rows + APPLY_WARPS - 1) / APPLY_WARPS);
      sparse_apply_kernel<D, NHT, LY::CAPR, 1><<<g2, APPLY_WARPS * 32, 0, st>>>(
          P, A.sup_count, A.sup_list, A.tau, A.rlb);
    }
    if (check_launch() != NATTN_OK) return NATTN_ECUDA;
  }
  {
    // tiles with rows whose candidates overflowed: Newton passes over their
    // full score rows and a tensor-core weight pass (one CTA per SM walks
    // the listed tiles; with none listed every CTA exits at once)
    constexpr int NHW = (2 * BN + 2 * D <= 512) ? 2 : 1;
    static_assert(NHW == NHT, "the wide kernel reads the threshold pass's row halves");
    using WL = WideLayout<D, BN, NHW>;
    auto kw = prefill_wide_kernel<D, BN, NHW>;
    if (allow_smem(kw, WL::ALLOC) != cudaSuccess) return NATTN_ECUDA;
    const unsigned wgrid = grid < (unsigned)num_sms() ? grid : (unsigned)num_sms();
    kw<<<wgrid, WL::THREADS, WL::ALLOC, st>>>(mq, mk, mv, A);
    if (check_launch() != NATTN_OK) return NATTN_ECUDA;
  }
  // rows the wide kernel left unsolved: exact row-wise recomputation
  float* slots = pl.row_slots ? reinterpret_cast<float*>(ws + pl.off_slots) : nullptr;
  return launch_rowwise(P, pl, A.ovf_rows, A.ovf_count, 0, slots, pl.row_grid, st);
}

template <int D, int PS, int MODE>
int launch_decode_mode(const nattn_args* a, const DecodeArgs& A, const CUtensorMap& mk,
                       const CUtensorMap& mv, cudaStream_t st) {
  // two stages (one page computing, the next loading): a CTA's time per page
  // is mostly its own barrier and product latency, so more CTAs per SM (three
  // for K+V pages of d = 128, five for K or V alone) move more bytes than
  // deeper rings do; with four stages the same passes ran 24-32 % slower
  constexpr int NS = 2;
  using L = DecodeSmem<D, D, PS, NS, MODE>;
  // only the sparse apply pass keeps a page list (two ints per page)
  const int bytes = L::BYTES_NOLIST + (MODE == DEC_APPLY ? 2 * A.pps * 4 : 0) + 1024;
  dim3 grid(A.nsplit, a->Hkv, a->B);
  if (A.R <= 8) {
    auto k = decode_split_kernel<D, D, PS, NS, 1, MODE>;
    if (allow_smem(k, bytes) != cudaSuccess) return NATTN_ECUDA;
    k<<<grid, DEC_THREADS, bytes, st>>>(mk, mv, A);
  } else {
    auto k = decode_split_kernel<D, D, PS, NS, 2, MODE>;
    if (allow_smem(k, bytes) != cudaSuccess) return NATTN_ECUDA;
    k<<<grid, DEC_THREADS, bytes, st>>>(mk, mv, A);
  }
  return check_launch();
}

template <int D, int PS>
int launch_decode(const nattn_args* a, const Problem& P, const Plan& pl, uint8_t* ws,
                  cudaStream_t st) {
  CUtensorMap mk, mv;
  const long long prow = (long long)a->num_pages * a->Hkv * PS;
  if (!make_map_2d(&mk, a->k, D, prow, PS) || !make_map_2d(&mv, a->v, D, prow, PS))
    return NATTN_ECUDA;
  DecodeArgs A;
  A.P = P;
  A.R = pl.R;
  A.nsplit = pl.nsplit;
  A.pps = pl.pps;
  A.opart = reinterpret_cast<float*>(ws + pl.off_opart);
  A.ml = reinterpret_cast<float*>(ws + pl.off_ml);
  A.scores = pl.sparse ? reinterpret_cast<float*>(ws + pl.off_scores) : nullptr;
  A.tau = pl.sparse ? reinterpret_cast<float*>(ws + pl.off_tau) : nullptr;
  A.pmask = pl.sparse ? reinterpret_cast<unsigned*>(ws + pl.off_pmask) : nullptr;
  A.pm_words = pl.sparse ? pl.pm_words : 0;
  const unsigned rows = (unsigned)((size_t)a->B * a->Hq * a->Tq);
  if (!pl.sparse) {
    A.zscale = a->scale * 1.4426950408889634f;
    A.uscale = 1.f;
    int rc = launch_decode_mode<D, PS, DEC_ONLINE>(a, A, mk, mv, st);
    if (rc) return rc;
    decode_combine_kernel<<<rows, 128, 0, st>>>(A, DEC_ONLINE);
    return check_launch();
  }
  A.uscale = (a->normalizer == NATTN_ENTMAX15) ? 0.5f : 1.0f;
  A.zscale = a->scale * A.uscale;
  int rc = launch_decode_mode<D, PS, DEC_SCORES>(a, A, mk, mv, st);
  if (rc) return rc;
  const int cap = 4096;  // candidates kept in shared memory (value + key index)
  const int tbytes = (64 + 2 * cap + pl.pm_words) * 4;
  if (allow_smem(decode_tau_kernel, tbytes) != cudaSuccess) return NATTN_ECUDA;
  decode_tau_kernel<<<rows, TAU_THREADS, tbytes, st>>>(A, const_cast<float*>(A.tau), cap);
  if (check_launch()) return NATTN_ECUDA;
  rc = launch_decode_mode<D, PS, DEC_APPLY>(a, A, mk, mv, st);
  if (rc) return rc;
  decode_combine_kernel<<<rows, 128, 0, st>>>(A, DEC_APPLY);
  return check_launch();
}

int run(const nattn_args* a) {
  int rc = validate(a);
  if (rc != NATTN_OK) return rc;
  if (a->B == 0 || a->Hq == 0 || a->Tq == 0) return NATTN_OK;
  const Plan pl = make_plan(a);
  if (pl.total > 0 && (a->workspace == nullptr || a->workspace_bytes < pl.total))
    return NATTN_EWORKSPACE;
  if (a->workspace && !aligned16(a->workspace)) return NATTN_EALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(a->stream);
  const Problem P = to_problem(a);
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  switch (pl.path) {
    case PATH_TC:
      if (a->d == 64) return launch_tc<64>(a, P, pl, ws, st);
      if (a->d == 128) return launch_tc<128>(a, P, pl, ws, st);
      return launch_tc<256>(a, P, pl, ws, st);
    case PATH_DECODE:
      if (a->page_size == 32) {
        if (a->d == 64) return launch_decode<64, 32>(a, P, pl, ws, st);
        if (a->d == 128) return launch_decode<128, 32>(a, P, pl, ws, st);
        return launch_decode<256, 32>(a, P, pl, ws, st);
      }
      if (a->d == 64) return launch_decode<64, 64>(a, P, pl, ws, st);
      if (a->d == 128) return launch_decode<128, 64>(a, P, pl, ws, st);
      return launch_decode<256, 64>(a, P, pl, ws, st);
    case PATH_ROWWISE: {
      const int nrows = (int)num_rows(a);
      float* slots = pl.row_slots ? reinterpret_cast<float*>(ws + pl.off_slots) : nullptr;
      return launch_rowwise(P, pl, nullptr, nullptr, nrows, slots, pl.row_grid, st);
    }
    default:
      return NATTN_EUNSUPPORTED;
  }
}


// ---------------------------------------------------------------------------
// Allocation-free paged decode: split partials in a fixed device array
// ---------------------------------------------------------------------------
// The array is this file's own; host code only ever sees a stand-in for its
// name, so the device address is looked up once per device and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kNoAllocDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocDevices] = {};
unsigned long long g_noalloc_ctx[kNoAllocDevices] = {};  // context id of the lookup

// Device address of the scratch array on the current device.  The first call
// per device does the lookup with that device current; the address is kept
// with the id of the context it belongs to and looked up again whenever the
// device's current context is a different one (after cudaDeviceReset, for
// instance, the module is loaded anew and the array may move).
int noalloc_scratch(void** out) {
  static CtxCurrentFn ctx_current = driver_fn<CtxCurrentFn>("cuCtxGetCurrent");
  static CtxIdFn ctx_id = driver_fn<CtxIdFn>("cuCtxGetId");
  if (!ctx_current || !ctx_id) return NATTN_ECUDA;
  auto current_id = [&](unsigned long long* id) {
    CUcontext ctx = nullptr;
    return ctx_current(&ctx) == CUDA_SUCCESS && ctx != nullptr &&
           ctx_id(ctx, id) == CUDA_SUCCESS;
  };
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocDevices)
    return NATTN_ECUDA;
  unsigned long long id = 0;
  // false before the runtime has bound its context to this thread; the
  // symbol lookup below does that
  const bool have_id = current_id(&id);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!have_id || g_noalloc_addr[dev] == nullptr || g_noalloc_ctx[dev] != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return NATTN_ECUDA;
    if (!have_id && !current_id(&id)) return NATTN_ECUDA;
    g_noalloc_addr[dev] = p;
    g_noalloc_ctx[dev] = id;
  }
  *out = g_noalloc_addr[dev];
  return NATTN_OK;
}

int decode_noalloc(const nattn_args* a) {
  int rc = validate(a);
  if (rc != NATTN_OK) return rc;
  if (a->B == 0 || a->Hq == 0 || a->Tq == 0) return NATTN_OK;
  if (!is_paged(a)) return NATTN_EUNSUPPORTED;
  if (a->normalizer != NATTN_SOFTMAX && a->normalizer != NATTN_SOFTMAX1)
    return NATTN_EUNSUPPORTED;
  Plan pl = make_plan(a);
  if (pl.path != PATH_DECODE) return NATTN_EUNSUPPORTED;
  // choose the split count so that the partials fit the array
  const size_t rows_per_split = (size_t)a->B * a->Hkv * pl.R;
  const size_t per_split = up256(rows_per_split * a->dv * 4) + up256(rows_per_split * 2 * 4);
  const int fit = (int)(NATTN_NOALLOC_SCRATCH_BYTES / per_split);
  if (fit < 1) return NATTN_ETOOLARGE;
  const int maxp = (a->Tk + a->page_size - 1) / a->page_size;
  if (pl.nsplit > fit) {
    pl.pps = (maxp + fit - 1) / fit;
    pl.nsplit = (maxp + pl.pps - 1) / pl.pps;
  }
  const size_t parts = rows_per_split * pl.nsplit;
  pl.off_opart = 0;
  pl.off_ml = up256(parts * a->dv * 4);
  pl.total = pl.off_ml + up256(parts * 2 * 4);
  if (pl.total > NATTN_NOALLOC_SCRATCH_BYTES) return NATTN_ETOOLARGE;
  void* base = nullptr;
  rc = noalloc_scratch(&base);
  if (rc != NATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(a->stream);
  const Problem P = to_problem(a);
  uint8_t* ws = static_cast<uint8_t*>(base);
  if (a->page_size == 32) {
    if (a->d == 64) return launch_decode<64, 32>(a, P, pl, ws, st);
    if (a->d == 128) return launch_decode<128, 32>(a, P, pl, ws, st);
    return launch_decode<256, 32>(a, P, pl, ws, st);
  }
  if (a->d == 64) return launch_decode<64, 64>(a, P, pl, ws, st);
  if (a->d == 128) return launch_decode<128, 64>(a, P, pl, ws, st);
  return launch_decode<256, 64>(a, P, pl, ws, st);
}

// ---------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------
int validate_bwd(const nattn_bwd_args* a) {
  if (a == nullptr) return NATTN_EINVAL;
  nattn_args f;
  memset(&f, 0, sizeof(f));
  f.q = a->q;
  f.k = a->k;
  f.v = a->v;
  f.out = a->grad_q;  // any non-null output pointer for the shared checks
  f.B = a->B;
  f.Hq = a->Hq;
  f.Hkv = a->Hkv;
  f.Tq = a->Tq;
  f.Tk = a->Tk;
  f.d = a->d;
  f.dv = a->dv;
  f.scale = a->scale;
  f.normalizer = a->normalizer;
  f.causal = a->causal;
  f.window = a->window;
  f.softcap = a->softcap;
  f.sinks = a->sinks;
  f.block_mask = a->block_mask;
  f.row_stat = const_cast<float*>(a->row_stat);
  int rc = validate(&f);
  if (rc != NATTN_OK) return rc;
  if (a->B == 0 || a->Hq == 0 || a->Tq == 0) return NATTN_OK;
  if (!a->out || !a->grad_out || !a->row_stat || !a->grad_q || !a->grad_k || !a->grad_v)
    return NATTN_EINVAL;
  if (!aligned16(a->out) || !aligned16(a->grad_out) || !aligned16(a->grad_q) ||
      !aligned16(a->grad_k) || !aligned16(a->grad_v))
    return NATTN_EALIGN;
  if (a->d != a->dv || (a->d != 64 && a->d != 128) || a->Tk < 1) return NATTN_EUNSUPPORTED;
  return NATTN_OK;
}

size_t bwd_workspace(const nattn_bwd_args* a) {
  return up256((size_t)a->B * a->Hq * a->Tq * 4);
}

// One backward: the per-row delta (a dot product for the softmax family,
// the dQ kernel's DELTA mode for the sparse normalizers), then the dQ kernel,
// then the dK/dV kernel; KIND 0 softmax family, 1 sparsemax, 2 1.5-entmax.
template <int D, int KIND, bool CAP>
int launch_bwd_kind(const nattn_bwd_args* a, BwdArgs& A, cudaStream_t st) {
  const long long BHq = (long long)a->B * a->Hq, BHkv = (long long)a->B * a->Hkv;
  // dQ kernel: 128-row query tiles, 64-key blocks
  CUtensorMap mq, mo, mk, mv;
  if (!make_map_3d(&mq, a->q, D, a->Tq, BHq, 128) ||
      !make_map_3d(&mo, a->grad_out, D, a->Tq, BHq, 128) ||
      !make_map_3d(&mk, a->k, D, a->Tk, BHkv, BWD_BN) ||
      !make_map_3d(&mv, a->v, D, a->Tk, BHkv, BWD_BN))
    return NATTN_ECUDA;
  const unsigned gq = (unsigned)(BHq * ((a->Tq + 127) / 128));
  using LQ = BwdQLayout<D, D>;
  if constexpr (KIND != 0) {
    auto k = bwd_dq_kernel<D, D, BWD_DELTA, KIND, CAP>;
    if (allow_smem(k, LQ::ALLOC) != cudaSuccess) return NATTN_ECUDA;
    k<<<gq, BWD_THREADS, LQ::ALLOC, st>>>(mq, mo, mk, mv, A);
  } else {
    const size_t rows = (size_t)BHq * a->Tq;
    bwd_delta_dot_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(A);
  }
  if (check_launch() != NATTN_OK) return NATTN_ECUDA;
  {
    auto k = bwd_dq_kernel<D, D, BWD_DQ, KIND, CAP>;
    if (allow_smem(k, LQ::ALLOC) != cudaSuccess) return NATTN_ECUDA;
    k<<<gq, BWD_THREADS, LQ::ALLOC, st>>>(mq, mo, mk, mv, A);
    if (check_launch() != NATTN_OK) return NATTN_ECUDA;
  }
  // dK/dV kernel: 128-key tiles, 64-row query blocks
  if (!make_map_3d(&mq, a->q, D, a->Tq, BHq, BWD_BQ) ||
      !make_map_3d(&mo, a->grad_out, D, a->Tq, BHq, BWD_BQ) ||
      !make_map_3d(&mk, a->k, D, a->Tk, BHkv, 128) ||
      !make_map_3d(&mv, a->v, D, a->Tk, BHkv, 128))
    return NATTN_ECUDA;
  using LK = BwdKVLayout<D, D>;
  auto k = bwd_dkdv_kernel<D, D, KIND, CAP>;
  if (allow_smem(k, LK::ALLOC) != cudaSuccess) return NATTN_ECUDA;
  const unsigned gk = (unsigned)(BHkv * ((a->Tk + 127) / 128));
  k<<<gk, BWD_THREADS, LK::ALLOC, st>>>(mq, mo, mk, mv, A);
  return check_launch();
}

template <int D>
int launch_bwd(const nattn_bwd_args* a, cudaStream_t st) {
  BwdArgs A;
  memset(&A, 0, sizeof(A));
  Problem& P = A.P;
  P.q = static_cast<const bf16*>(a->q);
  P.k = static_cast<const bf16*>(a->k);
  P.v = static_cast<const bf16*>(a->v);
  P.out = static_cast<bf16*>(const_cast<void*>(a->out));
  P.row_stat = const_cast<float*>(a->row_stat);
  P.B = a->B;
  P.Hq = a->Hq;
  P.Hkv = a->Hkv;
  P.Tq = a->Tq;
  P.Tk = a->Tk;
  P.d = a->d;
  P.dv = a->dv;
  P.scale = a->scale;
  P.norm = a->normalizer;
  P.causal = a->causal;
  P.window = a->window;
  P.softcap = a->softcap;
  P.sinks = a->sinks;
  P.block_mask = a->block_mask;
  P.bm_nq = (a->Tq + 127) / 128;
  P.bm_nk = (a->Tk + 127) / 128;
  A.dout = static_cast<const bf16*>(a->grad_out);
  A.dq = static_cast<bf16*>(a->grad_q);
  A.dk = static_cast<bf16*>(a->grad_k);
  A.dv = static_cast<bf16*>(a->grad_v);
  A.delta = static_cast<float*>(a->workspace);
  A.us = (a->normalizer == NATTN_ENTMAX15) ? 0.5f : 1.0f;
  const bool cap = a->softcap > 0.f;
  switch (a->normalizer) {
    case NATTN_SPARSEMAX:
      return cap ? launch_bwd_kind<D, 1, true>(a, A, st) : launch_bwd_kind<D, 1, false>(a, A, st);
    case NATTN_ENTMAX15:
      return cap ? launch_bwd_kind<D, 2, true>(a, A, st) : launch_bwd_kind<D, 2, false>(a, A, st);
    default:
      return cap ? launch_bwd_kind<D, 0, true>(a, A, st) : launch_bwd_kind<D, 0, false>(a, A, st);
  }
}

int run_bwd(const nattn_bwd_args* a) {
  int rc = validate_bwd(a);
  if (rc != NATTN_OK) return rc;
  if (a->B == 0 || a->Hq == 0 || a->Tq == 0) return NATTN_OK;
  if (a->workspace == nullptr || a->workspace_bytes < bwd_workspace(a)) return NATTN_EWORKSPACE;
  if (!aligned16(a->workspace)) return NATTN_EALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(a->stream);
  return a->d == 64 ? launch_bwd<64>(a, st) : launch_bwd<128>(a, st);
}

}  // namespace

namespace nattn {
// One bounded wait on an mbarrier phase that nothing completes: the wait
// gives up after its budget and records NATTN_ETIMEOUT (see
// nattn_selftest_wait_timeout in the header).
__global__ void selftest_wait_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, &abort_flag);
  __syncwarp();
}
}  // namespace nattn

extern "C" {

__attribute__((visibility("default"))) int nattn_fwd_ex(const nattn_args* a) { return run(a); }

__attribute__((visibility("default"))) int nattn_bwd(const nattn_bwd_args* a) {
  return run_bwd(a);
}

__attribute__((visibility("default"))) size_t nattn_bwd_workspace_size(const nattn_bwd_args* a) {
  if (validate_bwd(a) != NATTN_OK) return 0;
  if (a->B == 0 || a->Hq == 0 || a->Tq == 0) return 0;
  return bwd_workspace(a);
}

__attribute__((visibility("default"))) size_t nattn_workspace_size(const nattn_args* a) {
  if (validate(a) != NATTN_OK) return 0;
  if (a->B == 0 || a->Hq == 0 || a->Tq == 0) return 0;
  return make_plan(a).total;
}

__attribute__((visibility("default"))) int nattn_fwd(const void* q, const void* k, const void* v, void* out, float* row_stat,
              int B, int Hq, int Hkv, int Tq, int Tk, int d, int dv, float scale,
              int normalizer, int causal, int window, float softcap,
              const int32_t* block_table, const int32_t* seqlens, void* stream) {
  nattn_args a;
  memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.row_stat = row_stat;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Tq = Tq;
  a.Tk = Tk;
  a.d = d;
  a.dv = dv;
  a.scale = scale;
  a.normalizer = normalizer;
  a.causal = causal;
  a.window = window;
  a.softcap = softcap;
  a.block_table = block_table;
  a.seqlens = seqlens;
  a.stream = stream;
  if (block_table) {
    a.page_size = 64;
    a.block_table_stride = (Tk + 63) / 64;
    a.num_pages = 1;  // placeholder for the host checks below
  }
  int rc = validate(&a);
  if (rc != NATTN_OK) return rc;
  if (block_table && B > 0 && Hq > 0 && Tq > 0) {
    // The pool holds as many whole pages as the device allocations that
    // contain k and v reach past their start: page ids at or past that bound
    // are caught on the device (NATTN_EBOUNDS), so a bad table never reads
    // memory this process does not own.
    const size_t kb = bytes_to_alloc_end(k), vb = bytes_to_alloc_end(v);
    const size_t kpage = (size_t)Hkv * 64 * d * 2, vpage = (size_t)Hkv * 64 * dv * 2;
    size_t np = kb / kpage < vb / vpage ? kb / kpage : vb / vpage;
    if (np < 1) return NATTN_EINVAL;
    const size_t cap = (size_t)((1ll << 31) - 1) / ((size_t)Hkv * 64);
    a.num_pages = (int)(np < cap ? np : cap);
  }
  const size_t need = nattn_workspace_size(&a);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (need > 0) {
    if (cudaMallocAsync(&a.workspace, need, st) != cudaSuccess) return NATTN_ECUDA;
    a.workspace_bytes = need;
  }
  rc = run(&a);
  if (need > 0 && cudaFreeAsync(a.workspace, st) != cudaSuccess && rc == NATTN_OK)
    rc = NATTN_ECUDA;
  return rc;
}

__attribute__((visibility("default"))) int nattn_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return NATTN_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return NATTN_ECUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return NATTN_ECUDA;
  return v;
}

__attribute__((visibility("default"))) const char* nattn_strerror(int code) {
  switch (code) {
    case NATTN_OK: return "ok";
    case NATTN_EINVAL: return "invalid argument";
    case NATTN_EUNSUPPORTED: return "unsupported configuration";
    case NATTN_ETOOLARGE: return "problem too large for the requested output";
    case NATTN_EWORKSPACE: return "workspace missing or too small";
    case NATTN_ECUDA: return "CUDA runtime error";
    case NATTN_ETIMEOUT: return "device wait timed out";
    case NATTN_EBOUNDS: return "block table entry or sequence length out of range";
    case NATTN_EALIGN: return "pointer not 16-byte aligned";
    default: return "unknown error";
  }
}

__attribute__((visibility("default"))) int nattn_selftest_wait_timeout(void* stream) {
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return check_launch();
}

__attribute__((visibility("default"))) int nattn_version(void) { return kVersion; }

__attribute__((visibility("default"))) int nattn_decode_noalloc(const nattn_args* a) {
  return decode_noalloc(a);
}

}  // extern "C"
