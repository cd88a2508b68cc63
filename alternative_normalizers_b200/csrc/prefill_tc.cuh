// Prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA computes one 128-row query tile of one (batch, query head) against
// the key blocks its mask leaves visible; blocks entirely outside the causal
// band or the sliding window are never loaded or multiplied ("Attention
// variants", TensorCAD, section "Three ways to open it up": whole masked
// blocks are skipped, which is where the speed of causal and windowed
// attention comes from; section "What this leaves open": a kernel computes
// whole blocks, so a sliver costs a block).
//
// Warp roles (192 threads):
//   warps 0-3  normalizer warps: thread = query row = TMEM lane.  They read
//              the score tile S from TMEM, apply scale / soft-cap / mask and
//              the row normalizer, and write the bf16 weights P back into the
//              same TMEM columns (P aliases S).
//   warp 4     TMA producer: Q once, then a ring of K and a ring of V blocks.
//   warp 5     MMA issuer (one thread) and TMEM owner: S = Q K^T with both
//              operands in shared memory; O += P V with P read from TMEM.
//
// Modes:
//   ONLINE  softmax and softmax1 in one pass with a running maximum and
//           denominator.  softmax1 starts from the virtual logit-0 / value-0
//           sink ("HF Attention Normalizers", section "Important
//           Limitations": the Softmax1 denominator term is a virtual
//           logit-0/value-0 sink, and row max/denominator are saved), i.e.
//           m0 = 0, l0 = 1.  The running maximum is only moved (and O
//           rescaled) when it grows by more than 2^8, which keeps rescaling
//           off the common path.
//   TAU     sparse phase 1: S only, in two passes over the key blocks.  The
//           bound pass keeps 32 bucket maxima per thread (two three-input
//           max operations per four scores, no branches) and solves the
//           exact threshold of those distinct keys: a lower bound of the
//           row's.  The candidate pass keeps every key above that fixed
//           bound in a small buffer, and the exact threshold is solved on the
//           buffer at the end ("HF Attention Normalizers", section "Important
//           Limitations": the sparse kernels stream K/V tiles, solve the
//           global normalization threshold and save one threshold per query
//           row).  The second QK product is cheap next to per-score work on
//           the CUDA cores, which sets this mode's speed.  Rows whose
//           candidates overflow the buffer are listed for the row-wise
//           kernel.
// Sparse phase 2 is sparse_apply_kernel below: each row's exact threshold
// from its candidates, then an fp32 sum over its support.
#pragma once

#include "common.cuh"
#include "problem.cuh"

namespace nattn {

enum TcMode { TC_ONLINE = 0, TC_TAU = 1 };

constexpr int TC_THREADS = 192;
constexpr int TC_BM = 128;
// candidate buffer entries per row in the threshold pass (value + key index);
// with the bound pass's bound the candidates of a row are its support and a
// few keys more
template <int D>
struct TauCap {
  static constexpr int value = (D >= 256) ? 72 : 92;
};

struct TcArgs {
  Problem P;
  float zscale;      // ONLINE: scale * log2(e); TAU: scale * uscale
  float capscale;    // soft-cap: z = capscale * tanh(s * scale / cap)
  float* tau;        // [rows] TAU: the row maximum (threshold units)
  int* ovf_rows;     // TAU: rows whose candidate buffer overflowed
  int* ovf_count;    // TAU: number of such rows (zeroed before the launch)
  int* sup_count;    // TAU: [rows][halves] candidate counts (-1: the row overflowed)
  int2* sup_list;    // TAU: [rows][halves][sup_cap / halves] (value row of the key,
                     //      value less the row maximum in threshold units)
  float* rlb;        // TAU: [rows] lower bound of the threshold less the row maximum
  int* wide_tiles;   // TAU: tiles (ranks) with a row whose candidates overflowed
  int* wide_count;   // TAU: number of such tiles (zeroed before the launch)
  int sup_cap;
};

// Rows [row0, row0 + box) of head plane `plane` (batch * heads + head for the
// dense layout, the head for the packed one) of a Q / K / V tensor, 64
// columns from column x: dense tensor maps are [planes][rows][64-wide],
// packed ones [rows][planes][64-wide] (FlashAttention-style [total, H, d]).
__device__ __forceinline__ void tma_load_rows(uint32_t dst, const void* map, uint32_t bar, int x,
                                              int row0, int plane, bool packed) {
  if (packed)
    tma_load_3d(dst, map, bar, x, plane, row0);
  else
    tma_load_3d(dst, map, bar, x, row0, plane);
}

// Key (or value) block kb (keys [kb * BN, kb * BN + BN)) of sequence b, kv
// head g into a 128-byte-swizzled tile of DIM / 64 boxes of BN rows.  Paged
// mode: the map views the pool as rows [num_pages * Hkv * page_size][DIM]
// with one box per page; pages past the sequence's end load page 0 (their
// keys are masked), an out-of-range page id records NATTN_EBOUNDS and loads
// page 0 too ("HF Attention Normalizers", section "Differentiable Paged
// Attention": the kernel reads physical pages through the block table).
template <int DIM, int BN>
__device__ __forceinline__ void tma_load_kv(const Problem& P, const CUtensorMap* map, uint8_t* dst,
                                            uint32_t bar, int b, int g, int kb, const SeqInfo& s) {
  if (P.block_table != nullptr) {
    const int ps = P.page_size;
    for (int p = 0; p < BN / ps; ++p) {
      const int lp = (kb * BN) / ps + p;
      int page = 0;
      if (lp * ps < s.Lk) {
        page = P.block_table[(size_t)b * P.bt_stride + lp];
        if (page < 0 || page >= P.num_pages) {
          set_status(NATTN_EBOUNDS);
          page = 0;
        }
      }
#pragma unroll
      for (int x = 0; x < DIM / 64; ++x)
        tma_load_2d(smem_addr(dst + x * BN * 128 + p * ps * 128), map, bar, x * 64,
                    (page * P.Hkv + g) * ps);
    }
    return;
  }
  const bool packed = P.cu_q != nullptr;
#pragma unroll
  for (int x = 0; x < DIM / 64; ++x)
    tma_load_rows(smem_addr(dst + x * BN * 128), map, bar, x * 64,
                  packed ? s.k0 + kb * BN : kb * BN, packed ? g : b * P.Hkv + g, packed);
}

// Row of value row j of sequence b, kv head g in the V tensor viewed as rows
// of dv elements (the sparse gather's address of a support key).
__device__ __forceinline__ int value_row(const Problem& P, int b, int g, int j, const SeqInfo& s) {
  if (P.cu_q != nullptr) return (s.k0 + j) * P.Hkv + g;
  if (P.block_table != nullptr) {
    int page = P.block_table[(size_t)b * P.bt_stride + j / P.page_size];
    if (page < 0 || page >= P.num_pages) page = 0;  // recorded by the loads
    return (page * P.Hkv + g) * P.page_size + j % P.page_size;
  }
  return (b * P.Hkv + g) * P.Tk + j;
}

// NH = 2 splits every S row between two warps (columns [0, BN/2) and
// [BN/2, BN)).  In the online mode each half keeps its own running maximum,
// denominator and O accumulator in TMEM; in the threshold mode each half
// keeps its own candidate buffer and publishes its running bound for the
// other.  The halves are merged once in the epilogue.  Two normalizer warps
// per SM sub-partition hide each other's latency and each thread holds half a
// row in registers.
template <int D, int DV, int BN, int KST, int VST, int MODE, int NH = 1>
struct TcLayout {
  static constexpr int NWN = 4 * NH;                 // normalizer warps
  // Online, split rows where TMEM has no room for two O halves (d = 256:
  // 2 x 64 + 2 x 256 > 512): the halves share one O and one running maximum
  // (exchanged through shared memory every block), and each half writes its
  // 32 keys' P for the same PV product.  Two normalizer warps per SM
  // sub-partition instead of one.
  static constexpr bool SHARED_O = MODE == TC_ONLINE && NH == 2 && 2 * BN + 2 * DV > 512;
  // The threshold pass with split rows holds a 64-score chunk, the bucket
  // maxima and the candidate state per thread: it runs three whole
  // warpgroups (two idle warps) so that setmaxnreg can move registers from
  // the TMA / MMA warpgroup to the normalizer warpgroups:
  // 2 * 128 * 208 + 128 * 88 = 384 * 168, the launch's allocation (the
  // TMA producer's page walk needs more than 56).
  static constexpr bool REGSPLIT = (MODE == TC_TAU && NH == 2);
  static constexpr int REGS_NORM = 208, REGS_CTRL = 88;
  static constexpr int THREADS = REGSPLIT ? 384 : (NWN + 2) * 32;  // + TMA warp + MMA warp
  static_assert(!REGSPLIT || 2 * 128 * REGS_NORM + 128 * REGS_CTRL <= 384 * 168,
                "register split exceeds the launch's allocation");
  static constexpr int QBYTES = D * TC_BM * 2;
  static constexpr int KBYTES = D * BN * 2;
  static constexpr int VBYTES = (MODE == TC_TAU) ? 0 : DV * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + KST * KBYTES;
  static constexpr int OFF_BUF = OFF_V + VST * VBYTES;
  static constexpr int CAP = TauCap<D>::value;
  static constexpr int CAPR = CAP / NH;         // entries per row half
  static constexpr int CAP_STRIDE = CAPR + 1;    // int2 entries per row half
  // per row half: CAPR candidates (and one padding entry)
  static constexpr int BUFBYTES = (MODE == TC_TAU) ? CAP_STRIDE * TC_BM * NH * 8 : 0;
  // per normalizer thread: the 32 scores of the chunk it is appending from
  // (and, at the end of the bound pass, its 32 bucket maxima for the other
  // half of its row)
  static constexpr int STASHBYTES = (MODE == TC_TAU) ? NWN * 32 * 32 * 4 : 0;
  static constexpr int OFF_STASH = OFF_BUF + BUFBYTES;
  static constexpr int OFF_BAR = OFF_STASH + STASHBYTES;
  // S ring depth in TMEM: the threshold pass has no O accumulator, so it
  // keeps three or four S buffers (its normalizer warps can drift that many
  // blocks apart) and its Q tile: each QK product takes A (Q) from TMEM and
  // only B (K) from shared memory, which halves the product's shared-memory
  // reads (with both operands there a 128 x 128 x 16 product reads as many
  // bytes per cycle as shared memory delivers)
  static constexpr int NSB = (MODE == TC_TAU) ? (BN >= 128 ? 3 : 4) : 2;
  static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 2 * NSB + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // epilogue (m, l) exchange between row halves: reuses the Q tile, which
  // every product has finished reading once the last PV has completed
  static constexpr int OFF_XCH = OFF_Q;
  // shared O: the halves' block maxima (by block parity) and, at the end,
  // their denominators
  static constexpr int OFF_XM = OFF_MISC + 16;
  static constexpr int BYTES = OFF_XM + (SHARED_O ? 2 * 2 * TC_BM * 4 : 0);
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
  // TMEM columns: the S ring (NSB buffers of BN columns), then O (online)
  // or Q (threshold pass: bf16 pairs, D / 2 columns)
  static constexpr int TM_S = 0;  // S buffer s at column s * BN
  static constexpr int TM_O = 2 * BN;
  static constexpr int TM_Q = NSB * BN;
  static constexpr int TM_COLS_USED =
      (MODE == TC_TAU) ? NSB * BN + D / 2 : 2 * BN + (SHARED_O ? DV : NH * DV);
  static constexpr int TM_COLS = TM_COLS_USED <= 32    ? 32
                                 : TM_COLS_USED <= 64  ? 64
                                 : TM_COLS_USED <= 128 ? 128
                                 : TM_COLS_USED <= 256 ? 256
                                                       : 512;
  static_assert(TM_COLS_USED <= 512, "TMEM budget");
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
};

// Score transform for one raw dot product s.
__device__ __forceinline__ float tc_z(float s, const TcArgs& A) {
  if (A.P.softcap > 0.f) return A.capscale * fast_tanh(s * (A.P.scale / A.P.softcap));
  return s * A.zscale;
}

// The same transform for 64 raw dot products held as bits.  With a soft-cap,
// z = capscale * tanh(a s), a = scale / cap: when |a s| <= 1 for every score
// of the warp (scores within the cap, the usual case) tanh comes from the odd
// polynomial of tanh_odd_poly on the FMA pipe in packed pairs, leaving the
// MUFU pipe to the exponentials; otherwise from tanh.approx.
template <int N>
__device__ __forceinline__ void tc_zn(uint32_t* r, const TcArgs& A) {
  if (A.P.softcap > 0.f) {
    const float a = A.P.scale / A.P.softcap;
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < N; ++k) amax = fmaxf(amax, fabsf(__uint_as_float(r[k])));
    if (__all_sync(0xffffffffu, amax * fabsf(a) <= 1.f)) {
      TanhPoly c;
      tanh_odd_coeffs(A.capscale, c);
#pragma unroll
      for (int k = 0; k < N; k += 2) {
        float z0, z1;
        tanh_odd_poly2(__uint_as_float(r[k]), __uint_as_float(r[k + 1]), a, c, z0, z1);
        r[k] = __float_as_uint(z0);
        r[k + 1] = __float_as_uint(z1);
      }
    } else {
#pragma unroll
      for (int k = 0; k < N; ++k)
        r[k] = __float_as_uint(A.capscale * fast_tanh(__uint_as_float(r[k]) * a));
    }
  } else {
#pragma unroll
    for (int k = 0; k < N; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * A.zscale);
  }
}
__device__ __forceinline__ void tc_z64(uint32_t* r, const TcArgs& A) { tc_zn<64>(r, A); }

// Named barrier `id` over `nthreads` threads that also ANDs a flag across
// them: every participant leaves with the same answer (used where a thread
// that gave up a wait must not leave the others waiting at a barrier).
__device__ __forceinline__ bool bar_and(int id, int nthreads, bool flag) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(res)
      : "r"(flag ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return res != 0;
}

// Exact threshold of N values held in registers (shifted threshold units;
// -inf for no key) by tau_step from t0: every iterate is a lower bound of
// the threshold.  Returns it in shifted units.
template <int N>
__device__ __forceinline__ float reg_row_tau(const float (&w)[N], bool entmax, float t0,
                                             int max_it = 32) {
  float t = fmaxf(t0, -1.f);
  for (int it = 0; it < max_it; ++it) {
    // two partial sums per statistic shorten the dependent chains
    float c0 = 0.f, c1 = 0.f, a0 = 0.f, a1 = 0.f, q0 = 0.f, q1 = 0.f;
    float wmin = INFINITY;
#pragma unroll
    for (int i = 0; i < N; i += 2) {
      const bool in0 = w[i] > t, in1 = w[i + 1] > t;
      const float x0 = in0 ? w[i] : 0.f, x1 = in1 ? w[i + 1] : 0.f;
      c0 += in0 ? 1.f : 0.f;
      c1 += in1 ? 1.f : 0.f;
      a0 += x0;
      a1 += x1;
      q0 = fmaf(x0, x0, q0);
      q1 = fmaf(x1, x1, q1);
      wmin = fminf(wmin, fminf(in0 ? w[i] : INFINITY, in1 ? w[i + 1] : INFINITY));
    }
    if (tau_step(c0 + c1, a0 + a1, q0 + q1, wmin, entmax, t) != 0) break;
  }
  return t;
}

template <int D, int DV, int BN, int KST, int VST, int MODE, int NH = 1>
__global__ void __launch_bounds__((TcLayout<D, DV, BN, KST, VST, MODE, NH>::THREADS), 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, TcArgs A) {
  using LY = TcLayout<D, DV, BN, KST, VST, MODE, NH>;
  constexpr int NWN = LY::NWN;
  constexpr int NC = BN / NH;  // S columns per normalizer thread
  constexpr int NSB = LY::NSB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Problem& P = A.P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- tile selection: heaviest tiles (latest query rows) first ----------
  const int ntq = (P.Tq + TC_BM - 1) / TC_BM;
  const int BH = P.B * P.Hq;
  const int rank = blockIdx.x;
  const int qt = P.causal ? (ntq - 1 - rank / BH) : (rank / BH);
  const int bh = rank % BH;
  const int b = bh / P.Hq, h = bh % P.Hq;
  const int g = h / (P.Hq / P.Hkv);
  const int q0 = qt * TC_BM;
  // this sequence's lengths (packed and paged modes have their own)
  const SeqInfo sq = seq_info(P, b);
  const bool packed = P.cu_q != nullptr;
  const int qlast = min(q0 + TC_BM - 1, sq.Lq - 1);
  const RowRange r_first = row_range(sq.Lq, P.causal, P.window, q0, sq.Lk);
  const RowRange r_last = row_range(sq.Lq, P.causal, P.window, qlast, sq.Lk);
  const int klo = max(0, r_first.lo);
  const int khi = (q0 < sq.Lq) ? min(sq.Lk - 1, r_last.hi) : -1;
  const int kb0 = klo / BN;
  const int kend = (khi >= klo) ? khi / BN + 1 : kb0;
  // blocks of [kb0, kend) the block mask keeps (all of them without one)
  const int nblk = count_kept<BN>(P, b, h, h, qt, kb0, kend);
  // S tiles the MMA produces: the threshold pass multiplies every block twice
  const int nseq = (MODE == TC_TAU) ? 2 * nblk : nblk;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::OFF_BAR);
  const uint32_t bar_q = smem_addr(&bars[0]);
  auto bar_kfull = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto bar_kempty = [&](int s) { return smem_addr(&bars[1 + KST + s]); };
  auto bar_vfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + s]); };
  auto bar_vempty = [&](int s) { return smem_addr(&bars[1 + 2 * KST + VST + s]); };
  auto bar_sfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + s]); };
  auto bar_pfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + NSB + s]); };
  const uint32_t bar_pv = smem_addr(&bars[1 + 2 * KST + 2 * VST + 2 * NSB]);
  // threshold pass: Q has been copied into TMEM (one arrival per normalizer warp)
  const uint32_t bar_qtm = smem_addr(&bars[2 + 2 * KST + 2 * VST + 2 * NSB]);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + LY::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int s = 0; s < NSB; ++s) {
      mbar_init(bar_sfull(s), 1);
      mbar_init(bar_pfull(s), NWN);
    }
    mbar_init(bar_pv, 1);
    mbar_init(bar_qtm, NWN);
    *abort_flag = 0;
    misc[2] = 0;  // threshold pass: some row of the tile overflowed
    fence_barrier_init();
  }
  if (warp == NWN + 1) {
    tmem_alloc(smem_addr(&misc[0]), LY::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == NWN) {
    // ======================= TMA producer ===================================
    if constexpr (LY::REGSPLIT) regs_dec<LY::REGS_CTRL>();
    if (lane == 0 && nblk > 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      if (MODE != TC_TAU) tma_prefetch_desc(&tmv);
      mbar_expect_tx(bar_q, LY::QBYTES);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_rows(smem_addr(smem + LY::OFF_Q + x * TC_BM * 128), &tmq, bar_q, x * 64,
                      packed ? sq.q0 + q0 : q0, packed ? h : bh, packed);
      // the threshold pass streams the key blocks twice (bound pass, then
      // candidate pass)
      int kb = next_kept<BN>(P, b, h, h, qt, kb0, kend);
      for (int j = 0; j < nseq; ++j, kb = next_kept<BN>(P, b, h, h, qt, kb + 1, kend)) {
        if (j == nblk) kb = next_kept<BN>(P, b, h, h, qt, kb0, kend);
        const int ks = j % KST;
        if (j >= KST && !mbar_wait(bar_kempty(ks), ((j / KST) + 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_kfull(ks), LY::KBYTES);
        tma_load_kv<D, BN>(P, &tmk, smem + LY::OFF_K + ks * LY::KBYTES, bar_kfull(ks), b, g, kb,
                           sq);
        if constexpr (MODE != TC_TAU) {
          const int vs = j % VST;
          if (j >= VST && !mbar_wait(bar_vempty(vs), ((j / VST) + 1) & 1, abort_flag))
            break;
          mbar_expect_tx(bar_vfull(vs), LY::VBYTES);
          tma_load_kv<DV, BN>(P, &tmv, smem + LY::OFF_V + vs * LY::VBYTES, bar_vfull(vs), b, g,
                              kb, sq);
        }
      }
    }
  } else if (warp == NWN + 1) {
    // ======================= MMA issuer =====================================
    if constexpr (LY::REGSPLIT) regs_dec<LY::REGS_CTRL>();
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(TC_BM, BN, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16(TC_BM, DV, 0, 1);
      const uint32_t qbase = smem_addr(smem + LY::OFF_Q);
      bool ok = mbar_wait_spin(MODE == TC_TAU ? bar_qtm : bar_q, 0, abort_flag);
      tc_fence_after();
      for (int j = 0; ok && j <= nseq; ++j) {
        if (j < nseq) {
          const int sb = j % NSB, ks = j % KST;
          if (!mbar_wait_spin(bar_kfull(ks), (j / KST) & 1, abort_flag)) break;
          // S buffer sb held P_{j-2}.  With a PV product that reads it, that
          // product was issued by this thread before this QK and tcgen05.mma
          // operations from one thread execute in issue order, so no wait is
          // needed; without one (threshold pass) the normalizer warps must be
          // done reading S_{j-2}.
          if constexpr (MODE == TC_TAU) {
            if (j >= NSB && !mbar_wait_spin(bar_pfull(sb), ((j - NSB) / NSB) & 1, abort_flag))
              break;
          }
          tc_fence_after();
          const uint32_t kbase = smem_addr(smem + LY::OFF_K + ks * LY::KBYTES);
          const uint32_t sdst = tmem + LY::TM_S + sb * BN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t bd =
                sdesc_sw128(kbase + (kk >> 2) * BN * 128 + (kk & 3) * 32, 16, 1024);
            if constexpr (MODE == TC_TAU) {
              // A: dimensions [16 kk, 16 kk + 16) of Q, eight columns in TMEM
              umma_ts(sdst, tmem + LY::TM_Q + kk * 8, bd, IDESC_S, kk > 0 ? 1u : 0u);
            } else {
              const uint64_t ad =
                  sdesc_sw128(qbase + (kk >> 2) * TC_BM * 128 + (kk & 3) * 32, 16, 1024);
              umma_ss(sdst, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(bar_sfull(sb));
          umma_commit(bar_kempty(ks));
        }
        if constexpr (MODE != TC_TAU) {
          if (j >= 1) {
            const int jp = j - 1, sbp = jp % NSB, vs = jp % VST;
            if (!mbar_wait_spin(bar_pfull(sbp), (jp / NSB) & 1, abort_flag)) break;
            if (!mbar_wait_spin(bar_vfull(vs), (jp / VST) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t vbase = smem_addr(smem + LY::OFF_V + vs * LY::VBYTES);
            const uint32_t pt = tmem + LY::TM_S + sbp * BN;
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
              // half hh: its packed P sits at the start of its own S columns,
              // its keys are V rows [hh * NC, (hh + 1) * NC)
#pragma unroll
              for (int kk = 0; kk < NC / 16; ++kk) {
                // V block is [BN keys][DV] in 64-column boxes: MN-major B
                // operand, LBO = box stride, SBO = 8 key rows.
                const uint64_t bd =
                    sdesc_sw128(vbase + (hh * NC + kk * 16) * 128, BN * 128, 1024);
                if constexpr (LY::SHARED_O) {
                  // both halves' keys into the one O
                  umma_ts(tmem + LY::TM_O, pt + hh * NC + kk * 8, bd, IDESC_O,
                          (jp > 0 || hh > 0 || kk > 0) ? 1u : 0u);
                } else {
                  umma_ts(tmem + LY::TM_O + hh * DV, pt + hh * NC + kk * 8, bd, IDESC_O,
                          (jp > 0 || kk > 0) ? 1u : 0u);
                }
              }
            }
            umma_commit(bar_vempty(vs));
            umma_commit(bar_pv);
          }
        }
      }
    }
  } else if (warp >= NWN + 2) {
    // idle warps (register split only): they hand their registers over
    if constexpr (LY::REGSPLIT) regs_dec<LY::REGS_CTRL>();
  } else {
    // ======================= normalizer warps ==============================
    if constexpr (LY::REGSPLIT) regs_inc<LY::REGS_NORM>();
    const int quarter = warp & 3;        // TMEM lane quarter = query rows
    const int half = warp >> 2;          // which columns of the S row
    const int cbase = half * NC;
    const int row = quarter * 32 + lane;
    const int qi = q0 + row;
    const bool row_ok = qi < sq.Lq;
    RowRange rr = row_range(sq.Lq, P.causal, P.window, qi, sq.Lk);
    if (!row_ok) rr = RowRange{1, 0};
    if (rr.hi > sq.Lk - 1) rr.hi = sq.Lk - 1;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const size_t flat = row_index(P, b, h, qi, sq);
    // fast path: no soft-cap and a positive scale, so max(z) = scale * max(s)
    // and exp2(z - m) is one FFMA + EX2 per score
    const bool fast = !(P.softcap > 0.f) && A.zscale > 0.f;
    const float zs = A.zscale;
    const float izs = 1.f / A.zscale;

    float m_run, l_run = 0.f, tau = 0.f;
    // TAU state
    int2* const bufbase = reinterpret_cast<int2*>(smem + LY::OFF_BUF);
    int2* const mybuf = bufbase + (size_t)(half * TC_BM + row) * LY::CAP_STRIDE;
    int nbuf = 0;
    bool ovf = false;
    float lb = -INFINITY;  // lower bound of tau (threshold units)
    float thr = -INFINITY; // the same in stored units, less a rounding margin
    // bound pass: bucket k keeps the largest stored value of the columns
    // congruent to k mod 32 of this thread's part of the row
    float bk[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) bk[k] = -INFINITY;
    if constexpr (MODE == TC_ONLINE) {
      // the sink (softmax1's logit 0, or a learned per-head logit, in log2
      // units) belongs to exactly one half of the row
      const float sink2 = (half == 0) ? sink_logit(P, h) * 1.4426950408889634f : -INFINITY;
      m_run = sink2;
      l_run = (sink2 == -INFINITY) ? 0.f : 1.f;
      if constexpr (LY::SHARED_O) {
        // one running maximum for the row: both halves start from the sink,
        // whose unit weight half 0 alone counts
        m_run = sink_logit(P, h) * 1.4426950408889634f;
      }
    } else {
      m_run = -INFINITY;
    }
    const bool entmax = P.norm == NATTN_ENTMAX15;
    bool alive = true;

    const float vs = fast ? zs : 1.f;  // stored value -> threshold units
    // candidates are tested in stored units against a bound less a margin far
    // above the rounding of the bound's arithmetic
    auto to_thr = [&](float bnd) {
      const float bm = bnd - (fabsf(bnd) + 1.f) * 4e-6f;
      return fast ? bm * izs : bm;
    };
    // End of the bound pass (threshold mode).  The bucket maxima are distinct
    // keys of the row, and adding keys to a set only raises its threshold, so
    // the exact threshold of the bucket set is a lower bound of the row's:
    // every support key lies above it.  With split rows the two halves swap
    // their buckets once (through the stash, which the candidate pass uses
    // only afterwards) and both solve over all of them in registers.
    auto bound_pass_done = [&]() {
      constexpr int NB = 32 * NH;  // bucket maxima of the row
      float w[NB];
#pragma unroll
      for (int k = 0; k < 32; ++k) w[k] = bk[k];
      if constexpr (NH > 1) {
        // the other half of this thread's row is normalizer thread tid ^ 128
        static_assert(NWN == 8, "two halves of four warps");
        constexpr int NT = NWN * 32;
        float4* const sx = reinterpret_cast<float4*>(smem + LY::OFF_STASH);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          sx[q * NT + tid] = make_float4(bk[4 * q], bk[4 * q + 1], bk[4 * q + 2], bk[4 * q + 3]);
        asm volatile("bar.sync 1, %0;" ::"r"(NWN * 32) : "memory");
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 x = sx[q * NT + (tid ^ 128)];
          w[32 + 4 * q] = x.x;
          w[33 + 4 * q] = x.y;
          w[34 + 4 * q] = x.z;
          w[35 + 4 * q] = x.w;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NWN * 32) : "memory");
      }
      float bmax = w[0];
#pragma unroll
      for (int k = 1; k + 1 < NB; k += 2) bmax = fmax3(bmax, w[k], w[k + 1]);
      bmax = fmaxf(bmax, w[NB - 1]);
      m_run = bmax * vs;  // the row maximum (threshold units)
      if (m_run == -INFINITY) {
        lb = thr = -INFINITY;
        return;
      }
#pragma unroll
      for (int k = 0; k < NB; ++k) w[k] = fmaf(w[k], vs, -m_run);
      lb = m_run + reg_row_tau<NB>(w, entmax, -1.f);
      thr = to_thr(lb);
    };

    static_assert(NC == 64 || LY::SHARED_O, "each normalizer thread owns 64 columns of a block");
    // Wait for S(j) and load this thread's 64 scores of key block kbc: z
    // (threshold / log2 units) unless the fast path keeps raw scores; masked
    // entries become -inf.  False when the wait was given up.
    auto load_scores = [&](int j, int kbc, uint32_t(&r)[64]) -> bool {
      const int sb = j % NSB;
      if (!__all_sync(0xffffffffu, mbar_wait_spin(bar_sfull(sb), (j / NSB) & 1, abort_flag)))
        return false;
      tc_fence_after();
      const int jb = kbc * BN + cbase;  // first key of this thread's columns
      const bool edge = !(rr.lo <= jb && rr.hi >= jb + NC - 1);
      // visible keys of this row relative to jb: [klb, klb + span]
      int klb = rr.lo - jb;
      unsigned span = (unsigned)(rr.hi - rr.lo);
      if (rr.hi < rr.lo) {
        klb = NC;
        span = 0;
      }
      const uint32_t saddr = lane_base + LY::TM_S + sb * BN + cbase;
      tmem_ld32(saddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(saddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld_wait();
      if (!fast) {
        if constexpr (MODE == TC_TAU) {
          // per score: the packed polynomial form spills under this mode's
          // register split
#pragma unroll
          for (int k = 0; k < 64; ++k) r[k] = __float_as_uint(tc_z(__uint_as_float(r[k]), A));
        } else {
          tc_z64(r, A);
        }
      }
      if (edge) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if ((unsigned)(k - klb) > span) r[k] = __float_as_uint(-INFINITY);
      }
      return true;
    };
    // S(j) (or the P written over it) has been read: its buffer is free
    auto release = [&](int j) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull(j % NSB));
    };
    const int kfirst = next_kept<BN>(P, b, h, h, qt, kb0, kend);

    if constexpr (MODE == TC_ONLINE && LY::SHARED_O) {
      // Shared O: each half takes 32 of the block's 64 keys; the halves
      // exchange their block maxima (by block parity) so that both move the
      // one running maximum the same way, and each rescales half of O's
      // columns.  Every barrier here also ANDs the warps' progress, so that
      // all eight warps leave the loop together when a wait gives up.
      float* xm = reinterpret_cast<float*>(smem + LY::OFF_XM);
      bool ok_all = true;  // this warp's waits so far
      int kbc = kfirst;
      for (int j = 0; j < nblk; ++j, kbc = next_kept<BN>(P, b, h, h, qt, kbc + 1, kend)) {
        const int sb = j % NSB;
        const bool got =
            __all_sync(0xffffffffu, mbar_wait_spin(bar_sfull(sb), (j / NSB) & 1, abort_flag));
        uint32_t r[32];
        float mx = -INFINITY;
        const uint32_t saddr = lane_base + LY::TM_S + sb * BN + cbase;
        if (got) {
          tc_fence_after();
          const int jb = kbc * BN + cbase;  // first key of this thread's columns
          const bool edge = !(rr.lo <= jb && rr.hi >= jb + NC - 1);
          int klb = rr.lo - jb;
          unsigned span = (unsigned)(rr.hi - rr.lo);
          if (rr.hi < rr.lo) {
            klb = NC;
            span = 0;
          }
          tmem_ld32(saddr, r);
          tmem_ld_wait();
          if (!fast) tc_zn<32>(r, A);
          if (edge) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if ((unsigned)(k - klb) > span) r[k] = __float_as_uint(-INFINITY);
          }
          mx = max32_bits(r);
          if (fast) mx *= zs;
          xm[((j & 1) * 2 + half) * TC_BM + row] = mx;
        }
        if (!bar_and(2, NWN * 32, got && ok_all)) {
          alive = false;
          break;
        }
        mx = fmaxf(mx, xm[((j & 1) * 2 + (half ^ 1)) * TC_BM + row]);
        const float mnew = fmaxf(m_run, mx);
        const bool resc = mnew > m_run + 8.f;
        const float m_use = resc ? mnew : m_run;
        const float alpha = resc ? fast_exp2(m_run - mnew) : 1.f;
        const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
        const float fa = fast ? zs : 1.f;  // p = exp2(x * fa - msafe)
        float s0 = 0.f, s1 = 0.f;
        uint32_t pk[16];  // 32 scores -> 16 packed columns at the start of this half's own
        exp2_packn<32>(&r[0], fa, msafe, s0, s1, pk);
        tmem_st16(saddr, pk);
        tmem_st_wait();
        l_run = l_run * alpha + (s0 + s1);
        // rescale when the maximum moved, after PV(j-1) has completed; each
        // half takes half of O's columns (both have the same alpha)
        if (__any_sync(0xffffffffu, resc) && j > 0) {
          if (__all_sync(0xffffffffu, mbar_wait_spin(bar_pv, (j - 1) & 1, abort_flag))) {
            tc_fence_after();
            const uint32_t oaddr = lane_base + LY::TM_O + half * (DV / 2);
#pragma unroll 1
            for (int c = 0; c < DV / 64; ++c) {
              uint32_t o[32];
              tmem_ld32(oaddr + c * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32(oaddr + c * 32, o);
            }
            tmem_st_wait();
          } else {
            ok_all = false;  // the next block's barrier takes every warp out
          }
        }
        m_run = m_use;
        release(j);
      }
      if (!ok_all) alive = false;
    } else if constexpr (MODE == TC_ONLINE) {
      int kbc = kfirst;  // key block of step j
      for (int j = 0; j < nblk; ++j, kbc = next_kept<BN>(P, b, h, h, qt, kbc + 1, kend)) {
        uint32_t r[64];
        if (!load_scores(j, kbc, r)) {
          alive = false;
          break;
        }
        const uint32_t paddr = lane_base + LY::TM_S + (j % NSB) * BN + cbase;  // packed P

        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; k += 4) {
          mx0 = fmaxf(mx0, __uint_as_float(r[k]));
          mx1 = fmaxf(mx1, __uint_as_float(r[k + 1]));
          mx2 = fmaxf(mx2, __uint_as_float(r[k + 2]));
          mx3 = fmaxf(mx3, __uint_as_float(r[k + 3]));
        }
        float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        if (fast) mx *= zs;
        const float mnew = fmaxf(m_run, mx);
        const bool resc = mnew > m_run + 8.f;
        const float m_use = resc ? mnew : m_run;
        const float alpha = resc ? fast_exp2(m_run - mnew) : 1.f;
        const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
        const float fa = fast ? zs : 1.f;  // p = exp2(x * fa - msafe)
        float s0 = 0.f, s1 = 0.f;
        uint32_t pk[32];  // 64 scores -> 32 packed columns
        exp2_pack64(&r[0], fa, msafe, s0, s1, pk);
        // P(j) goes over S(j)'s own columns; the products in flight read or
        // write the other S buffer and O
        tmem_st32(paddr, pk);
        tmem_st_wait();
        l_run = l_run * alpha + (s0 + s1);
        // Rescale O when the maximum moved (warp-uniform TMEM access).  With
        // two S buffers QK(j) can complete before PV(j-1) is even issued, so
        // PV(j-1) may still be accumulating into O here: the rescale waits
        // for it (reading and rewriting O under an in-flight product loses
        // that product's sum).  PV(j) waits for this block's P, which is
        // released after the rescale.
        if (__any_sync(0xffffffffu, resc) && j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait_spin(bar_pv, (j - 1) & 1, abort_flag))) {
            alive = false;
            break;
          }
          tc_fence_after();
          const uint32_t oaddr = lane_base + LY::TM_O + half * DV;
#pragma unroll 1
          for (int c = 0; c < DV / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(oaddr + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(oaddr + c * 32, o);
          }
          tmem_st_wait();
        }
        m_run = m_use;
        release(j);
      }
    } else {
      // Q into TMEM: each thread its row's share of the head dimensions, read
      // from the 128-byte-swizzled tile the TMA left in shared memory (16-byte
      // chunk c of row r sits at chunk c ^ (r % 8)); column k holds
      // dimensions 2k (low half) and 2k + 1, the layout of an A operand
      if (nblk > 0) {
        alive = mbar_wait(bar_q, 0, abort_flag);
        constexpr int DH = D / NH;              // dimensions per thread
        constexpr int PD = DH < 64 ? DH : 64;   // per TMEM store
#pragma unroll
        for (int p0 = 0; p0 < DH; p0 += PD) {
          const int dim0 = half * DH + p0;
          const uint8_t* qrow = smem + LY::OFF_Q + (dim0 / 64) * TC_BM * 128 + row * 128;
          uint32_t w[PD / 2];
#pragma unroll
          for (int c = 0; c < PD / 8; ++c) {
            const int cc = (dim0 % 64) / 8 + c;
            const uint4 x = *reinterpret_cast<const uint4*>(qrow + ((cc ^ (row & 7)) * 16));
            w[4 * c] = x.x;
            w[4 * c + 1] = x.y;
            w[4 * c + 2] = x.z;
            w[4 * c + 3] = x.w;
          }
          if constexpr (PD == 64)
            tmem_st32(lane_base + LY::TM_Q + dim0 / 2, w);
          else
            tmem_st16(lane_base + LY::TM_Q + dim0 / 2, w);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_qtm);
      alive = __all_sync(0xffffffffu, alive);
      // bound pass: bucket maxima
      int kbc = kfirst;
      for (int j = 0; alive && j < nblk; ++j, kbc = next_kept<BN>(P, b, h, h, qt, kbc + 1, kend)) {
        uint32_t r[64];
        if (!load_scores(j, kbc, r)) {
          alive = false;
          break;
        }
#pragma unroll
        for (int k = 0; k < 32; ++k)
          bk[k] = fmax3(bk[k], __uint_as_float(r[k]), __uint_as_float(r[k + 32]));
        release(j);
      }
      // every normalizer warp takes the bound's named barriers exactly once,
      // also for a tile without key blocks or after a wait was given up
      bound_pass_done();
      // candidate pass: every key above the bound
      kbc = kfirst;
      for (int j = nblk; alive && j < nseq; ++j, kbc = next_kept<BN>(P, b, h, h, qt, kbc + 1, kend)) {
        uint32_t r[64];
        if (!load_scores(j, kbc, r)) {
          alive = false;
          break;
        }
        const int j0 = kbc * BN + cbase;  // key of column 0

#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t* rc = &r[c * 32];
          const bool want = max32_bits(rc) > thr && !ovf;
          if (!__any_sync(0xffffffffu, want)) continue;
          // candidate mask: bit k set when value k is above t, taken from the
          // sign of t - v (-inf values give +inf: never candidates)
          // (four independent eight-bit chains, merged at the end)
          auto cand_mask = [&](float t) {
            unsigned part[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              unsigned mk = 0;
#pragma unroll
              for (int k = 8 * q + 7; k >= 8 * q; --k)
                mk = __funnelshift_l(__float_as_uint(t - __uint_as_float(rc[k])), mk, 1);
              part[q] = mk;
            }
            return part[0] | (part[1] << 8) | (part[2] << 16) | (part[3] << 24);
          };
          unsigned msk = want ? cand_mask(thr) : 0u;
          // the chunk goes to this thread's stash in shared memory so that
          // appends run once per candidate, not once per key (16-byte
          // pieces interleaved across the normalizer threads: conflict-free
          // stores; a thread reads back only what it wrote)
          constexpr int NT = NWN * 32;
          float* const sst = reinterpret_cast<float*>(smem + LY::OFF_STASH);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(sst)[q * NT + tid] =
                make_float4(__uint_as_float(rc[4 * q]), __uint_as_float(rc[4 * q + 1]),
                            __uint_as_float(rc[4 * q + 2]), __uint_as_float(rc[4 * q + 3]));
          auto stash = [&](int k) { return sst[((k >> 2) * NT + tid) * 4 + (k & 3)]; };
          const int kj = j0 + c * 32;
          // append candidates (lowest key first) while there is room; a key a
          // rounding step below the bound is harmless (the exact solve drops
          // it)
          auto append = [&](int room) {
            int2* ptr = mybuf + nbuf;
            int na = 0;
            // two candidates per trip, so that two stash loads are in flight
            while (msk && na + 1 < room) {
              const int k0 = __ffs(msk) - 1;
              msk &= msk - 1;
              const int k1 = msk ? __ffs(msk) - 1 : -1;
              msk &= msk - 1;  // no-op when msk is already 0
              const float v0 = stash(k0);
              const float v1 = (k1 >= 0) ? stash(k1) : 0.f;
              *ptr = make_int2(kj + k0, __float_as_int(v0));
              if (k1 >= 0) ptr[1] = make_int2(kj + k1, __float_as_int(v1));
              ptr += (k1 >= 0) ? 2 : 1;
              na += (k1 >= 0) ? 2 : 1;
            }
            if (msk && na < room) {  // room for one more
              const int k = __ffs(msk) - 1;
              msk &= msk - 1;
              *ptr++ = make_int2(kj + k, __float_as_int(stash(k)));
              ++na;
            }
            nbuf += na;
          };
          // a row whose buffer cannot take this chunk's candidates has a
          // support far wider than the buffer (with the bucket bound the
          // candidates are the support and about one key more): it stops
          // collecting, and the wide kernel takes its tile
          if (nbuf + __popc(msk) > LY::CAPR) {
            ovf = true;
            msk = 0;
          }
          if (__any_sync(0xffffffffu, msk != 0)) append(32);
        }
        release(j);
      }
    }


    // ---- epilogue ----------------------------------------------------------
    if constexpr (MODE == TC_TAU) {
      // Each row half writes its candidates out as they are (value row of
      // the key, value less the row maximum in threshold units); the apply
      // kernel solves every row's exact threshold with a warp per row and
      // gathers its support.  A row whose candidates overflowed in either
      // half is marked (count -1) and its tile listed for the wide kernel.
      bool ovf_r = ovf;
      float lb_r = lb;
      if constexpr (NH > 1) {
        float2* xs = reinterpret_cast<float2*>(smem + LY::OFF_Q);  // Q is no longer read
        xs[half * TC_BM + row] = make_float2(lb, ovf ? 1.f : 0.f);
        asm volatile("bar.sync 1, %0;" ::"r"(NWN * 32) : "memory");
        const float2 o = xs[(NH - 1 - half) * TC_BM + row];
        lb_r = fmaxf(lb, o.x);  // both halves' bounds bound the row
        ovf_r = ovf || o.y != 0.f;
      }
      if (row_ok) {
        const size_t seg = flat * NH + half;
        if (ovf_r) {
          A.sup_count[seg] = -1;
          if (half == 0) atomicOr(&misc[2], 1u);
        } else {
          int2* dst = A.sup_list + seg * LY::CAPR;
          for (int i = 0; i < nbuf; ++i) {
            const int2 e = mybuf[i];
            dst[i] = make_int2(value_row(P, b, g, e.x, sq),
                               __float_as_int(fmaf(__int_as_float(e.y), vs, -m_run)));
          }
          A.sup_count[seg] = nbuf;
        }
        if (half == 0) {
          A.tau[flat] = m_run;         // row maximum (threshold units)
          A.rlb[flat] = lb_r - m_run;  // a lower bound of tau less it
        }
      }
    } else {
      // with two S buffers the last two PVs may both be in flight here (S(j)
      // only guarantees PV(j - 2)): wait for both
      const bool have_o =
          __all_sync(0xffffffffu, alive && nblk > 0 &&
                                      mbar_wait_last2(bar_pv, nblk - 1, nblk > 1, abort_flag));
      tc_fence_after();
      // combine the halves: scale factors ca (half 0) and cb (half 1)
      float ca = 1.f, cb = 0.f, stat = tau;
      if constexpr (MODE == TC_ONLINE) {
        float m0 = m_run, l0 = l_run, m1 = -INFINITY, l1 = 0.f;
        if constexpr (NH > 1) {
          float2* xch = reinterpret_cast<float2*>(smem + LY::OFF_XCH);
          xch[half * TC_BM + row] = make_float2(m_run, l_run);
          asm volatile("bar.sync 1, %0;" ::"r"(NWN * 32) : "memory");
          const float2 a0 = xch[row], a1 = xch[TC_BM + row];
          m0 = a0.x;
          l0 = a0.y;
          m1 = a1.x;
          l1 = a1.y;
        }
        const float M = fmaxf(m0, m1);
        const float msafe = (M == -INFINITY) ? 0.f : M;
        const float e0 = fast_exp2(m0 - msafe), e1 = fast_exp2(m1 - msafe);
        const float l = l0 * e0 + l1 * e1;
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        ca = e0 * inv;
        cb = e1 * inv;
        stat = (l > 0.f) ? (msafe + log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
      // this thread writes output columns [half * DV / NH, (half + 1) * DV / NH)
      constexpr int OC = DV / NH;
      bf16* orow = P.out + flat * DV + half * OC;
      const uint32_t oaddr = lane_base + LY::TM_O + half * OC;
#pragma unroll 1
      for (int c = 0; c < OC / 32; ++c) {
        uint32_t r[32], r1[32];
        // (shared O: this half's columns of the one O, already both halves'
        // sum)
        constexpr bool TWO_O = NH > 1 && !LY::SHARED_O;
        if (have_o) {
          tmem_ld32(oaddr + c * 32, r);
          if constexpr (TWO_O) tmem_ld32(oaddr + DV + c * 32, r1);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = r1[k] = 0u;
        }
        float o[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          o[k] = __uint_as_float(r[k]) * ca;
          if constexpr (TWO_O) o[k] = fmaf(__uint_as_float(r1[k]), cb, o[k]);
        }
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint4 v;
            v.x = pack_bf16(o[k + 0], o[k + 1]);
            v.y = pack_bf16(o[k + 2], o[k + 3]);
            v.z = pack_bf16(o[k + 4], o[k + 5]);
            v.w = pack_bf16(o[k + 6], o[k + 7]);
            dst[k / 8] = v;
          }
        }
      }
      if (row_ok && P.row_stat && half == 0) P.row_stat[flat] = stat;
      if constexpr (MODE == TC_ONLINE) {
        if (row_ok && P.row_nnz && half == 0) {
          int n = 0;
          if (rr.hi >= rr.lo) {
            if (P.block_mask == nullptr) {
              n = rr.hi - rr.lo + 1;
            } else {
              for (int kb = kb0; kb < kend; ++kb)
                if (block_kept(P, b, h, qt, (kb * BN) >> 7))
                  n += max(0, min(rr.hi, kb * BN + BN - 1) - max(rr.lo, kb * BN) + 1);
            }
          }
          P.row_nnz[flat] = n;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == NWN + 1) tmem_dealloc(tmem, LY::TM_COLS);
  if constexpr (MODE == TC_TAU) {
    if (tid == 0 && misc[2] != 0) A.wide_tiles[atomicAdd(A.wide_count, 1)] = rank;
  }
}


// Sparse phase 2: RPW query rows per warp (32 / RPW lanes each).  A row's
// candidates (every key above a lower bound of its threshold, written by the
// threshold pass) give the exact threshold by the Newton iteration of
// tau_step, with the sums taken across the row's lanes; then
// O = sum over the support of p_j V_j in fp32 on CUDA cores.  The support of
// sparsemax / 1.5-entmax is a handful of keys per row, so this reads
// |support| value rows instead of multiplying every block, and the weights
// enter the sum in full precision.  The kernel is bound by latency: with
// short supports (sparsemax) by its dependent steps, so two rows per warp
// share them; with longer ones (1.5-entmax) by the value-row loads in
// flight, which the registers of one row per warp hold more of.  Lane l of a
// row owns output columns [l * PER, (l+1) * PER).
constexpr int APPLY_WARPS = 4;

template <int DV, int NSEG, int CAPR, int RPW>
__global__ void __launch_bounds__(APPLY_WARPS * 32)
    sparse_apply_kernel(Problem P, const int* __restrict__ sup_count,
                        const int2* __restrict__ sup_list, const float* __restrict__ rmax,
                        const float* __restrict__ rlb) {
  constexpr int LPR = 32 / RPW;                 // lanes per row
  constexpr int PER = DV / LPR;                 // columns per lane (2 .. 16)
  constexpr int NCAND = NSEG * CAPR;            // candidates a row can have
  constexpr int NE = (NCAND + LPR - 1) / LPR;   // candidate slots per lane
  constexpr int G = 8 / RPW;                    // value rows per gather step
  constexpr unsigned RMASK = (LPR == 32) ? 0xffffffffu : ((1u << LPR) - 1u);
  __shared__ int2 sup[APPLY_WARPS][RPW][NCAND];  // (value row, weight) of the support
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int hw = lane / LPR, hl = lane % LPR;   // row of the warp, lane of the row
  const size_t rows =
      P.cu_q != nullptr ? (size_t)P.total_q * P.Hq : (size_t)P.B * P.Hq * P.Tq;
  // packed: rows past the last sequence belong to no sequence
  const size_t owned =
      P.cu_q != nullptr ? min(rows, (size_t)min(P.cu_q[P.B], P.total_q) * P.Hq) : rows;
  const size_t row0 = ((size_t)blockIdx.x * APPLY_WARPS + wid) * RPW;
  if (row0 >= owned) return;  // every row of the warp idle
  const size_t flat = row0 + hw;
  // a row that is not there, or that overflowed (the row-wise pass writes
  // it), still takes part in the warp's shuffles with no candidates
  const bool there = flat < owned;
  int c[NSEG];
  bool ovf = false;
  int ntot = 0;
#pragma unroll
  for (int sg = 0; sg < NSEG; ++sg) {
    c[sg] = there ? sup_count[flat * NSEG + sg] : 0;
    ovf |= c[sg] < 0;
  }
#pragma unroll
  for (int sg = 0; sg < NSEG; ++sg) {
    c[sg] = ovf ? 0 : min(c[sg], CAPR);
    ntot += c[sg];
  }
  // slot r of lane l holds entry r * LPR + l of the concatenated segments
  const int2* lst = sup_list + flat * NCAND;
  float w[NE];
  int vr[NE];
#pragma unroll
  for (int r = 0; r < NE; ++r) {
    const int e = r * LPR + hl;
    int at = -1;
    if (e < c[0]) {
      at = e;
    } else if constexpr (NSEG > 1) {
      if (e - c[0] < c[1]) at = CAPR + (e - c[0]);
    }
    const int2 x = (at >= 0) ? lst[at] : make_int2(0, __float_as_int(-INFINITY));
    vr[r] = x.x;
    w[r] = __int_as_float(x.y);
  }
  const bool entmax = P.norm == NATTN_ENTMAX15;
  float t = (ntot > 0) ? fmaxf(rlb[flat], -1.f) : INFINITY;  // less the row maximum
  // the rows of the warp iterate until all have converged
  bool done = ntot == 0;
  for (int it = 0; it < 64 && !__all_sync(0xffffffffu, done); ++it) {
    float cnt = 0.f, s1 = 0.f, s2 = 0.f, wmin = INFINITY;
#pragma unroll
    for (int r = 0; r < NE; ++r) {
      if (w[r] > t) {
        cnt += 1.f;
        s1 += w[r];
        s2 = fmaf(w[r], w[r], s2);
        wmin = fminf(wmin, w[r]);
      }
    }
    // xor butterflies inside the lanes of the row: every lane of the row
    // ends with the same sums
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) {
      cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
      s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      s2 += __shfl_xor_sync(0xffffffffu, s2, off);
      wmin = fminf(wmin, __shfl_xor_sync(0xffffffffu, wmin, off));
    }
    if (done) continue;
    done = tau_step(cnt, s1, s2, wmin, entmax, t) != 0;
  }
  const float tau = t;
  // the support, compacted in candidate order into this row's list
  int nsup = 0;
  const unsigned lt = (1u << hl) - 1u;
#pragma unroll
  for (int r = 0; r < NE; ++r) {
    const float x = w[r] - tau;
    const bool in = x > 0.f;
    const unsigned bal = (__ballot_sync(0xffffffffu, in) >> (LPR * hw)) & RMASK;
    if (in)
      sup[wid][hw][nsup + __popc(bal & lt)] =
          make_int2(vr[r], __float_as_int(entmax ? x * x : x));
    nsup += __popc(bal);
  }
  __syncwarp();
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  const bf16* vbase = P.v + hl * PER;
  // one value row's slice of this lane: PER bf16 in PER / 2 words
  constexpr int NW = PER / 2;
  auto load_row = [&](const bf16* vr_, uint32_t (&x)[NW]) {
    if constexpr (NW >= 4) {
#pragma unroll
      for (int q = 0; q < NW / 4; ++q) {
        const uint4 v = reinterpret_cast<const uint4*>(vr_)[q];
        x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
      }
    } else if constexpr (NW == 2) {
      const uint2 v = *reinterpret_cast<const uint2*>(vr_);
      x[0] = v.x; x[1] = v.y;
    } else {
      x[0] = *reinterpret_cast<const uint32_t*>(vr_);
    }
  };
  // G value rows per step, their loads issued before any is used (each row
  // of the warp at its own pace: no shuffles from here on)
  auto fma_row = [&](float p, const uint32_t (&x)[NW]) {
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      acc[2 * k] += p * bf16lo(x[k]);
      acc[2 * k + 1] += p * bf16hi(x[k]);
    }
  };
  int e = 0;
  for (; e + G <= nsup; e += G) {
    int2 en[G];
    uint32_t x[G][NW];
#pragma unroll
    for (int u = 0; u < G; ++u) en[u] = sup[wid][hw][e + u];
#pragma unroll
    for (int u = 0; u < G; ++u) load_row(vbase + (size_t)en[u].x * DV, x[u]);
#pragma unroll
    for (int u = 0; u < G; ++u) fma_row(__int_as_float(en[u].y), x[u]);
  }
  for (; e < nsup; ++e) {
    const int2 en = sup[wid][hw][e];
    uint32_t x[NW];
    load_row(vbase + (size_t)en.x * DV, x);
    fma_row(__int_as_float(en.y), x);
  }
  if (!there || ovf) return;
  bf16* o = P.out + flat * DV + hl * PER;
  uint32_t ov[NW];
#pragma unroll
  for (int k = 0; k < NW; ++k) ov[k] = pack_bf16(acc[2 * k], acc[2 * k + 1]);
  if constexpr (NW >= 4) {
#pragma unroll
    for (int q = 0; q < NW / 4; ++q)
      reinterpret_cast<uint4*>(o)[q] = make_uint4(ov[4 * q], ov[4 * q + 1], ov[4 * q + 2], ov[4 * q + 3]);
  } else if constexpr (NW == 2) {
    *reinterpret_cast<uint2*>(o) = make_uint2(ov[0], ov[1]);
  } else {
    *reinterpret_cast<uint32_t*>(o) = ov[0];
  }
  if (hl == 0) {
    if (P.row_stat) P.row_stat[flat] = (ntot > 0) ? rmax[flat] + tau : INFINITY;
    if (P.row_nnz) P.row_nnz[flat] = nsup;
  }
}

}  // namespace nattn
