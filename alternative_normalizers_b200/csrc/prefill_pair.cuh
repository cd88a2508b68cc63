// Online softmax / softmax1 prefill with two query tiles per CTA.
//
// The CTA takes the same 128 query rows of two query heads that read the same
// key/value head (grouped-query attention with an even group), so both tiles
// walk the same visible key blocks and every K/V block brought in by TMA
// feeds two products.  Each tile owns one S buffer and one O accumulator in
// TMEM (2 x (128 + 128) = 512 columns) and one normalizer warpgroup.  The
// single MMA thread interleaves the tiles:
//
//     ... PV_A(j)  QK_A(j+1)  PV_B(j)  QK_B(j+1)  PV_A(j+1) ...
//
// so while warpgroup A turns S_A(j+1) into P it is the other tile's products
// that keep the tensor pipe busy, and the hand-off latencies of one tile
// (S ready -> normalizer, P ready -> PV issue) are covered by the other
// tile's work.  P is written back over its own S columns; the QK that next
// overwrites them is issued after the PV that reads them, and tcgen05.mma
// operations from one thread execute in issue order.
//
// softmax1 starts each row from the virtual logit-0 / value-0 sink ("HF
// Attention Normalizers", section "Important Limitations"): m0 = 0, l0 = 1.
#pragma once

#include "common.cuh"
#include "prefill_tc.cuh"
#include "problem.cuh"

namespace nattn {

// 12 warps: two normalizer warpgroups (warps 0-7), then a third warpgroup
// with the TMA warp (8), the MMA warp (9) and two warps with no role.  The
// block is launched at 168 registers a thread (384 x 168 = 64512); the third
// warpgroup gives back down to 72 and the normalizer warpgroups take 216,
// enough to hold a whole S row: 2 x 128 x 216 + 128 x 72 = 64512.  (With 56
// for the TMA / MMA warps the step ran 0.4 % slower.)
constexpr int PAIR_THREADS = 384;
constexpr int PAIR_REGS_NORM = 216;
constexpr int PAIR_REGS_CTRL = 72;
static_assert(2 * 128 * PAIR_REGS_NORM + 128 * PAIR_REGS_CTRL <= PAIR_THREADS * 168,
              "register split exceeds the launch allocation");

template <int D, int KST, int VST>
struct PairLayout {
  static constexpr int BN = 128;
  static constexpr int QBYTES = D * TC_BM * 2;  // one tile
  static constexpr int KBYTES = D * BN * 2;
  static constexpr int VBYTES = D * BN * 2;
  static constexpr int OFF_Q = 0;               // tile 0, then tile 1
  static constexpr int OFF_K = 2 * QBYTES;
  static constexpr int OFF_V = OFF_K + KST * KBYTES;
  static constexpr int OFF_BAR = OFF_V + VST * VBYTES;
  // q, kfull/kempty, vfull/vempty, sfull[2], pfull[2], pvdone[2], qempty
  static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 6 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // work-sorted schedule: (sequence, query tile) entries, heaviest first
  static constexpr int SCHED_MAX = 512;
  static constexpr int OFF_SCHED = OFF_MISC + 16;
  static constexpr int BYTES = OFF_SCHED + SCHED_MAX * 4 + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int TM_S = 0;                // tile t: TM_S + t * BN
  static constexpr int TM_O = 2 * BN;           // tile t: TM_O + t * D
  static constexpr int TM_COLS = (2 * BN + 2 * D <= 256) ? 256 : 512;
  static_assert(2 * BN + 2 * D <= 512, "TMEM budget");
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
};

// One unit of work: the same 128 query rows of the two query heads h0, h0 + 1
// (one GQA group) of batch b, and the visible key blocks [kb0, kb0 + nblk).
struct PairTile {
  int b, h0, g, bh0, q0, kb0, kend, nblk;  // nblk: blocks in [kb0, kend) a block mask keeps
  SeqInfo s;                               // the sequence's lengths / first tokens
};

// Tile of heaviest-first rank `rank`: under the causal mask the last query
// tiles see the most keys, so ranks walk the query tiles from the last.
// Layouts of Q / K / V the kernel is compiled for.
enum PairLayoutKind { PAIR_DENSE = 0, PAIR_PACKED = 1, PAIR_PAGED = 2 };

template <int LAY>
__device__ __forceinline__ PairTile pair_tile_at(const Problem& P, int b, int hp, int qt) {
  PairTile T;
  T.b = b;
  T.h0 = 2 * hp;
  T.g = T.h0 / (P.Hq / P.Hkv);
  T.bh0 = T.b * P.Hq + T.h0;
  T.q0 = qt * TC_BM;
  if constexpr (LAY == PAIR_DENSE)
    T.s = SeqInfo{P.Tq, P.Tk, 0, 0};
  else
    T.s = seq_info(P, T.b);
  const int qlast = min(T.q0 + TC_BM - 1, T.s.Lq - 1);
  const RowRange r_first = row_range(T.s.Lq, P.causal, P.window, T.q0, T.s.Lk);
  const RowRange r_last = row_range(T.s.Lq, P.causal, P.window, qlast, T.s.Lk);
  const int klo = max(0, r_first.lo);
  const int khi = (T.q0 < T.s.Lq) ? min(T.s.Lk - 1, r_last.hi) : -1;
  T.kb0 = klo / 128;
  T.kend = (khi >= klo) ? khi / 128 + 1 : T.kb0;
  T.nblk = count_kept<128>(P, T.b, T.h0, T.h0 + 1, qt, T.kb0, T.kend);
  return T;
}
template <int LAY>
__device__ __forceinline__ PairTile pair_tile(const Problem& P, int rank) {
  const int ntq = (P.Tq + TC_BM - 1) / TC_BM;
  const int HP = P.Hq / 2;  // head pairs per batch
  const int BP = P.B * HP;
  const int qt = P.causal ? (ntq - 1 - rank / BP) : (rank / BP);
  const int bp = rank % BP;
  return pair_tile_at<LAY>(P, bp / HP, bp % HP, qt);
}

// Persistent schedule: CTA c of G takes, in round k, rank k*G + c (k even)
// or k*G + G-1-c (k odd).  Over heaviest-first ranks this snake evens out
// the CTAs' total work.  Ranks only grow, so the first one past the end
// ends the CTA's walk.
__device__ __forceinline__ int pair_rank(int round, int c, int G) {
  return round * G + ((round & 1) ? (G - 1 - c) : c);
}

// One normalizer warp of tile t = warp / 4: thread = query row = TMEM lane of
// its lane quarter.  The S row is read from TMEM once per block and held in
// registers (128 values) for the maximum and the exponentials.
// `g0` counts the blocks of the CTA's earlier tiles: barrier phases run on
// across tiles.  Returns false if a wait gave up.
template <int D, int KST, int VST, bool CAP, bool BM>
__device__ __forceinline__ bool prefill_pair_normalizer(
    const TcArgs& A, uint8_t* smem, uint32_t tmem, int warp, int lane, int b, int q0, int bh0,
    int kb0, int kend, int nblk, const SeqInfo& sq, int g0, uint32_t bar_sf, uint32_t bar_pf,
    uint32_t bar_pvt, volatile int* abort_flag) {
  using LY = PairLayout<D, KST, VST>;
  constexpr int BN = LY::BN;
  const Problem& P = A.P;
  const int t = warp >> 2, quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const int qi = q0 + row;
  const bool row_ok = qi < sq.Lq;
  RowRange rr = row_range(sq.Lq, P.causal, P.window, qi, sq.Lk);
  if (!row_ok) rr = RowRange{1, 0};
  if (rr.hi > sq.Lk - 1) rr.hi = sq.Lk - 1;
  const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
  const uint32_t sbase = lane_base + LY::TM_S + t * BN;
  const uint32_t obase = lane_base + LY::TM_O + t * D;
  const size_t flat = row_index(P, b, (bh0 + t) % P.Hq, qi, sq);
  // CAP: soft-cap (or a non-positive scale), scores go through tc_z; else
  // max(z) = scale * max(s) and exp2(z - m) is one FFMA + EX2 per score
  constexpr bool fast = !CAP;
  const float fa = fast ? A.zscale : 1.f;  // p = exp2(x * fa - m)
  // the running state starts from the sink (softmax1: logit 0; a learned
  // per-head sink: its logit, here in log2 units): m0 = sink, l0 = 1
  const float sink2 = sink_logit(P, (bh0 + t) % P.Hq) * 1.4426950408889634f;
  float m_run = sink2;
  float l_run = (sink2 == -INFINITY) ? 0.f : 1.f;
  bool alive = true;
  // block mask: the pair walks the blocks either head keeps; a block this
  // tile's head drops is masked whole
  const int qb = q0 >> 7, hp = bh0 % P.Hq, hown = hp + t;
  int kb = BM ? next_kept<BN>(P, b, hp, hp + 1, qb, kb0, kend) : kb0;
  int nvis = 0;  // visible keys in kept blocks (row_nnz)

  for (int j = 0; j < nblk; ++j) {
    if (!__all_sync(0xffffffffu, mbar_wait_busy(bar_sf, (g0 + j) & 1, abort_flag))) {
      alive = false;
      break;
    }
    tc_fence_after();
    const int jb = kb * BN;
    const bool own = !BM || block_kept(P, b, hown, qb, kb);
    const bool edge = !own || !(rr.lo <= jb && rr.hi >= jb + BN - 1);
    int kl = rr.lo - jb;
    unsigned span = (unsigned)(rr.hi - rr.lo);
    if (rr.hi < rr.lo || !own) {
      kl = BN;
      span = 0;
    } else if (BM) {
      nvis += max(0, min(rr.hi, jb + BN - 1) - max(rr.lo, jb) + 1);
    }
    kb = BM ? next_kept<BN>(P, b, hp, hp + 1, qb, kb + 1, kend) : kb + 1;
    // the whole S row (128 scores) in registers: one TMEM read per block;
    // x is the raw score on the fast path, else z in log2 units; masked
    // entries -inf
    uint32_t r[BN];
#pragma unroll
    for (int c = 0; c < BN / 32; ++c)
      tmem_ld32(sbase + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
    tmem_ld_wait();
    if (!fast) {
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) tc_z64(&r[c * 64], A);
    }
    if (edge) {
#pragma unroll
      for (int k = 0; k < BN; ++k)
        if ((unsigned)(k - kl) > span) r[k] = __float_as_uint(-INFINITY);
    }
    float mx = fmaxf(fmaxf(max32_bits(&r[0]), max32_bits(&r[32])),
                     fmaxf(max32_bits(&r[64]), max32_bits(&r[96])));
    mx *= fa;
    const float mnew = fmaxf(m_run, mx);
    const bool resc = mnew > m_run + 8.f;  // move the maximum only when it grows by 2^8
    const float m_use = resc ? mnew : m_run;
    const float alpha = resc ? fast_exp2(m_run - mnew) : 1.f;
    const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t pk[32];
      exp2_pack64(&r[hh * 64], fa, msafe, s0, s1, pk);
      // packed P of keys [64 hh, 64 hh + 64) over S columns already read
      tmem_st32(sbase + hh * 32, pk);
    }
    tmem_st_wait();
    l_run = l_run * alpha + (s0 + s1);
    if (__any_sync(0xffffffffu, resc) && j > 0) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar_pvt, (g0 + j - 1) & 1, abort_flag))) {
        alive = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(obase + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        tmem_st32(obase + c * 32, o);
      }
      tmem_st_wait();
    }
    m_run = m_use;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_pf);
  }

  // ---- epilogue -------------------------------------------------------------
  const bool have_o = __all_sync(
      0xffffffffu, alive && nblk > 0 && mbar_wait(bar_pvt, (g0 + nblk - 1) & 1, abort_flag));
  tc_fence_after();
  const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
  const float msafe = (m_run == -INFINITY) ? 0.f : m_run;
  const float stat = (l_run > 0.f) ? (msafe + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
  bf16* orow = P.out + flat * D;
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    if (have_o) {
      tmem_ld32(obase + c * 32, r);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) r[k] = 0u;
    }
    if (row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
      for (int k = 0; k < 32; k += 8) {
        uint4 v;
        v.x = pack_bf16(__uint_as_float(r[k + 0]) * inv, __uint_as_float(r[k + 1]) * inv);
        v.y = pack_bf16(__uint_as_float(r[k + 2]) * inv, __uint_as_float(r[k + 3]) * inv);
        v.z = pack_bf16(__uint_as_float(r[k + 4]) * inv, __uint_as_float(r[k + 5]) * inv);
        v.w = pack_bf16(__uint_as_float(r[k + 6]) * inv, __uint_as_float(r[k + 7]) * inv);
        dst[k / 8] = v;
      }
    }
  }
  if (row_ok && P.row_stat) P.row_stat[flat] = stat;
  if (row_ok && P.row_nnz)
    P.row_nnz[flat] = BM ? nvis : (rr.hi >= rr.lo ? rr.hi - rr.lo + 1 : 0);
  return alive;
}

// BM: a block mask is given; LAY: dense, packed or paged Q / K / V (separate
// instances, so that the dense launches without a block mask carry none of
// the other cases' per-block work)
template <int D, int KST, int VST, bool CAP, bool BM, int LAY>
__global__ void __launch_bounds__(PAIR_THREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, TcArgs A) {
  using LY = PairLayout<D, KST, VST>;
  constexpr int BN = LY::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Problem& P = A.P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- persistent: this CTA walks tiles pair_rank(0..), see pair_rank ----
  const int ntq = (P.Tq + TC_BM - 1) / TC_BM;
  const int ntiles = P.B * (P.Hq / 2) * ntq;
  const int G = gridDim.x, cta = blockIdx.x;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::OFF_BAR);
  const uint32_t bar_q = smem_addr(&bars[0]);
  auto bar_kfull = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto bar_kempty = [&](int s) { return smem_addr(&bars[1 + KST + s]); };
  auto bar_vfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + s]); };
  auto bar_vempty = [&](int s) { return smem_addr(&bars[1 + 2 * KST + VST + s]); };
  auto bar_sfull = [&](int t) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + t]); };
  auto bar_pfull = [&](int t) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + 2 + t]); };
  auto bar_pv = [&](int t) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + 4 + t]); };
  // the MMAs that read the Q tiles of a tile are done: the next tile's Q may load
  const uint32_t bar_qempty = smem_addr(&bars[1 + 2 * KST + 2 * VST + 6]);
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull(t), 1);
      mbar_init(bar_pfull(t), 4);
      mbar_init(bar_pv(t), 1);
    }
    mbar_init(bar_qempty, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_addr(&misc[0]), LY::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  // ---- schedule ------------------------------------------------------------
  // Sequences of one length (dense, paged chunks of equal length): every
  // tile of a query-tile index does the same work, so the heaviest-first
  // ranks are already sorted.  Packed requests of different lengths: the
  // (sequence, query tile) entries are ranked by their work (visible key
  // blocks), heaviest first, ties by index: the same order in every CTA.  An
  // entry stands for its head pairs, walked consecutively, and the snake of
  // pair_rank runs over that list; entries without work are left out.  (With
  // the padded ranks, where short requests leave empty slots, the snake's
  // balance was 70 % of ideal on requests of 4096/2048/1536/512 tokens; over
  // the sorted list 97 %.)
  constexpr bool SORTED = LAY == PAIR_PACKED;
  const int HP = P.Hq / 2;
  int* sched = reinterpret_cast<int*>(smem + LY::OFF_SCHED);
  int nwalk = ntiles;
  bool use_sched = false;
  if constexpr (SORTED) {
    const int ncombo = P.B * ntq;
    if (ncombo <= LY::SCHED_MAX) {
      use_sched = true;
      int* keys = reinterpret_cast<int*>(smem + LY::OFF_K);  // the K ring: nothing loaded yet
      int* s_nwork = sched + LY::SCHED_MAX;
      if (tid == 0) *s_nwork = 0;
      for (int c = tid; c < ncombo; c += PAIR_THREADS) {
        const int bb = c / ntq, qt = c % ntq;
        keys[c] = pair_tile_at<LAY>(P, bb, 0, qt).nblk;
      }
      __syncthreads();
      int mine = 0;
      for (int c = tid; c < ncombo; c += PAIR_THREADS) {
        const int kc = keys[c];
        int pos = 0;
        for (int c2 = 0; c2 < ncombo; ++c2) {
          const int k2 = keys[c2];
          pos += (k2 > kc || (k2 == kc && c2 < c)) ? 1 : 0;
        }
        sched[pos] = c;
        mine += kc > 0 ? 1 : 0;
      }
      if (mine) atomicAdd(s_nwork, mine);
      __syncthreads();
      nwalk = *s_nwork * HP;
    }
  }
  auto tile_of = [&](int idx) -> PairTile {
    if (use_sched) {
      const int c = sched[idx / HP];
      return pair_tile_at<LAY>(P, c / ntq, idx % HP, c % ntq);
    }
    return pair_tile<LAY>(P, idx);
  };

  if (warp < 8) {
    regs_inc<PAIR_REGS_NORM>();
    // normalizer warpgroups: see prefill_pair_normalizer above
    int g0 = 0;
    for (int round = 0;; ++round) {
      const int rank = pair_rank(round, cta, G);
      if (rank >= (SORTED ? nwalk : ntiles)) break;
      const PairTile T = SORTED ? tile_of(rank) : pair_tile<LAY>(P, rank);
      if (!prefill_pair_normalizer<D, KST, VST, CAP, BM>(A, smem, tmem, warp, lane, T.b, T.q0,
                                                      T.bh0, T.kb0, T.kend, T.nblk, T.s, g0,
                                                      bar_sfull(warp >> 2),
                                                      bar_pfull(warp >> 2), bar_pv(warp >> 2),
                                                      abort_flag))
        break;
      g0 += T.nblk;
    }
  } else {
    regs_dec<PAIR_REGS_CTRL>();
    if (warp == 8 && lane == 0) {
      // ======================= TMA producer =================================
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      constexpr bool packed = LAY == PAIR_PACKED;
      int g0 = 0, tq = 0;  // blocks and tiles (with blocks) already loaded
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int rank = pair_rank(round, cta, G);
        if (rank >= (SORTED ? nwalk : ntiles)) break;
        const PairTile T = SORTED ? tile_of(rank) : pair_tile<LAY>(P, rank);
        if (T.nblk == 0) continue;
        // the previous tile's QK products have read its Q tiles
        if (tq > 0 && !mbar_wait(bar_qempty, (tq - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_q, 2 * LY::QBYTES);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tma_load_rows(smem_addr(smem + LY::OFF_Q + t * LY::QBYTES + x * TC_BM * 128), &tmq,
                          bar_q, x * 64, packed ? T.s.q0 + T.q0 : T.q0,
                          packed ? T.h0 + t : T.bh0 + t, packed);
        int kb = next_kept<BN>(P, T.b, T.h0, T.h0 + 1, T.q0 >> 7, T.kb0, T.kend);
        for (int j = 0; j < T.nblk; ++j, kb = next_kept<BN>(P, T.b, T.h0, T.h0 + 1, T.q0 >> 7,
                                                            kb + 1, T.kend)) {
          const int gj = g0 + j;
          const int ks = gj % KST;
          if (gj >= KST && !mbar_wait(bar_kempty(ks), ((gj / KST) + 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar_kfull(ks), LY::KBYTES);
          uint8_t* kdst = smem + LY::OFF_K + ks * LY::KBYTES;
          if constexpr (LAY == PAIR_DENSE) {
#pragma unroll
            for (int x = 0; x < D / 64; ++x)
              tma_load_3d(smem_addr(kdst + x * BN * 128), &tmk, bar_kfull(ks), x * 64, kb * BN,
                          T.b * P.Hkv + T.g);
          } else {
            tma_load_kv<D, BN>(P, &tmk, kdst, bar_kfull(ks), T.b, T.g, kb, T.s);
          }
          const int vs = gj % VST;
          if (gj >= VST && !mbar_wait(bar_vempty(vs), ((gj / VST) + 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar_vfull(vs), LY::VBYTES);
          uint8_t* vdst = smem + LY::OFF_V + vs * LY::VBYTES;
          if constexpr (LAY == PAIR_DENSE) {
#pragma unroll
            for (int x = 0; x < D / 64; ++x)
              tma_load_3d(smem_addr(vdst + x * BN * 128), &tmv, bar_vfull(vs), x * 64, kb * BN,
                          T.b * P.Hkv + T.g);
          } else {
            tma_load_kv<D, BN>(P, &tmv, vdst, bar_vfull(vs), T.b, T.g, kb, T.s);
          }
        }
        g0 += T.nblk;
        ++tq;
      }
    } else if (warp == 9 && lane == 0) {
      // ======================= MMA issuer ===================================
      constexpr uint32_t IDESC_S = idesc_bf16(TC_BM, BN, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16(TC_BM, D, 0, 1);
      auto issue_qk = [&](int t, int gj) {
        const uint32_t qbase = smem_addr(smem + LY::OFF_Q + t * LY::QBYTES);
        const uint32_t kbase = smem_addr(smem + LY::OFF_K + (gj % KST) * LY::KBYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad =
              sdesc_sw128(qbase + (kk >> 2) * TC_BM * 128 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(kbase + (kk >> 2) * BN * 128 + (kk & 3) * 32, 16, 1024);
          umma_ss(tmem + LY::TM_S + t * BN, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_sfull(t));
      };
      int g0 = 0, tq = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int rank = pair_rank(round, cta, G);
        if (rank >= (SORTED ? nwalk : ntiles)) break;
        const PairTile T = SORTED ? tile_of(rank) : pair_tile<LAY>(P, rank);
        const int nblk = T.nblk;
        if (nblk == 0) continue;
        ok = mbar_wait_busy(bar_q, tq & 1, abort_flag);
        tc_fence_after();
        // prologue: both tiles' scores of the first block (S of either tile
        // held the previous tile's last P, whose PV was issued before)
        if (ok && mbar_wait_busy(bar_kfull(g0 % KST), (g0 / KST) & 1, abort_flag)) {
          tc_fence_after();
          issue_qk(0, g0);
          issue_qk(1, g0);
          umma_commit(bar_kempty(g0 % KST));
          if (nblk == 1) umma_commit(bar_qempty);
        } else {
          ok = false;
        }
        for (int j = 0; ok && j < nblk; ++j) {
          const int gj = g0 + j;
          const int vs = gj % VST;
          if (!mbar_wait_busy(bar_vfull(vs), (gj / VST) & 1, abort_flag)) {
            ok = false;
            break;
          }
          bool k_next = false;
          for (int t = 0; t < 2; ++t) {
            if (!mbar_wait_busy(bar_pfull(t), gj & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t vbase = smem_addr(smem + LY::OFF_V + vs * LY::VBYTES);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              // V block [BN keys][D] in 64-column boxes: MN-major B operand
              const uint64_t bd = sdesc_sw128(vbase + kk * 16 * 128, BN * 128, 1024);
              umma_ts(tmem + LY::TM_O + t * D, tmem + LY::TM_S + t * BN + kk * 8, bd, IDESC_O,
                      (j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(bar_pv(t));
            if (t == 1) umma_commit(bar_vempty(vs));
            if (j + 1 < nblk) {
              // this tile's next scores go in behind its PV (issue order)
              if (t == 0) {
                if (!mbar_wait_busy(bar_kfull((gj + 1) % KST), ((gj + 1) / KST) & 1,
                                    abort_flag)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                k_next = true;
              }
              issue_qk(t, gj + 1);
              if (t == 1 && k_next) {
                umma_commit(bar_kempty((gj + 1) % KST));
                if (j + 2 == nblk) umma_commit(bar_qempty);
              }
            }
          }
        }
        g0 += nblk;
        ++tq;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, LY::TM_COLS);
}

}  // namespace nattn
