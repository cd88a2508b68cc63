// Sparse prefill for rows whose support is too wide for the threshold pass's
// candidate buffers (tcgen05 + TMEM + TMA).
//
// The threshold pass lists every 128-row tile in which some row overflowed
// its buffer.  This kernel takes one such tile per CTA and finds the exact
// threshold of each overflowed row from its full score row, without any
// buffer: Newton's method from the left on the convex, decreasing
// g(t) = sum relu(u - t)^k - 1 (k = 1 sparsemax, k = 2 1.5-entmax), one pass
// over the row's key blocks per iteration, each pass accumulating the count,
// sum and sum of squares of the scores above the current iterate (the
// iteration of tau_step; every iterate is a lower bound of the threshold, and the closed-form threshold of the set above it is
// accepted once it satisfies the optimality conditions).  The iteration
// starts from the lower bound the bound pass found.  When every overflowed
// row of the tile has converged, one more pass forms the exact weights
// p = relu(u - tau)^k in bf16 over the S columns in TMEM and multiplies them
// by V on the tensor cores ("HF Attention Normalizers", section "Important
// Limitations": the sparse kernels stream K/V tiles, solve the global
// normalization threshold and save one threshold per query row).  Its cost
// does not depend on the support's width.  A row that has not converged
// after WIDE_PASSES iterations is listed for the row-wise kernel.
//
// Warp roles and TMEM layout are those of the single-tile online kernel: the
// normalizer warps (each S row split between two warps for d <= 128), a TMA
// producer and an MMA issuer; two S buffers and one O accumulator per row
// half.
#pragma once

#include "prefill_tc.cuh"

namespace nattn {

constexpr int WIDE_PASSES = 12;  // Newton passes at most

template <int D, int BN, int NH>
struct WideLayout {
  static constexpr int NWN = 4 * NH;
  static constexpr int THREADS = (NWN + 2) * 32;
  static constexpr int KST = 2, VST = 2, NSB = 2;
  static constexpr int NC = BN / NH;  // S columns per normalizer thread
  static constexpr int QBYTES = D * TC_BM * 2;
  static constexpr int KBYTES = D * BN * 2;
  static constexpr int VBYTES = D * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + KST * KBYTES;
  // per-pass partial sums of the row halves, double-buffered by pass
  static constexpr int OFF_XCH = OFF_V + VST * VBYTES;
  static constexpr int XCHBYTES = 2 * NH * TC_BM * 16;
  static constexpr int OFF_BAR = OFF_XCH + XCHBYTES;
  // q, kfull/kempty, vfull/vempty, sfull/pfull, pv, the pass decision, the
  // halves' sums of a pass
  static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 2 * NSB + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // misc: TMEM base, abort flag, tile-wide flags, then one counter per pass
  // of the rows that have not converged
  static constexpr int BYTES = OFF_MISC + 16 + 4 * (WIDE_PASSES + 1);
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int TM_S = 0;
  static constexpr int TM_O = NSB * BN;
  static constexpr int TM_COLS_USED = NSB * BN + NH * D;
  static constexpr int TM_COLS = TM_COLS_USED <= 256 ? 256 : 512;
  static_assert(TM_COLS_USED <= 512, "TMEM budget");
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(NC == 64, "each normalizer thread owns 64 columns of a block");
};

template <int D, int BN, int NH>
__global__ void __launch_bounds__((4 * NH + 2) * 32, 1)
    prefill_wide_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, TcArgs A) {
  using LY = WideLayout<D, BN, NH>;
  constexpr int NWN = LY::NWN, NC = LY::NC, NSB = LY::NSB, KST = LY::KST, VST = LY::VST;
  constexpr int DV = D;
  // one CTA per SM walks the tiles the threshold pass listed
  const int ntile = *A.wide_count;
  if ((int)blockIdx.x >= ntile) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Problem& P = A.P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + LY::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);
  // notconv[p]: normalizer warps with an overflowed row still iterating
  // after Newton pass p
  int* notconv = reinterpret_cast<int*>(&misc[4]);
  if (tid == 0) *abort_flag = 0;
  if (warp == NWN + 1) {
    tmem_alloc(smem_addr(&misc[0]), LY::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  for (int ti = blockIdx.x; ti < ntile; ti += gridDim.x) {
  // ---- the tile: the threshold pass's rank of it ---------------------------
  const int ntq = (P.Tq + TC_BM - 1) / TC_BM;
  const int BH = P.B * P.Hq;
  const int rank = A.wide_tiles[ti];
  const int qt = P.causal ? (ntq - 1 - rank / BH) : (rank / BH);
  const int bh = rank % BH;
  const int b = bh / P.Hq, h = bh % P.Hq;
  const int g = h / (P.Hq / P.Hkv);
  const int q0 = qt * TC_BM;
  const SeqInfo sq = seq_info(P, b);
  const bool packed = P.cu_q != nullptr;
  const int qlast = min(q0 + TC_BM - 1, sq.Lq - 1);
  const RowRange r_first = row_range(sq.Lq, P.causal, P.window, q0, sq.Lk);
  const RowRange r_last = row_range(sq.Lq, P.causal, P.window, qlast, sq.Lk);
  const int klo = max(0, r_first.lo);
  const int khi = (q0 < sq.Lq) ? min(sq.Lk - 1, r_last.hi) : -1;
  const int kb0 = klo / BN;
  const int kend = (khi >= klo) ? khi / BN + 1 : kb0;
  const int nblk = count_kept<BN>(P, b, h, h, qt, kb0, kend);

  const uint32_t bar_q = smem_addr(&bars[0]);
  auto bar_kfull = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto bar_kempty = [&](int s) { return smem_addr(&bars[1 + KST + s]); };
  auto bar_vfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + s]); };
  auto bar_vempty = [&](int s) { return smem_addr(&bars[1 + 2 * KST + VST + s]); };
  auto bar_sfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + s]); };
  auto bar_pfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + NSB + s]); };
  const uint32_t bar_pv = smem_addr(&bars[1 + 2 * KST + 2 * VST + 2 * NSB]);
  // the normalizer warps' decision after each Newton pass (one arrival each)
  const uint32_t bar_dec = smem_addr(&bars[2 + 2 * KST + 2 * VST + 2 * NSB]);
  // both halves of every row have published their sums of a Newton pass (an
  // mbarrier with a bounded wait, not a named barrier: a warp that gives up
  // on a wait leaves the others a bounded wait too)
  const uint32_t bar_x = smem_addr(&bars[3 + 2 * KST + 2 * VST + 2 * NSB]);

  // every barrier of the previous tile is idle (its last operations were
  // waited for before the closing __syncthreads)
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
    mbar_init(bar_dec, NWN);
    mbar_init(bar_x, NWN);
    for (int p = 0; p <= WIDE_PASSES; ++p) notconv[p] = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // Whether pass p (p >= 1) forms the weights: every row has converged after
  // Newton pass p - 1, or the Newton passes are used up.  The decision of
  // pass p - 1 is complete once all normalizer warps have arrived on bar_dec
  // for it (phase (p - 1) & 1).
  auto apply_pass = [&](int p, bool& ok) -> bool {
    if (p == 0) return false;
    ok = ok && mbar_wait(bar_dec, (p - 1) & 1, abort_flag);
    return p == WIDE_PASSES || *reinterpret_cast<volatile int*>(&notconv[p - 1]) == 0;
  };

  if (warp == NWN) {
    // ======================= TMA producer ===================================
    if (lane == 0 && nblk > 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      mbar_expect_tx(bar_q, LY::QBYTES);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_rows(smem_addr(smem + LY::OFF_Q + x * TC_BM * 128), &tmq, bar_q, x * 64,
                      packed ? sq.q0 + q0 : q0, packed ? h : bh, packed);
      bool ok = true, applied = false;
      int J = 0;  // K blocks loaded over all passes
      for (int p = 0; ok; ++p) {
        const bool apply = apply_pass(p, ok);
        if (!ok) break;
        applied = apply;
        int kb = next_kept<BN>(P, b, h, h, qt, kb0, kend);
        for (int j = 0; j < nblk; ++j, ++J, kb = next_kept<BN>(P, b, h, h, qt, kb + 1, kend)) {
          const int ks = J % KST;
          if (J >= KST && !mbar_wait(bar_kempty(ks), ((J / KST) + 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar_kfull(ks), LY::KBYTES);
          tma_load_kv<D, BN>(P, &tmk, smem + LY::OFF_K + ks * LY::KBYTES, bar_kfull(ks), b, g,
                             kb, sq);
          if (apply) {
            const int vs = j % VST;
            if (j >= VST && !mbar_wait(bar_vempty(vs), ((j / VST) + 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            mbar_expect_tx(bar_vfull(vs), LY::VBYTES);
            tma_load_kv<DV, BN>(P, &tmv, smem + LY::OFF_V + vs * LY::VBYTES, bar_vfull(vs), b,
                                g, kb, sq);
          }
        }
        if (apply) break;
      }
      // drain: the last loads' slots released (their commits have landed)
      // before the barriers are initialized again for the next tile
      for (int L = max(0, J - KST); ok && L < J; ++L)
        ok = mbar_wait(bar_kempty(L % KST), (L / KST) & 1, abort_flag);
      for (int jv = max(0, nblk - VST); ok && applied && jv < nblk; ++jv)
        ok = mbar_wait(bar_vempty(jv % VST), (jv / VST) & 1, abort_flag);
    }
  } else if (warp == NWN + 1) {
    // ======================= MMA issuer =====================================
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(TC_BM, BN, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16(TC_BM, DV, 0, 1);
      const uint32_t qbase = smem_addr(smem + LY::OFF_Q);
      bool ok = mbar_wait_spin(bar_q, 0, abort_flag);
      tc_fence_after();
      int J = 0;  // S tiles over all passes
      // PV of block jp of the weight pass (S tile J - 1)
      auto issue_pv = [&](int jp, int Jp) -> bool {
        const int sbp = Jp % NSB, vs = jp % VST;
        if (!mbar_wait_spin(bar_pfull(sbp), (Jp / NSB) & 1, abort_flag)) return false;
        if (!mbar_wait_spin(bar_vfull(vs), (jp / VST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_addr(smem + LY::OFF_V + vs * LY::VBYTES);
        const uint32_t pt = tmem + LY::TM_S + sbp * BN;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
#pragma unroll
          for (int kk = 0; kk < NC / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(vbase + (hh * NC + kk * 16) * 128, BN * 128, 1024);
            umma_ts(tmem + LY::TM_O + hh * DV, pt + hh * NC + kk * 8, bd, IDESC_O,
                    (jp > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(bar_vempty(vs));
        umma_commit(bar_pv);
        return true;
      };
      for (int p = 0; ok; ++p) {
        const bool apply = apply_pass(p, ok);
        if (!ok) break;
        for (int j = 0; j < nblk; ++j, ++J) {
          const int sb = J % NSB, ks = J % KST;
          if (!mbar_wait_spin(bar_kfull(ks), (J / KST) & 1, abort_flag)) {
            ok = false;
            break;
          }
          // the normalizer warps are done with S tile J - NSB (read, or its
          // weights stored and, in the weight pass, multiplied: that product
          // was issued by this thread before this QK)
          if (J >= NSB && !mbar_wait_spin(bar_pfull(sb), ((J - NSB) / NSB) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kbase = smem_addr(smem + LY::OFF_K + ks * LY::KBYTES);
          const uint32_t sdst = tmem + LY::TM_S + sb * BN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad =
                sdesc_sw128(qbase + (kk >> 2) * TC_BM * 128 + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kbase + (kk >> 2) * BN * 128 + (kk & 3) * 32, 16, 1024);
            umma_ss(sdst, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_sfull(sb));
          umma_commit(bar_kempty(ks));
          if (apply && j >= 1 && !issue_pv(j - 1, J - 1)) {
            ok = false;
            break;
          }
        }
        if (apply) {
          if (ok) ok = issue_pv(nblk - 1, J - 1);
          break;
        }
      }
    }
  } else {
    // ======================= normalizer warps ==============================
    const int quarter = warp & 3;  // TMEM lane quarter = query rows
    const int half = warp >> 2;    // which columns of the S row
    const int cbase = half * NC;
    const int row = quarter * 32 + lane;
    const int qi = q0 + row;
    const bool row_ok = qi < sq.Lq;
    RowRange rr = row_range(sq.Lq, P.causal, P.window, qi, sq.Lk);
    if (!row_ok) rr = RowRange{1, 0};
    if (rr.hi > sq.Lk - 1) rr.hi = sq.Lk - 1;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const size_t flat = row_index(P, b, h, qi, sq);
    const bool fast = !(P.softcap > 0.f) && A.zscale > 0.f;
    const bool entmax = P.norm == NATTN_ENTMAX15;
    // this row is one the threshold pass could not finish
    const bool wide = row_ok && A.sup_count[flat * NH] < 0;
    // row maximum (threshold units) and the iterate, less the maximum
    const float m = wide ? A.tau[flat] : 0.f;
    float t = wide ? fmaxf(A.rlb[flat], -1.f) : 0.f;
    bool conv = !wide;  // converged (or not iterating at all)
    bool alive = nblk > 0;
    int nnz = 0;

    // Wait for S tile J and load this thread's 64 scores of key block kbc in
    // threshold units less the row maximum; masked entries become -inf
    auto load_w = [&](int J, int kbc, float (&w)[64]) -> bool {
      const int sb = J % NSB;
      if (!__all_sync(0xffffffffu, mbar_wait_spin(bar_sfull(sb), (J / NSB) & 1, abort_flag)))
        return false;
      tc_fence_after();
      const int jb = kbc * BN + cbase;
      const bool edge = !(rr.lo <= jb && rr.hi >= jb + NC - 1);
      int klb = rr.lo - jb;
      unsigned span = (unsigned)(rr.hi - rr.lo);
      if (rr.hi < rr.lo) {
        klb = NC;
        span = 0;
      }
      uint32_t r[64];
      const uint32_t saddr = lane_base + LY::TM_S + sb * BN + cbase;
      tmem_ld32(saddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(saddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld_wait();
      if (fast) {
#pragma unroll
        for (int k = 0; k < 64; ++k) w[k] = fmaf(__uint_as_float(r[k]), A.zscale, -m);
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) w[k] = tc_z(__uint_as_float(r[k]), A) - m;
      }
      if (edge) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if ((unsigned)(k - klb) > span) w[k] = -INFINITY;
      }
      return true;
    };
    auto release = [&](int J) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull(J % NSB));
    };
    const int kfirst = next_kept<BN>(P, b, h, h, qt, kb0, kend);
    float4* const xch = reinterpret_cast<float4*>(smem + LY::OFF_XCH);

    int J = 0;
    bool apply = false;
    for (int p = 0; alive; ++p) {
      if (p > 0) {
        alive = mbar_wait(bar_dec, (p - 1) & 1, abort_flag);
        apply = p == WIDE_PASSES || *reinterpret_cast<volatile int*>(&notconv[p - 1]) == 0;
        if (!alive) break;
      }
      float cnt = 0.f, s1 = 0.f, s2 = 0.f, wmin = INFINITY;
      int kbc = kfirst;
      for (int j = 0; j < nblk; ++j, ++J, kbc = next_kept<BN>(P, b, h, h, qt, kbc + 1, kend)) {
        float w[64];
        if (!load_w(J, kbc, w)) {
          alive = false;
          break;
        }
        if (!apply) {
          // Newton pass: the statistics of the scores above the iterate
          if (!conv) {
#pragma unroll
            for (int k = 0; k < 64; ++k) {
              if (w[k] > t) {
                cnt += 1.f;
                s1 += w[k];
                s2 = fmaf(w[k], w[k], s2);
                wmin = fminf(wmin, w[k]);
              }
            }
          }
        } else {
          // weight pass: p = relu(w - tau)^k as bf16 pairs over this thread's
          // own S columns, once the previous block's PV has completed
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 64; k += 2) {
            float x0 = wide ? w[k] - t : 0.f, x1 = wide ? w[k + 1] - t : 0.f;
            nnz += (x0 > 0.f) + (x1 > 0.f);
            x0 = fmaxf(x0, 0.f);
            x1 = fmaxf(x1, 0.f);
            if (entmax) {
              x0 *= x0;
              x1 *= x1;
            }
            pk[k / 2] = pack_bf16(x0, x1);
          }
          if (j > 0 && !__all_sync(0xffffffffu, mbar_wait_spin(bar_pv, (j - 1) & 1, abort_flag))) {
            alive = false;
            break;
          }
          tc_fence_after();
          tmem_st32(lane_base + LY::TM_S + (J % NSB) * BN + cbase, pk);
          tmem_st_wait();
        }
        release(J);
      }
      if (!alive || apply) break;
      // the row's sums over both halves (double-buffered by pass parity: the
      // writes of pass p + 2 follow the completion of pass p + 1's exchange,
      // which every warp reaches only after reading pass p's)
      float4 mine = make_float4(cnt, s1, s2, wmin);
      if constexpr (NH > 1) {
        xch[((p & 1) * NH + half) * TC_BM + row] = mine;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_x);
        if (!__all_sync(0xffffffffu, mbar_wait(bar_x, p & 1, abort_flag))) {
          alive = false;
          break;
        }
        const float4 o = xch[((p & 1) * NH + (1 - half)) * TC_BM + row];
        // the same order in both halves: the iterate stays identical
        const float4 a0 = half == 0 ? mine : o, a1 = half == 0 ? o : mine;
        mine = make_float4(a0.x + a1.x, a0.y + a1.y, a0.z + a1.z, fminf(a0.w, a1.w));
      }
      // (a step that cannot move t leaves it at the root within rounding:
      // g(t) >= 0 at every iterate, and the Newton step is g / |g'|)
      if (!conv) conv = tau_step(mine.x, mine.y, mine.z, mine.w, entmax, t) != 0;
      // one vote per warp for another Newton pass, then the decision
      if (__any_sync(0xffffffffu, !conv) && lane == 0) atomicAdd(&notconv[p], 1);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dec);
    }

    // ---- epilogue: the overflowed rows of the tile --------------------------
    const bool have_o =
        __all_sync(0xffffffffu, alive && apply && mbar_wait(bar_pv, (nblk - 1) & 1, abort_flag));
    tc_fence_after();
    int nnz_row = nnz;
    if constexpr (NH > 1) {
      float4* x2 = reinterpret_cast<float4*>(smem + LY::OFF_XCH);
      asm volatile("bar.sync 1, %0;" ::"r"(NWN * 32) : "memory");
      x2[half * TC_BM + row] = make_float4(__int_as_float(nnz), 0.f, 0.f, 0.f);
      asm volatile("bar.sync 1, %0;" ::"r"(NWN * 32) : "memory");
      nnz_row = __float_as_int(x2[row].x) + __float_as_int(x2[TC_BM + row].x);
    }
    // rows still iterating after the last Newton pass go to the row-wise pass
    const bool solved = wide && conv;
    if (wide && !solved && half == 0) {
      const int slot = atomicAdd(A.ovf_count, 1);
      A.ovf_rows[slot] = (int)flat;
    }
    // this thread writes output columns [half * DV / NH, (half + 1) * DV / NH)
    constexpr int OC = DV / NH;
    bf16* orow = P.out + flat * DV + half * OC;
    const uint32_t oaddr = lane_base + LY::TM_O + half * OC;
#pragma unroll 1
    for (int c = 0; c < OC / 32; ++c) {
      uint32_t r0[32], r1[32];
      if (have_o) {
        tmem_ld32(oaddr + c * 32, r0);
        if constexpr (NH > 1) tmem_ld32(oaddr + DV + c * 32, r1);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) r0[k] = r1[k] = 0u;
      }
      if (solved) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
          float o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            o[e] = __uint_as_float(r0[k + e]);
            if constexpr (NH > 1) o[e] += __uint_as_float(r1[k + e]);
          }
          uint4 v;
          v.x = pack_bf16(o[0], o[1]);
          v.y = pack_bf16(o[2], o[3]);
          v.z = pack_bf16(o[4], o[5]);
          v.w = pack_bf16(o[6], o[7]);
          dst[k / 8] = v;
        }
      }
    }
    if (solved && half == 0) {
      if (P.row_stat) P.row_stat[flat] = m + t;
      if (P.row_nnz) P.row_nnz[flat] = nnz_row;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  }  // tiles

  if (warp == NWN + 1) tmem_dealloc(tmem, LY::TM_COLS);
}

}  // namespace nattn
