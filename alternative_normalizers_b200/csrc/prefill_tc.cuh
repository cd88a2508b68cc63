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
//   TAU     sparse phase 1: S only.  Each row streams its scores once and
//           keeps a small buffer of the only entries that can still be in the
//           support (those above a running lower bound of tau); the exact
//           threshold is solved on that buffer at the end ("HF Attention
//           Normalizers", section "Important Limitations": the sparse kernels
//           stream K/V tiles, solve the global normalization threshold and
//           save one threshold per query row).  Rows whose candidates
//           overflow the buffer are listed for the row-wise kernel.
//   APPLY   sparse phase 2: p = relu(z - tau) or relu(z/2 - tau)^2 with tau
//           fixed, O += P V; no maximum, no division, no rescale.
#pragma once

#include "common.cuh"
#include "problem.cuh"

namespace nattn {

enum TcMode { TC_ONLINE = 0, TC_TAU = 1, TC_APPLY = 2 };

constexpr int TC_THREADS = 192;
constexpr int TC_BM = 128;
constexpr int TAU_CAP = 128;  // candidate buffer entries per row

struct TcArgs {
  Problem P;
  float zscale;      // ONLINE: scale * log2(e); TAU/APPLY: scale * uscale
  float capscale;    // soft-cap: z = capscale * tanh(s * scale / cap)
  float* tau;        // [B*Hq*Tq]: written by TAU, read by APPLY
  int* ovf_rows;     // TAU: rows whose candidate buffer overflowed
  int* ovf_count;    // TAU: number of such rows (zeroed before the launch)
};

template <int D, int DV, int BN, int KST, int VST, int MODE>
struct TcLayout {
  static constexpr int QBYTES = D * TC_BM * 2;
  static constexpr int KBYTES = D * BN * 2;
  static constexpr int VBYTES = (MODE == TC_TAU) ? 0 : DV * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + KST * KBYTES;
  static constexpr int OFF_BUF = OFF_V + VST * VBYTES;
  static constexpr int BUFBYTES = (MODE == TC_TAU) ? TAU_CAP * TC_BM * 4 : 0;
  static constexpr int OFF_BAR = OFF_BUF + BUFBYTES;
  static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
  // TMEM columns: S double buffer, then O
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = BN;
  static constexpr int TM_O = 2 * BN;
  static constexpr int TM_COLS_USED = (MODE == TC_TAU) ? 2 * BN : 2 * BN + DV;
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

// Per-thread exact threshold over the candidate buffer (values in threshold
// units u).  Same method as the block-level solver of the row-wise kernel:
// Newton from the left on g(t) = sum relu(u - t)^k, accepting the closed-form
// threshold of {u > t} once it satisfies the optimality conditions.
// `t0` is a lower bound of tau in shifted units (u - m).  With `newton_only`
// it returns after `iters` Newton steps (a valid lower bound, for pruning).
__device__ __forceinline__ float thread_tau(const float* buf, int n, float m, bool entmax,
                                            float t0, int iters, bool newton_only) {
  float t = fmaxf(t0, -1.f);
  for (int it = 0; it < iters; ++it) {
    float cnt = 0.f, s1 = 0.f, s2 = 0.f, wmin = INFINITY;
    for (int k = 0; k < n; ++k) {
      const float w = buf[k * TC_BM] - m;
      if (w > t) {
        cnt += 1.f;
        s1 += w;
        s2 += w * w;
        wmin = fminf(wmin, w);
      }
    }
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
    if (!newton_only && valid && ts >= t && wmin > ts) return ts + m;
    if (!(tn > t)) break;
    t = tn;
  }
  return t + m;
}

template <int D, int DV, int BN, int KST, int VST, int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, TcArgs A) {
  using LY = TcLayout<D, DV, BN, KST, VST, MODE>;
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
  const int qlast = min(q0 + TC_BM - 1, P.Tq - 1);
  const RowRange r_first = row_range(P, q0, P.Tk);
  const RowRange r_last = row_range(P, qlast, P.Tk);
  const int klo = max(0, r_first.lo);
  const int khi = min(P.Tk - 1, r_last.hi);
  const int kb0 = klo / BN;
  const int nblk = (khi >= klo) ? (khi / BN - kb0 + 1) : 0;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::OFF_BAR);
  const uint32_t bar_q = smem_addr(&bars[0]);
  auto bar_kfull = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto bar_kempty = [&](int s) { return smem_addr(&bars[1 + KST + s]); };
  auto bar_vfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + s]); };
  auto bar_vempty = [&](int s) { return smem_addr(&bars[1 + 2 * KST + VST + s]); };
  auto bar_sfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + s]); };
  auto bar_pfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + 2 + s]); };
  const uint32_t bar_pv = smem_addr(&bars[1 + 2 * KST + 2 * VST + 4]);
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
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_sfull(s), 1);
      mbar_init(bar_pfull(s), 128);
    }
    mbar_init(bar_pv, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(&misc[0]), LY::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 4) {
    // ======================= TMA producer ===================================
    if (lane == 0 && nblk > 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      if (MODE != TC_TAU) tma_prefetch_desc(&tmv);
      mbar_expect_tx(bar_q, LY::QBYTES);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_addr(smem + LY::OFF_Q + x * TC_BM * 128), &tmq, bar_q, x * 64, q0,
                    bh);
      for (int j = 0; j < nblk; ++j) {
        const int kb = kb0 + j;
        const int ks = j % KST;
        if (j >= KST && !mbar_wait(bar_kempty(ks), ((j / KST) + 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_kfull(ks), LY::KBYTES);
        uint8_t* kdst = smem + LY::OFF_K + ks * LY::KBYTES;
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
          tma_load_3d(smem_addr(kdst + x * BN * 128), &tmk, bar_kfull(ks), x * 64, kb * BN,
                      b * P.Hkv + g);
        if constexpr (MODE != TC_TAU) {
          const int vs = j % VST;
          if (j >= VST && !mbar_wait(bar_vempty(vs), ((j / VST) + 1) & 1, abort_flag))
            break;
          mbar_expect_tx(bar_vfull(vs), LY::VBYTES);
          uint8_t* vdst = smem + LY::OFF_V + vs * LY::VBYTES;
#pragma unroll
          for (int x = 0; x < DV / 64; ++x)
            tma_load_3d(smem_addr(vdst + x * BN * 128), &tmv, bar_vfull(vs), x * 64,
                        kb * BN, b * P.Hkv + g);
        }
      }
    }
  } else if (warp == 5) {
    // ======================= MMA issuer =====================================
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(TC_BM, BN, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16(TC_BM, DV, 0, 1);
      const uint32_t qbase = smem_addr(smem + LY::OFF_Q);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      tc_fence_after();
      for (int j = 0; ok && j <= nblk; ++j) {
        if (j < nblk) {
          const int sb = j & 1, ks = j % KST;
          if (!mbar_wait(bar_kfull(ks), (j / KST) & 1, abort_flag)) break;
          if (j >= 2) {
            // S buffer sb is free once P_{j-2} has been consumed
            if constexpr (MODE == TC_TAU) {
              if (!mbar_wait(bar_pfull(sb), ((j - 2) / 2) & 1, abort_flag)) break;
            } else {
              if (!mbar_wait(bar_pv, (j - 2) & 1, abort_flag)) break;
            }
          }
          tc_fence_after();
          const uint32_t kbase = smem_addr(smem + LY::OFF_K + ks * LY::KBYTES);
          const uint32_t sdst = tmem + (sb ? LY::TM_S1 : LY::TM_S0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad =
                sdesc_sw128(qbase + (kk >> 2) * TC_BM * 128 + (kk & 3) * 32, 16, 1024);
            const uint64_t bd =
                sdesc_sw128(kbase + (kk >> 2) * BN * 128 + (kk & 3) * 32, 16, 1024);
            umma_ss(sdst, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_sfull(sb));
          umma_commit(bar_kempty(ks));
        }
        if constexpr (MODE != TC_TAU) {
          if (j >= 1) {
            const int jp = j - 1, sbp = jp & 1, vs = jp % VST;
            if (!mbar_wait(bar_pfull(sbp), (jp / 2) & 1, abort_flag)) break;
            if (!mbar_wait(bar_vfull(vs), (jp / VST) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t vbase = smem_addr(smem + LY::OFF_V + vs * LY::VBYTES);
            const uint32_t pt = tmem + (sbp ? LY::TM_S1 : LY::TM_S0);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              // V block is [BN keys][DV] in 64-column boxes: MN-major B
              // operand, LBO = box stride, SBO = 8 key rows.
              const uint64_t bd = sdesc_sw128(vbase + kk * 16 * 128, BN * 128, 1024);
              umma_ts(tmem + LY::TM_O, pt + kk * 8, bd, IDESC_O,
                      (jp > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(bar_vempty(vs));
            umma_commit(bar_pv);
          }
        }
      }
    }
  } else {
    // ======================= normalizer warps (0-3) ========================
    const int row = warp * 32 + lane;
    const int qi = q0 + row;
    const bool row_ok = qi < P.Tq;
    RowRange rr = row_range(P, qi, P.Tk);
    if (!row_ok) rr = RowRange{1, 0};
    if (rr.hi > P.Tk - 1) rr.hi = P.Tk - 1;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const size_t flat = ((size_t)bh * P.Tq + qi);

    float m_run, l_run = 0.f, tau = 0.f;
    // TAU state
    float* buf = reinterpret_cast<float*>(smem + LY::OFF_BUF) + row;
    int nbuf = 0;
    bool ovf = false;
    float lb = -INFINITY;  // lower bound of tau (threshold units)
    if constexpr (MODE == TC_ONLINE) {
      m_run = (P.norm == NATTN_SOFTMAX1) ? 0.f : -INFINITY;
      l_run = (P.norm == NATTN_SOFTMAX1) ? 1.f : 0.f;
    } else {
      m_run = -INFINITY;
    }
    if constexpr (MODE == TC_APPLY) tau = row_ok ? A.tau[flat] : INFINITY;
    const bool entmax = P.norm == NATTN_ENTMAX15;
    bool alive = true;

    for (int j = 0; j < nblk; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_sfull(sb), (j / 2) & 1, abort_flag))) {
        alive = false;
        break;
      }
      tc_fence_after();
      const int j0 = (kb0 + j) * BN;
      const bool edge = !(rr.lo <= j0 && rr.hi >= j0 + BN - 1);
      const uint32_t saddr = lane_base + (sb ? LY::TM_S1 : LY::TM_S0);

      if constexpr (MODE == TC_ONLINE) {
        // pass 1: row maximum of this block
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(saddr + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            float z = tc_z(__uint_as_float(r[k]), A);
            if (edge) {
              const int jj = j0 + c * 32 + k;
              z = (jj >= rr.lo && jj <= rr.hi) ? z : -INFINITY;
            }
            mx = fmaxf(mx, z);
          }
        }
        const float mnew = fmaxf(m_run, mx);
        const bool resc = mnew > m_run + 8.f;
        const float m_use = resc ? mnew : m_run;
        const float alpha = resc ? fast_exp2(m_run - mnew) : 1.f;
        const float msafe = (m_use == -INFINITY) ? 0.f : m_use;
        // pass 2: weights, row sum, bf16 P into the S columns
        float sum = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(saddr + c * 32, r);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            float z0 = tc_z(__uint_as_float(r[k]), A);
            float z1 = tc_z(__uint_as_float(r[k + 1]), A);
            if (edge) {
              const int jj = j0 + c * 32 + k;
              z0 = (jj >= rr.lo && jj <= rr.hi) ? z0 : -INFINITY;
              z1 = (jj + 1 >= rr.lo && jj + 1 <= rr.hi) ? z1 : -INFINITY;
            }
            const float p0 = fast_exp2(z0 - msafe);
            const float p1 = fast_exp2(z1 - msafe);
            sum += p0 + p1;
            pk[k >> 1] = pack_bf16(p0, p1);
          }
          tmem_st16(saddr + c * 16, pk);
        }
        tmem_st_wait();
        l_run = l_run * alpha + sum;
        // rescale O when the maximum moved (warp-uniform TMEM access)
        if (__any_sync(0xffffffffu, resc) && j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar_pv, (j - 1) & 1, abort_flag))) {
            alive = false;
            break;
          }
          tc_fence_after();
          const uint32_t oaddr = lane_base + LY::TM_O;
#pragma unroll 1
          for (int c = 0; c < DV / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(oaddr + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
            tmem_st32(oaddr + c * 32, r);
          }
          tmem_st_wait();
        }
        m_run = m_use;
      } else if constexpr (MODE == TC_APPLY) {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(saddr + c * 32, r);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            float x0 = fmaxf(tc_z(__uint_as_float(r[k]), A) - tau, 0.f);
            float x1 = fmaxf(tc_z(__uint_as_float(r[k + 1]), A) - tau, 0.f);
            if (entmax) {
              x0 *= x0;
              x1 *= x1;
            }
            if (edge) {
              const int jj = j0 + c * 32 + k;
              x0 = (jj >= rr.lo && jj <= rr.hi) ? x0 : 0.f;
              x1 = (jj + 1 >= rr.lo && jj + 1 <= rr.hi) ? x1 : 0.f;
            }
            pk[k >> 1] = pack_bf16(x0, x1);
          }
          tmem_st16(saddr + c * 16, pk);
        }
        tmem_st_wait();
      } else {  // TC_TAU
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(saddr + c * 32, r);
          tmem_ld_wait();
          float u[32];
          float cmax = -INFINITY;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            float z = tc_z(__uint_as_float(r[k]), A);
            if (edge) {
              const int jj = j0 + c * 32 + k;
              z = (jj >= rr.lo && jj <= rr.hi) ? z : -INFINITY;
            }
            u[k] = z;
            cmax = fmaxf(cmax, z);
          }
          m_run = fmaxf(m_run, cmax);
          lb = fmaxf(lb, m_run - 1.f);  // tau >= max - 1
          if (cmax > lb && !ovf) {
            if (nbuf + 32 > TAU_CAP) {
              // raise the lower bound with a few Newton steps, then compact
              lb = thread_tau(buf, nbuf, m_run, entmax, lb - m_run, 4, true);
              int w = 0;
              for (int k = 0; k < nbuf; ++k) {
                const float x = buf[k * TC_BM];
                if (x > lb) buf[(w++) * TC_BM] = x;
              }
              nbuf = w;
            }
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              if (u[k] > lb) {
                if (nbuf < TAU_CAP) {
                  buf[nbuf * TC_BM] = u[k];
                  ++nbuf;
                } else {
                  ovf = true;
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_pfull(sb));
    }

    // ---- epilogue ----------------------------------------------------------
    if constexpr (MODE == TC_TAU) {
      if (row_ok) {
        float t = INFINITY;
        if (ovf) {
          const int slot = atomicAdd(A.ovf_count, 1);
          A.ovf_rows[slot] = (int)flat;
        } else if (m_run != -INFINITY) {
          t = thread_tau(buf, nbuf, m_run, entmax, lb - m_run, 64, false);
        }
        A.tau[flat] = t;
      }
    } else {
      const bool have_o =
          __all_sync(0xffffffffu, alive && nblk > 0 &&
                                      mbar_wait(bar_pv, (nblk - 1) & 1, abort_flag));
      tc_fence_after();
      float inv = 1.f, stat = tau;
      if constexpr (MODE == TC_ONLINE) {
        inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
        const float msafe = (m_run == -INFINITY) ? 0.f : m_run;
        stat = (l_run > 0.f) ? (msafe + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      }
      bf16* orow = P.out + flat * DV;
      const uint32_t oaddr = lane_base + LY::TM_O;
#pragma unroll 1
      for (int c = 0; c < DV / 32; ++c) {
        uint32_t r[32];
        if (have_o) {
          tmem_ld32(oaddr + c * 32, r);
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
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, LY::TM_COLS);
}

}  // namespace nattn
