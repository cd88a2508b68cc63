// Backward pass of the attention forward on the 5th-generation tensor cores.
//
// The forward keeps one statistic per query row (the log-sum-exp for the
// softmax family, the threshold tau for sparsemax / 1.5-entmax); the backward
// recomputes the weights block by block from it and accumulates the query,
// key and value gradients ("HF Attention Normalizers", section "Important
// Limitations": row statistics saved, probabilities recomputed during the
// fused backward).  With L = sum(dO * O), dP = dO V^T and, per row i, the
// normalizer's Jacobian in the form
//
//     dZ_ij = w_ij (dP_ij - delta_i)
//
//   softmax / softmax1 / sinks:  w = p,               delta_i = dO_i . O_i
//   sparsemax:                   w = 1[z > tau],      delta_i = sum_j w dP / sum_j w
//   1.5-entmax:                  w = relu(z/2 - tau), delta_i = sum_j w dP / sum_j w
//
// (the sparse Jacobians of Martins & Astudillo 2016 and Peters et al. 2019;
// the 1/2 of z/2 and the 2 of p = w^2 cancel), then dS = dZ * dz/ds with
// dz/ds = scale (or scale (1 - tanh^2) under the soft-cap), and
//
//     dV = P^T dO,   dK = dS^T Q,   dQ = dS K.
//
// Two kernels share the work without atomics:
//   bwd_dq_kernel    one CTA per 128-row query tile, walking its visible
//                    64-key blocks: S = Q K^T and dP = dO V^T into TMEM
//                    (double-buffered), dS from the normalizer warps into
//                    shared memory, dQ += dS K into TMEM.  Its DELTA mode runs
//                    first for the sparse normalizers and only accumulates
//                    sum w dP and sum w per row.
//   bwd_dkdv_kernel  one CTA per 128-key tile of one key/value head, walking
//                    the 64-row query blocks of every query head of the group
//                    that see it: S^T = K Q^T and dP^T = V dO^T into TMEM
//                    (double-buffered), P^T and dS^T into shared memory, then
//                    dV += P^T dO and dK += dS^T Q into TMEM.
// The weights and dS reach the tensor cores from shared memory (bf16), so no
// TMEM store ever overlaps a product in flight.
#pragma once

#include "common.cuh"
#include "problem.cuh"
#include "prefill_tc.cuh"

namespace nattn {

struct BwdArgs {
  Problem P;            // q, k, v, out (the forward output), row_stat, sinks, mask
  const bf16* dout;     // [B, Hq, Tq, dv]
  bf16* dq;             // [B, Hq, Tq, d]
  bf16* dk;             // [B, Hkv, Tk, d]
  bf16* dv;             // [B, Hkv, Tk, dv]
  float* delta;         // [B * Hq * Tq] per-row term of the Jacobian
  float us;             // threshold units: 1 (sparsemax) or 1/2 (1.5-entmax)
};

constexpr int BWD_THREADS = 192;  // 4 normalizer warps + TMA warp + MMA warp
constexpr int BWD_BN = 64;        // keys per block (dQ kernel)
constexpr int BWD_BQ = 64;        // queries per block (dK/dV kernel)

enum BwdMode { BWD_DELTA = 0, BWD_DQ = 1 };

// One score's contribution, from the raw dot product s, the row's saved
// statistic st (log-sum-exp in log2 units for the softmax family, tau for
// the sparse normalizers), its delta and dP: the weight p (for dV) and dS
// without the constant factor `scale` (applied to dQ and dK once, in the
// epilogues; under the soft-cap dS keeps the 1 - tanh^2 of dz/ds).
// KIND: 0 softmax / softmax1 / sinks, 1 sparsemax, 2 1.5-entmax.
template <int KIND, bool CAP>
struct BwdOp {
  float a;  // CAP: scale / cap; else scale * log2(e) (KIND 0) or scale * us
  float b;  // CAP: cap * log2(e) (KIND 0) or cap * us
  __device__ __forceinline__ void eval(float s, float st, float dl, float dp, float& p,
                                       float& ds, float& w) const {
    float x, gcap = 1.f;
    if (CAP) {
      const float t = fast_tanh(s * a);
      x = fmaf(t, b, -st);
      gcap = fmaf(-t, t, 1.f);
    } else {
      x = fmaf(s, a, -st);
    }
    if (KIND == 0) {
      p = fast_exp2(x);
      w = p;
    } else if (KIND == 1) {
      p = fmaxf(x, 0.f);
      w = x > 0.f ? 1.f : 0.f;
    } else {
      const float r = fmaxf(x, 0.f);
      p = r * r;
      w = r;
    }
    ds = w * (dp - dl);
    if (CAP) ds *= gcap;
  }
};

template <int KIND, bool CAP>
__device__ __forceinline__ BwdOp<KIND, CAP> make_op(const BwdArgs& A) {
  const float unit = (KIND == 0) ? 1.4426950408889634f : A.us;
  BwdOp<KIND, CAP> op;
  op.a = CAP ? A.P.scale / A.P.softcap : A.P.scale * unit;
  op.b = CAP ? A.P.softcap * unit : 0.f;
  return op;
}

// Saved statistic of a row in the units BwdOp::eval takes.
__device__ __forceinline__ float bwd_stat2(const Problem& P, float st) {
  return (P.norm == NATTN_SOFTMAX || P.norm == NATTN_SOFTMAX1) ? st * 1.4426950408889634f
                                                                : st;
}

// Write 64 bf16 values (32 packed words) as one 128-byte row `r` of a
// 128-byte-swizzled tile (the K-major layout the MMA descriptors read).
__device__ __forceinline__ void st_row128(uint8_t* tile, int r, const uint32_t (&pk)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(tile + sw128(r, c)) =
        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

// softmax family: delta_i = dO_i . O_i, one warp per row.
__global__ void __launch_bounds__(256) bwd_delta_dot_kernel(BwdArgs A) {
  const Problem& P = A.P;
  const size_t rows = (size_t)P.B * P.Hq * P.Tq;
  const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const bf16* o = P.out + row * P.dv;
  const bf16* g = A.dout + row * P.dv;
  float acc = 0.f;
  for (int c = lane * 2; c < P.dv; c += 64) {
    const uint32_t a = *reinterpret_cast<const uint32_t*>(o + c);
    const uint32_t b = *reinterpret_cast<const uint32_t*>(g + c);
    acc = fmaf(bf16lo(a), bf16lo(b), acc);
    acc = fmaf(bf16hi(a), bf16hi(b), acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) A.delta[row] = acc;
}

// ---------------------------------------------------------------------------
// dQ (and the sparse delta) kernel
// ---------------------------------------------------------------------------
template <int D, int DV>
struct BwdQLayout {
  static constexpr int BN = BWD_BN;
  static constexpr int KST = 4, VST = 4;  // K and V blocks in flight
  static constexpr int QBYTES = 128 * D * 2;
  static constexpr int OBYTES = 128 * DV * 2;
  static constexpr int KBYTES = BN * D * 2;
  static constexpr int VBYTES = BN * DV * 2;
  static constexpr int DSBYTES = 128 * BN * 2;  // one dS buffer [128 q][64 keys]
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_O = OFF_Q + QBYTES;
  static constexpr int OFF_K = OFF_O + OBYTES;
  static constexpr int OFF_V = OFF_K + KST * KBYTES;
  static constexpr int OFF_DS = OFF_V + VST * VBYTES;
  static constexpr int OFF_BAR = OFF_DS + 2 * DSBYTES;
  // q, kfull/kempty, vfull/vempty, sfull[2], dsfull[2], dsempty[2], done
  static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 6 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int ALLOC = OFF_MISC + 16 + 1024;
  static constexpr int TM_S = 0;        // S buffer b at column b * BN
  static constexpr int TM_DP = 2 * BN;  // dP buffer b at TM_DP + b * BN
  static constexpr int TM_DQ = 4 * BN;
  static constexpr int TM_COLS = 512;
  static_assert(TM_DQ + D <= TM_COLS, "TMEM budget");
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
};

template <int D, int DV, int MODE, int KIND, bool CAP>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmo,
                  const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  BwdArgs A) {
  using LY = BwdQLayout<D, DV>;
  constexpr int BN = LY::BN, KST = LY::KST, VST = LY::VST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Problem& P = A.P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // heaviest tiles (latest query rows) first
  const int ntq = (P.Tq + 127) / 128;
  const int BH = P.B * P.Hq;
  const int qt = P.causal ? (ntq - 1 - (int)blockIdx.x / BH) : ((int)blockIdx.x / BH);
  const int bh = (int)blockIdx.x % BH;
  const int b = bh / P.Hq, h = bh % P.Hq;
  const int g = h / (P.Hq / P.Hkv);
  const int q0 = qt * 128;
  const int qlast = min(q0 + 127, P.Tq - 1);
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
  auto bar_dsfull = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + 2 + s]); };
  auto bar_dsempty = [&](int s) { return smem_addr(&bars[1 + 2 * KST + 2 * VST + 4 + s]); };
  const uint32_t bar_done = smem_addr(&bars[1 + 2 * KST + 2 * VST + 6]);
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
      mbar_init(bar_dsfull(s), 4);
      mbar_init(bar_dsempty(s), 1);
    }
    mbar_init(bar_done, 1);
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
      tma_prefetch_desc(&tmo);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      mbar_expect_tx(bar_q, LY::QBYTES + LY::OBYTES);
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_addr(smem + LY::OFF_Q + x * 128 * 128), &tmq, bar_q, x * 64, q0, bh);
      for (int x = 0; x < DV / 64; ++x)
        tma_load_3d(smem_addr(smem + LY::OFF_O + x * 128 * 128), &tmo, bar_q, x * 64, q0, bh);
      for (int j = 0; j < nblk; ++j) {
        const int kb = kb0 + j;
        const int ks = j % KST, vs = j % VST;
        if (j >= KST && !mbar_wait(bar_kempty(ks), ((j / KST) + 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_kfull(ks), LY::KBYTES);
        for (int x = 0; x < D / 64; ++x)
          tma_load_3d(smem_addr(smem + LY::OFF_K + ks * LY::KBYTES + x * BN * 128), &tmk,
                      bar_kfull(ks), x * 64, kb * BN, b * P.Hkv + g);
        if (j >= VST && !mbar_wait(bar_vempty(vs), ((j / VST) + 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_vfull(vs), LY::VBYTES);
        for (int x = 0; x < DV / 64; ++x)
          tma_load_3d(smem_addr(smem + LY::OFF_V + vs * LY::VBYTES + x * BN * 128), &tmv,
                      bar_vfull(vs), x * 64, kb * BN, b * P.Hkv + g);
      }
    }
  } else if (warp == 5) {
    // ======================= MMA issuer =====================================
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
      constexpr uint32_t IDESC_DQ = idesc_bf16(128, D, 0, 1);
      const uint32_t qbase = smem_addr(smem + LY::OFF_Q);
      const uint32_t obase = smem_addr(smem + LY::OFF_O);
      bool ok = mbar_wait_spin(bar_q, 0, abort_flag);
      tc_fence_after();
      for (int j = 0; ok && j <= nblk; ++j) {
        if (j < nblk) {
          const int sb = j & 1, ks = j % KST, vs = j % VST;
          if (!mbar_wait_spin(bar_kfull(ks), (j / KST) & 1, abort_flag)) break;
          if (!mbar_wait_spin(bar_vfull(vs), (j / VST) & 1, abort_flag)) break;
          // buffer sb last held block j - 2, whose normalizer pass is done
          if (j >= 2 && !mbar_wait_spin(bar_dsfull(sb), ((j - 2) >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t kbase = smem_addr(smem + LY::OFF_K + ks * LY::KBYTES);
          const uint32_t vbase = smem_addr(smem + LY::OFF_V + vs * LY::VBYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tmem + LY::TM_S + sb * BN,
                    sdesc_sw128(qbase + (kk >> 2) * 128 * 128 + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(kbase + (kk >> 2) * BN * 128 + (kk & 3) * 32, 16, 1024),
                    IDESC_S, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < DV / 16; ++kk)
            umma_ss(tmem + LY::TM_DP + sb * BN,
                    sdesc_sw128(obase + (kk >> 2) * 128 * 128 + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(vbase + (kk >> 2) * BN * 128 + (kk & 3) * 32, 16, 1024),
                    IDESC_S, kk > 0 ? 1u : 0u);
          umma_commit(bar_sfull(sb));
          umma_commit(bar_vempty(vs));
          if (MODE == BWD_DELTA) umma_commit(bar_kempty(ks));
        }
        if (MODE == BWD_DQ && j >= 1) {
          const int jp = j - 1, sbp = jp & 1, ks = jp % KST;
          if (!mbar_wait_spin(bar_dsfull(sbp), (jp >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t dsb = smem_addr(smem + LY::OFF_DS + sbp * LY::DSBYTES);
          const uint32_t kbase = smem_addr(smem + LY::OFF_K + ks * LY::KBYTES);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            // A = dS [128 q][64 keys] K-major; B = K block [64 keys][D] MN-major
            umma_ss(tmem + LY::TM_DQ, sdesc_sw128(dsb + kk * 32, 16, 1024),
                    sdesc_sw128(kbase + kk * 16 * 128, BN * 128, 1024), IDESC_DQ,
                    (jp > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar_kempty(ks));
          umma_commit(bar_dsempty(sbp));
        }
      }
      umma_commit(bar_done);
    }
  } else {
    // ======================= normalizer warps ==============================
    const int row = warp * 32 + lane;
    const int qi = q0 + row;
    const bool row_ok = qi < P.Tq;
    RowRange rr = row_range(P, qi, P.Tk);
    if (!row_ok) rr = RowRange{1, 0};
    if (rr.hi > P.Tk - 1) rr.hi = P.Tk - 1;
    const size_t flat = (size_t)bh * P.Tq + qi;
    const BwdOp<KIND, CAP> op = make_op<KIND, CAP>(A);
    const float stat2 = row_ok ? bwd_stat2(P, P.row_stat[flat]) : 0.f;
    const float dlt = (MODE == BWD_DQ && row_ok) ? A.delta[flat] : 0.f;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    float acc_wdp = 0.f, acc_w = 0.f;
    bool alive = true;
    for (int j = 0; j < nblk; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_spin(bar_sfull(sb), (j >> 1) & 1, abort_flag))) {
        alive = false;
        break;
      }
      tc_fence_after();
      uint32_t s[BN], dp[BN];
      tmem_ld32(lane_base + LY::TM_S + sb * BN, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(lane_base + LY::TM_S + sb * BN + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(lane_base + LY::TM_DP + sb * BN, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_ld32(lane_base + LY::TM_DP + sb * BN + 32,
                *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
      tmem_ld_wait();
      // visible keys of this row relative to the block: [kl, kl + span]
      const int jb = (kb0 + j) * BN;
      const int kl = rr.lo - jb;
      const unsigned span = rr.hi >= rr.lo ? (unsigned)(rr.hi - rr.lo) : 0u;
      // a block the block mask drops counts as masked whole
      const bool any = rr.hi >= rr.lo && block_kept(P, b, h, qt, jb >> 7);
      uint32_t pk[32];
#pragma unroll
      for (int k = 0; k < BN; k += 2) {
        float d2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float p, ds, w;
          op.eval(__uint_as_float(s[k + e]), stat2, dlt, __uint_as_float(dp[k + e]), p, ds, w);
          const bool vis = any && (unsigned)(k + e - kl) <= span;
          d2[e] = vis ? ds : 0.f;
          if (MODE == BWD_DELTA && vis) {
            acc_wdp = fmaf(w, __uint_as_float(dp[k + e]), acc_wdp);
            acc_w += w;
          }
        }
        pk[k >> 1] = pack_bf16(d2[0], d2[1]);
      }
      if (MODE == BWD_DQ) {
        // the dQ product of block j - 2 has read this dS buffer
        if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait_spin(bar_dsempty(sb), ((j - 2) >> 1) & 1,
                                                              abort_flag))) {
          alive = false;
          break;
        }
        st_row128(smem + LY::OFF_DS + sb * LY::DSBYTES, row, pk);
        fence_proxy_async();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dsfull(sb));
    }
    if (MODE == BWD_DELTA) {
      if (row_ok) A.delta[flat] = acc_w > 0.f ? acc_wdp / acc_w : 0.f;
    } else {
      const bool have = __all_sync(0xffffffffu,
                                   alive && nblk > 0 && mbar_wait(bar_done, 0, abort_flag));
      tc_fence_after();
      bf16* drow = A.dq + flat * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(lane_base + LY::TM_DQ + c * 32, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = 0u;
        }
        if (row_ok) {
          // dS left out the constant factor `scale`
          const float sc = P.scale;
          uint4* dst = reinterpret_cast<uint4*>(drow + c * 32);
#pragma unroll
          for (int k = 0; k < 32; k += 8)
            dst[k / 8] = make_uint4(
                pack_bf16(__uint_as_float(r[k]) * sc, __uint_as_float(r[k + 1]) * sc),
                pack_bf16(__uint_as_float(r[k + 2]) * sc, __uint_as_float(r[k + 3]) * sc),
                pack_bf16(__uint_as_float(r[k + 4]) * sc, __uint_as_float(r[k + 5]) * sc),
                pack_bf16(__uint_as_float(r[k + 6]) * sc, __uint_as_float(r[k + 7]) * sc));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, LY::TM_COLS);
}

// ---------------------------------------------------------------------------
// dK / dV kernel
// ---------------------------------------------------------------------------
template <int D, int DV>
struct BwdKVLayout {
  static constexpr int BQ = BWD_BQ;
  static constexpr int QST = 3;  // query / dO / statistics slots in flight
  static constexpr int KBYTES = 128 * D * 2;
  static constexpr int VBYTES = 128 * DV * 2;
  static constexpr int QBYTES = BQ * D * 2;
  static constexpr int OBYTES = BQ * DV * 2;
  static constexpr int PBYTES = 128 * BQ * 2;  // one P^T or dS^T buffer [128 keys][64 q]
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KBYTES;
  static constexpr int OFF_Q = OFF_V + VBYTES;          // QST slots
  static constexpr int OFF_O = OFF_Q + QST * QBYTES;    // QST slots
  static constexpr int OFF_P = OFF_O + QST * OBYTES;    // P^T, 2 buffers
  static constexpr int OFF_DS = OFF_P + 2 * PBYTES;     // dS^T, 2 buffers
  static constexpr int OFF_ST = OFF_DS + 2 * PBYTES;    // QST slots of (stat2[64], delta[64])
  static constexpr int OFF_BAR = OFF_ST + QST * 2 * BQ * 4;
  // kv, qfull[QST], qempty[QST], sfull[2], pfull[2], pempty[2], done
  static constexpr int NBAR = 1 + 2 * QST + 6 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int ALLOC = OFF_MISC + 16 + 1024;
  static constexpr int TM_S = 0;         // S^T buffer b at b * BQ
  static constexpr int TM_DP = 2 * BQ;   // dP^T buffer b at TM_DP + b * BQ
  static constexpr int TM_DK = 4 * BQ;
  static constexpr int TM_DV = TM_DK + D;
  static constexpr int TM_COLS = 512;
  static_assert(TM_DV + DV <= TM_COLS, "TMEM budget");
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
};

// Query rows (inclusive) that see key j: the rows whose visible range (see
// row_range) contains j.
__device__ __forceinline__ RowRange key_query_range(const Problem& P, int j) {
  const int delta = P.Tk - P.Tq;  // query i sits at key position i + delta
  int lo = 0, hi = P.Tq - 1;
  if (P.causal) lo = max(lo, j - delta);
  if (P.window > 0) {
    hi = min(hi, j - delta + P.window - 1);
    if (!P.causal) lo = max(lo, j - delta - P.window + 1);
  }
  return RowRange{lo, hi};
}

template <int D, int DV, int KIND, bool CAP>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmo,
                    const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    BwdArgs A) {
  using LY = BwdKVLayout<D, DV>;
  constexpr int BQ = LY::BQ, QST = LY::QST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Problem& P = A.P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // key tiles that see the most query rows first (the earliest, when causal)
  const int BG = P.B * P.Hkv;
  const int kt = (int)blockIdx.x / BG;
  const int bg = (int)blockIdx.x % BG;
  const int b = bg / P.Hkv, g = bg % P.Hkv;
  const int group = P.Hq / P.Hkv;
  const int k0 = kt * 128;
  const int klast = min(k0 + 127, P.Tk - 1);
  // query rows that see some key of the tile: the union of the two ends' ranges
  const RowRange qa = key_query_range(P, k0), qb = key_query_range(P, klast);
  const int qlo = max(0, min(qa.lo, qb.lo)), qhi = min(P.Tq - 1, max(qa.hi, qb.hi));
  const int qb0 = qlo / BQ;
  const int nqb = (qhi >= qlo) ? (qhi / BQ - qb0 + 1) : 0;
  const int nit = nqb * group;  // items: (head of the group, query block)

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::OFF_BAR);
  const uint32_t bar_kv = smem_addr(&bars[0]);
  auto bar_qfull = [&](int s) { return smem_addr(&bars[1 + s]); };
  auto bar_qempty = [&](int s) { return smem_addr(&bars[1 + QST + s]); };
  auto bar_sfull = [&](int s) { return smem_addr(&bars[1 + 2 * QST + s]); };
  auto bar_pfull = [&](int s) { return smem_addr(&bars[3 + 2 * QST + s]); };
  auto bar_pempty = [&](int s) { return smem_addr(&bars[5 + 2 * QST + s]); };
  const uint32_t bar_done = smem_addr(&bars[7 + 2 * QST]);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + LY::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);
  float* stats = reinterpret_cast<float*>(smem + LY::OFF_ST);  // slot q: [q * 128, +128)

  if (tid == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(bar_qfull(s), 1);
      mbar_init(bar_qempty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_sfull(s), 1);
      mbar_init(bar_pfull(s), 4);
      mbar_init(bar_pempty(s), 1);
    }
    mbar_init(bar_done, 1);
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
  auto item = [&](int it, int& h, int& q0) {
    h = g * group + it / nqb;
    q0 = (qb0 + it % nqb) * BQ;
  };

  if (warp == 4) {
    // ======================= producer: TMA + the rows' statistics ==========
    if (nit > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmo);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        mbar_expect_tx(bar_kv, LY::KBYTES + LY::VBYTES);
        for (int x = 0; x < D / 64; ++x)
          tma_load_3d(smem_addr(smem + LY::OFF_K + x * 128 * 128), &tmk, bar_kv, x * 64, k0, bg);
        for (int x = 0; x < DV / 64; ++x)
          tma_load_3d(smem_addr(smem + LY::OFF_V + x * 128 * 128), &tmv, bar_kv, x * 64, k0, bg);
      }
      for (int it = 0; it < nit; ++it) {
        const int qs = it % QST;
        if (it >= QST && !__all_sync(0xffffffffu, mbar_wait(bar_qempty(qs),
                                                            ((it / QST) + 1) & 1, abort_flag)))
          break;
        int h, q0;
        item(it, h, q0);
        const size_t fbase = ((size_t)b * P.Hq + h) * P.Tq;
        for (int c = lane; c < BQ; c += 32) {
          const int qi = q0 + c;
          const bool ok = qi < P.Tq;
          stats[qs * 2 * BQ + c] = ok ? bwd_stat2(P, P.row_stat[fbase + qi]) : 0.f;
          stats[qs * 2 * BQ + BQ + c] = ok ? A.delta[fbase + qi] : 0.f;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(bar_qfull(qs), LY::QBYTES + LY::OBYTES);
          for (int x = 0; x < D / 64; ++x)
            tma_load_3d(smem_addr(smem + LY::OFF_Q + qs * LY::QBYTES + x * BQ * 128), &tmq,
                        bar_qfull(qs), x * 64, q0, b * P.Hq + h);
          for (int x = 0; x < DV / 64; ++x)
            tma_load_3d(smem_addr(smem + LY::OFF_O + qs * LY::OBYTES + x * BQ * 128), &tmo,
                        bar_qfull(qs), x * 64, q0, b * P.Hq + h);
        }
        __syncwarp();
      }
    }
  } else if (warp == 5) {
    // ======================= MMA issuer =====================================
    if (lane == 0 && nit > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, BQ, 0, 0);
      constexpr uint32_t IDESC_DK = idesc_bf16(128, D, 0, 1);
      constexpr uint32_t IDESC_DV = idesc_bf16(128, DV, 0, 1);
      const uint32_t kbase = smem_addr(smem + LY::OFF_K);
      const uint32_t vbase = smem_addr(smem + LY::OFF_V);
      bool ok = mbar_wait_spin(bar_kv, 0, abort_flag);
      tc_fence_after();
      for (int it = 0; ok && it <= nit; ++it) {
        if (it < nit) {
          const int s = it & 1, qs = it % QST;
          if (!mbar_wait_spin(bar_qfull(qs), (it / QST) & 1, abort_flag)) break;
          // TMEM buffer s last held item it - 2, read once pfull(it - 2)
          // completed, which the previous iteration waited for
          tc_fence_after();
          const uint32_t qbase = smem_addr(smem + LY::OFF_Q + qs * LY::QBYTES);
          const uint32_t obase = smem_addr(smem + LY::OFF_O + qs * LY::OBYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tmem + LY::TM_S + s * BQ,
                    sdesc_sw128(kbase + (kk >> 2) * 128 * 128 + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(qbase + (kk >> 2) * BQ * 128 + (kk & 3) * 32, 16, 1024),
                    IDESC_S, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < DV / 16; ++kk)
            umma_ss(tmem + LY::TM_DP + s * BQ,
                    sdesc_sw128(vbase + (kk >> 2) * 128 * 128 + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(obase + (kk >> 2) * BQ * 128 + (kk & 3) * 32, 16, 1024),
                    IDESC_S, kk > 0 ? 1u : 0u);
          umma_commit(bar_sfull(s));
        }
        if (it >= 1) {
          const int ip = it - 1, sp = ip & 1, qsp = ip % QST;
          if (!mbar_wait_spin(bar_pfull(sp), (ip >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t pb = smem_addr(smem + LY::OFF_P + sp * LY::PBYTES);
          const uint32_t db = smem_addr(smem + LY::OFF_DS + sp * LY::PBYTES);
          const uint32_t qbase = smem_addr(smem + LY::OFF_Q + qsp * LY::QBYTES);
          const uint32_t obase = smem_addr(smem + LY::OFF_O + qsp * LY::OBYTES);
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk) {
            // dV += P^T dO: A = P^T [128 keys][64 q] K-major, B = dO [64 q][DV] MN-major
            umma_ss(tmem + LY::TM_DV, sdesc_sw128(pb + kk * 32, 16, 1024),
                    sdesc_sw128(obase + kk * 16 * 128, BQ * 128, 1024), IDESC_DV,
                    (ip > 0 || kk > 0) ? 1u : 0u);
            // dK += dS^T Q: A = dS^T [128 keys][64 q], B = Q [64 q][D] MN-major
            umma_ss(tmem + LY::TM_DK, sdesc_sw128(db + kk * 32, 16, 1024),
                    sdesc_sw128(qbase + kk * 16 * 128, BQ * 128, 1024), IDESC_DK,
                    (ip > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar_qempty(qsp));
          umma_commit(bar_pempty(sp));
        }
      }
      umma_commit(bar_done);
    }
  } else {
    // ======================= normalizer warps: thread = key row ============
    const int row = warp * 32 + lane;
    const int kj = k0 + row;
    const bool key_ok = kj < P.Tk;
    RowRange qr = key_query_range(P, kj);
    if (!key_ok) qr = RowRange{1, 0};
    const BwdOp<KIND, CAP> op = make_op<KIND, CAP>(A);
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    bool alive = true;
    for (int it = 0; it < nit; ++it) {
      const int s = it & 1, qs = it % QST;
      int h, q0;
      item(it, h, q0);
      // qfull carries the producer's stores of the rows' statistics (it has
      // completed before sfull(s) can); sfull(s) the products
      if (!__all_sync(0xffffffffu, mbar_wait_spin(bar_qfull(qs), (it / QST) & 1, abort_flag) &&
                                       mbar_wait_spin(bar_sfull(s), (it >> 1) & 1, abort_flag))) {
        alive = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[BQ], dp[BQ];
      tmem_ld32(lane_base + LY::TM_S + s * BQ, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(lane_base + LY::TM_S + s * BQ + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(lane_base + LY::TM_DP + s * BQ, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_ld32(lane_base + LY::TM_DP + s * BQ + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
      tmem_ld_wait();
      const float4* st4 = reinterpret_cast<const float4*>(stats + qs * 2 * BQ);
      const float4* dl4 = st4 + BQ / 4;
      // visible query columns of this key: [cl, cl + span]
      const int cl = qr.lo - q0;
      const unsigned span = qr.hi >= qr.lo ? (unsigned)(qr.hi - qr.lo) : 0u;
      // a block the block mask drops counts as masked whole
      const bool any = qr.hi >= qr.lo && block_kept(P, b, h, q0 >> 7, kt);
      uint32_t ppk[32], dpk[32];
#pragma unroll
      for (int c4 = 0; c4 < BQ; c4 += 4) {
        const float4 sa = st4[c4 / 4], da = dl4[c4 / 4];
        const float stv[4] = {sa.x, sa.y, sa.z, sa.w};
        const float dlv[4] = {da.x, da.y, da.z, da.w};
        float pp[4], dd[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float p, ds, w;
          op.eval(__uint_as_float(sv[c4 + e]), stv[e], dlv[e], __uint_as_float(dp[c4 + e]), p,
                  ds, w);
          const bool vis = any && (unsigned)(c4 + e - cl) <= span;
          pp[e] = vis ? p : 0.f;
          dd[e] = vis ? ds : 0.f;
        }
        ppk[c4 >> 1] = pack_bf16(pp[0], pp[1]);
        ppk[(c4 >> 1) + 1] = pack_bf16(pp[2], pp[3]);
        dpk[c4 >> 1] = pack_bf16(dd[0], dd[1]);
        dpk[(c4 >> 1) + 1] = pack_bf16(dd[2], dd[3]);
      }
      // the dK/dV products of item it - 2 have read these buffers
      if (it >= 2 && !__all_sync(0xffffffffu, mbar_wait_spin(bar_pempty(s), ((it - 2) >> 1) & 1,
                                                              abort_flag))) {
        alive = false;
        break;
      }
      st_row128(smem + LY::OFF_P + s * LY::PBYTES, row, ppk);
      st_row128(smem + LY::OFF_DS + s * LY::PBYTES, row, dpk);
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull(s));
    }
    const bool have =
        __all_sync(0xffffffffu, alive && nit > 0 && mbar_wait(bar_done, 0, abort_flag));
    tc_fence_after();
    // dS left out the constant factor `scale`: dK takes it here
    auto store = [&](uint32_t tcol, bf16* dst, int cols, float sc) {
#pragma unroll 1
      for (int c = 0; c < cols / 32; ++c) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(lane_base + tcol + c * 32, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = 0u;
        }
        if (key_ok) {
          uint4* o = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int k = 0; k < 32; k += 8)
            o[k / 8] = make_uint4(
                pack_bf16(__uint_as_float(r[k]) * sc, __uint_as_float(r[k + 1]) * sc),
                pack_bf16(__uint_as_float(r[k + 2]) * sc, __uint_as_float(r[k + 3]) * sc),
                pack_bf16(__uint_as_float(r[k + 4]) * sc, __uint_as_float(r[k + 5]) * sc),
                pack_bf16(__uint_as_float(r[k + 6]) * sc, __uint_as_float(r[k + 7]) * sc));
        }
      }
    };
    const size_t krow = ((size_t)b * P.Hkv + g) * P.Tk + kj;
    store(LY::TM_DK, A.dk + krow * D, D, P.scale);
    store(LY::TM_DV, A.dv + krow * DV, DV, 1.f);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, LY::TM_COLS);
}

}  // namespace nattn
