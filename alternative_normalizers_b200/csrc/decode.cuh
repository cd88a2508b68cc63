// Paged split-KV decode.
//
// The KV cache is a pool of fixed-size pages read through a block table
// ("HF Attention Normalizers", section "Differentiable Paged Attention": the
// kernel reads physical K/V pages directly through the block table and never
// gathers them).  One CTA owns (sequence b, kv head g, split s): a run of
// whole pages of one sequence, and every query row of the kv-head group
// (group = Hq / Hkv heads x Tq new tokens, at most 16 rows), so each K/V page
// is read from HBM once for all the heads that share it.
//
// The path is bound by HBM bandwidth (4 KiB of K+V per token at Hkv = 8,
// d = 128), so the design is about the loads: each (page, kv head) slab is
// contiguous in the pool and is brought into shared memory by TMA in 64-column
// boxes with the 128-byte swizzle, one mbarrier per stage.  A CTA's time per
// page is mostly latency (the page's barrier, the products, the block
// barriers), so the ring is two stages deep and the bytes in flight come from
// three to five CTAs per SM.  The arithmetic per page is tiny (16 x 64 x 128
// per product) and runs on warp-level mma.sync so that it never competes with
// the loads for issue slots; row reductions use warp shuffles.
//
// Modes:
//   ONLINE  softmax / softmax1: running (max, sum, O) per split in log2 units,
//           merged by decode_combine_kernel (softmax1 adds its sink once there).
//   SCORES  sparse pass 1: write every score (in threshold units) to scratch
//           straight from the product's accumulators, and the split's row
//           maximum.
//   APPLY   sparse pass 3: given tau per row, skip pages with no weight above
//           zero (their V is never loaded), accumulate p V for the rest.
#pragma once

#include "common.cuh"
#include "problem.cuh"
#include "rowwise.cuh"

namespace nattn {

enum DecodeMode { DEC_ONLINE = 0, DEC_SCORES = 1, DEC_APPLY = 2 };

struct DecodeArgs {
  Problem P;
  int R;          // query rows per CTA = group * Tq (<= 16)
  int nsplit;     // splits per sequence
  int pps;        // pages per split
  float zscale;   // multiplies raw dot products (scale, x log2e for ONLINE)
  float uscale;   // threshold units: 1 (sparsemax) or 0.5 (entmax15)
  // scratch
  float* opart;   // [B*Hkv*nsplit*R][dv]
  float* ml;      // [B*Hkv*nsplit*R][2]      (ONLINE: m, l; SCORES: max)
  float* scores;  // [B*Hq*Tq][Tk]            (SCORES / APPLY)
  const float* tau;  // [B*Hq*Tq]             (APPLY)
  // pages of each row holding a nonzero weight, one bit per page, written by
  // the threshold kernel and read by APPLY: [B*Hq*Tq][pm_words]
  unsigned* pmask;
  int pm_words;
};

constexpr int DEC_THREADS = 128;

template <int D, int DV, int PS, int NS, int MODE>
struct DecodeSmem {
  static constexpr int KBYTES = (MODE == DEC_APPLY) ? 0 : PS * D * 2;
  static constexpr int VBYTES = (MODE == DEC_SCORES) ? 0 : PS * DV * 2;
  static constexpr int STAGE = KBYTES + VBYTES;
  static constexpr int SSTRIDE = PS + 4;             // floats per score row
  static constexpr int PSTRIDE = PS * 2 + 16;        // bytes per P row
  static constexpr int OFF_S = NS * STAGE;
  static constexpr int OFF_P = OFF_S + 16 * SSTRIDE * 4;
  // APPLY keeps P as bf16 hi + lo planes (weights to ~16 mantissa bits)
  static constexpr int OFF_PL = OFF_P + 16 * PSTRIDE;
  static constexpr int OFF_A = OFF_PL + ((MODE == DEC_APPLY) ? 16 * PSTRIDE : 0);
  static constexpr int OFF_BAR = OFF_A + 16 * 4;
  static constexpr int OFF_FLAGS = OFF_BAR + NS * 8;
  static constexpr int OFF_LIST = OFF_FLAGS + NS * 4;
  static constexpr int BYTES_NOLIST = OFF_LIST;
};

// Query fragment of the score product S^T = K Q^T (B operand, col-major:
// b0 = Q[row][k0 + 2t, +1], b1 = Q[row][k0 + 8 + 2t, +1]).
template <int D, int NTR>
__device__ __forceinline__ void load_q_frags(const DecodeArgs& A, int b, int g,
                                             uint32_t (&qf)[D / 16][NTR][2]) {
  const Problem& P = A.P;
  const int lane = threadIdx.x & 31, gq = lane >> 2, t = lane & 3;
  const int group = P.Hq / P.Hkv;
#pragma unroll
  for (int nt = 0; nt < NTR; ++nt) {
    const int r = nt * 8 + gq;
    const bool ok = r < A.R;
    const int hh = ok ? r / P.Tq : 0, i = ok ? r % P.Tq : 0;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        P.q + (((size_t)b * P.Hq + g * group + hh) * P.Tq + i) * D);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qf[kk][nt][0] = ok ? qrow[kk * 8 + t] : 0u;
      qf[kk][nt][1] = ok ? qrow[kk * 8 + 4 + t] : 0u;
    }
  }
}

template <int D, int DV, int PS, int NS, int NTR, int MODE>
__global__ void __launch_bounds__(DEC_THREADS)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, DecodeArgs A) {
  using L = DecodeSmem<D, DV, PS, NS, MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Problem& P = A.P;
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, t4 = lane & 3;
  const int R = A.R;
  const int group = P.Hq / P.Hkv;

  const int Lk = P.seqlens[b];
  if (Lk < 1 || Lk > P.Tk || Lk > P.bt_stride * PS) {
    if (tid == 0 && s == 0) set_status(NATTN_EBOUNDS);
    return;
  }
  const int npages = (Lk + PS - 1) / PS;
  const int p_begin = s * A.pps;
  const int p_end = min(p_begin + A.pps, npages);
  if (p_begin >= p_end) return;

  float* S = reinterpret_cast<float*>(smem + L::OFF_S);
  uint8_t* Pb = smem + L::OFF_P;
  uint8_t* Pl = smem + L::OFF_PL;
  float* alpha = reinterpret_cast<float*>(smem + L::OFF_A);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  int* badflag = reinterpret_cast<int*>(smem + L::OFF_FLAGS);
  int* plist = reinterpret_cast<int*>(smem + L::OFF_LIST);  // [2 * pps]
  __shared__ int s_count;
  __shared__ volatile int s_abort;

  // ---- APPLY: which pages of this split carry any nonzero weight ----------
  int count = p_end - p_begin;
  if constexpr (MODE == DEC_APPLY) {
    // a page is loaded when any row of the group has a nonzero weight in it
    // (bits set by the threshold kernel)
    int* pflag = plist + A.pps;
    for (int p = p_begin + tid; p < p_end; p += DEC_THREADS) {
      unsigned any = 0;
      for (int r = 0; r < R; ++r) {
        const int hh = r / P.Tq, i = r % P.Tq;
        const size_t row = ((size_t)b * P.Hq + g * group + hh) * P.Tq + i;
        any |= (A.pmask[row * A.pm_words + (p >> 5)] >> (p & 31)) & 1u;
      }
      pflag[p - p_begin] = (int)any;
    }
    __syncthreads();
    if (tid == 0) {  // compact in page order so the sums are deterministic
      int n = 0;
      for (int p = p_begin; p < p_end; ++p)
        if (pflag[p - p_begin]) plist[n++] = p;
      s_count = n;
    }
    __syncthreads();
    count = s_count;
  }

  if (tid == 0) {
    for (int st = 0; st < NS; ++st) mbar_init(smem_addr(&bars[st]), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  auto page_of = [&](int it) -> int {
    if constexpr (MODE == DEC_APPLY) return plist[it];
    return p_begin + it;
  };
  auto issue = [&](int it) {
    const int st = it % NS;
    const int p = page_of(it);
    int page = P.block_table[(size_t)b * P.bt_stride + p];
    int bad = 0;
    if (page < 0 || page >= P.num_pages) {
      bad = 1;
      page = 0;
      set_status(NATTN_EBOUNDS);
    }
    badflag[st] = bad;
    const uint32_t bar = smem_addr(&bars[st]);
    mbar_expect_tx(bar, L::STAGE);
    const int row0 = (page * P.Hkv + g) * PS;
    uint8_t* stage = smem + st * L::STAGE;
    if constexpr (MODE != DEC_APPLY) {
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx)
        tma_load_2d(smem_addr(stage + bx * PS * 128), &tmk, bar, bx * 64, row0);
    }
    if constexpr (MODE != DEC_SCORES) {
#pragma unroll
      for (int bx = 0; bx < DV / 64; ++bx)
        tma_load_2d(smem_addr(stage + L::KBYTES + bx * PS * 128), &tmv, bar, bx * 64,
                    row0);
    }
  };

  if (tid == 0) {
    for (int it = 0; it < NS && it < count; ++it) issue(it);
  }

  uint32_t qf[D / 16][NTR][2];
  if constexpr (MODE != DEC_APPLY) load_q_frags<D, NTR>(A, b, g, qf);

  // running statistics of the rows this warp owns (rows warp, warp+4, ...)
  float m_run[4], l_run[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    m_run[k] = -INFINITY;
    l_run[k] = 0.f;
  }
  constexpr int NOT = DV / 32;  // n-tiles of 8 output columns per warp (DV/4 columns)
  float oacc[NOT > 0 ? NOT : 1][4];
#pragma unroll
  for (int n = 0; n < NOT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[n][e] = 0.f;

  // SCORES: each thread's score rows (nt * 8 + 2 * t4 + h) in the scratch,
  // and their running maxima over the thread's keys
  float* srow[NTR][2];
  float mreg[NTR][2];
#pragma unroll
  for (int nt = 0; nt < NTR; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = nt * 8 + 2 * t4 + h;
      srow[nt][h] = nullptr;
      mreg[nt][h] = -INFINITY;
      if constexpr (MODE == DEC_SCORES)
        if (r < R)
          srow[nt][h] = A.scores +
                        (((size_t)b * P.Hq + g * group + r / P.Tq) * P.Tq + r % P.Tq) * P.Tk;
    }

  // zero the unused P rows once (rows >= R stay zero)
  for (int x = tid; x < (L::OFF_A - L::OFF_P) / 4; x += DEC_THREADS)
    reinterpret_cast<uint32_t*>(Pb)[x] = 0u;
  __syncthreads();

  for (int it = 0; it < count; ++it) {
    const int st = it % NS;
    const uint32_t par = (it / NS) & 1;
    const int p = page_of(it);
    const int j0 = p * PS;
    const bool got = mbar_wait(smem_addr(&bars[st]), par, &s_abort);
    if (!__syncthreads_and(got)) break;  // every thread leaves together
    uint8_t* stage = smem + st * L::STAGE;
    const bool bad = badflag[st] != 0;

    if constexpr (MODE != DEC_SCORES) {
      // a partial last page may hold stale values past the sequence end:
      // zero those V rows so that 0-weights never meet NaN/Inf
      if (j0 + PS > Lk) {
        const int valid = Lk - j0;
        uint8_t* vs = stage + L::KBYTES;
        for (int x = tid; x < (PS - valid) * (DV / 8); x += DEC_THREADS) {
          const int row = valid + x / (DV / 8), c = x % (DV / 8);
          *reinterpret_cast<uint4*>(vs + (c / 8) * PS * 128 + sw128(row, c % 8)) =
              make_uint4(0, 0, 0, 0);
        }
      }
    }

    if constexpr (MODE != DEC_APPLY) {
      // ---- scores S^T[tok][row] = K Q^T on mma.sync ----------------------
      for (int mt = warp; mt < PS / 16; mt += DEC_THREADS / 32) {
        float c[NTR][4];
#pragma unroll
        for (int nt = 0; nt < NTR; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
        const int row = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int chunk = kk * 2 + (lane >> 4);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(smem_addr(stage + (chunk >> 3) * PS * 128 + sw128(row, chunk & 7)), a0,
                  a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NTR; ++nt)
            mma_bf16_16816(c[nt], a0, a1, a2, a3, qf[kk][nt][0], qf[kk][nt][1]);
        }
#pragma unroll
        for (int nt = 0; nt < NTR; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = nt * 8 + 2 * t4 + (e & 1);
            const int tok = mt * 16 + gq + 8 * (e >> 1);
            if (r < R) {
              const int i = r % P.Tq;
              const int j = j0 + tok;
              const RowRange rr = row_range(P, i, Lk);
              float z = c[nt][e] * A.zscale;
              if (P.softcap > 0.f) {
                // soft-cap acts on scale * s; zscale = scale * extra factor
                const float sc = c[nt][e] * P.scale;
                z = P.softcap * fast_tanh(sc / P.softcap) * (A.zscale / P.scale);
              }
              const bool ok = !bad && j >= rr.lo && j <= rr.hi;
              if constexpr (MODE == DEC_SCORES) {
                // straight from the accumulators: 8 lanes cover 8
                // consecutive keys of a row (32-byte segments)
                const float zz = ok ? z : -INFINITY;
                if (j < Lk) srow[nt][e & 1][j] = zz;
                mreg[nt][e & 1] = fmaxf(mreg[nt][e & 1], zz);
              } else {
                S[r * L::SSTRIDE + tok] = ok ? z : -INFINITY;
              }
            }
          }
        }
      }
      if constexpr (MODE != DEC_SCORES) __syncthreads();
    }

    if constexpr (MODE == DEC_ONLINE) {
      // ---- online softmax over this page (log2 units) --------------------
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = warp + 4 * k;
        if (r >= R) break;
        float mx = -INFINITY;
        for (int jj = lane; jj < PS; jj += 32) mx = fmaxf(mx, S[r * L::SSTRIDE + jj]);
        mx = warp_max(mx);
        const float mnew = fmaxf(m_run[k], mx);
        const float msafe = (mnew == -INFINITY) ? 0.f : mnew;
        const float a = fast_exp2(m_run[k] - msafe);  // 0 when m_run = -inf
        float sum = 0.f;
        for (int jj = lane; jj < PS; jj += 32) {
          const float pz = fast_exp2(S[r * L::SSTRIDE + jj] - msafe);
          sum += pz;
          reinterpret_cast<bf16*>(Pb + r * L::PSTRIDE)[jj] = __float2bfloat16_rn(pz);
        }
        sum = warp_sum(sum);
        l_run[k] = l_run[k] * a + sum;
        m_run[k] = mnew;
        if (lane == 0) alpha[r] = a;
      }
      __syncthreads();
    }

    if constexpr (MODE == DEC_APPLY) {
      // weights from the stored scores and tau
      for (int r = warp; r < R; r += DEC_THREADS / 32) {
        const int hh = r / P.Tq, i = r % P.Tq;
        const size_t row = ((size_t)b * P.Hq + g * group + hh) * P.Tq + i;
        const float tr = A.tau[row];
        for (int jj = lane; jj < PS; jj += 32) {
          const int j = j0 + jj;
          float w = 0.f;
          if (j < Lk && !bad) {
            const float u = A.scores[row * P.Tk + j];
            const float x = fmaxf(u - tr, 0.f);
            w = (P.norm == NATTN_ENTMAX15) ? x * x : x;
          }
          const bf16 wh = __float2bfloat16_rn(w);
          reinterpret_cast<bf16*>(Pb + r * L::PSTRIDE)[jj] = wh;
          reinterpret_cast<bf16*>(Pl + r * L::PSTRIDE)[jj] =
              __float2bfloat16_rn(w - __bfloat162float(wh));
        }
      }
      __syncthreads();
    }

    if constexpr (MODE != DEC_SCORES) {
      // ---- O[row][col] (+)= P[row][tok] V[tok][col] on mma.sync ----------
      if constexpr (MODE == DEC_ONLINE) {
        const float a_lo = (gq < R) ? alpha[gq] : 1.f;
        const float a_hi = (gq + 8 < R) ? alpha[gq + 8] : 1.f;
#pragma unroll
        for (int n = 0; n < NOT; ++n) {
          oacc[n][0] *= a_lo;
          oacc[n][1] *= a_lo;
          oacc[n][2] *= a_hi;
          oacc[n][3] *= a_hi;
        }
      }
      const uint8_t* vs = stage + L::KBYTES;
      const int col0 = warp * (DV / 4);
#pragma unroll
      for (int kk = 0; kk < PS / 16; ++kk) {
        uint32_t a0, a1, a2, a3, l0 = 0, l1 = 0, l2 = 0, l3 = 0;
        {
          const int prow = (lane & 7) + 8 * ((lane >> 3) & 1);
          const int pchunk = kk * 2 + (lane >> 4);
          ldsm_x4(smem_addr(Pb + prow * L::PSTRIDE + pchunk * 16), a0, a1, a2, a3);
          if constexpr (MODE == DEC_APPLY)
            ldsm_x4(smem_addr(Pl + prow * L::PSTRIDE + pchunk * 16), l0, l1, l2, l3);
        }
#pragma unroll
        for (int n = 0; n < NOT; n += 2) {
          const int tok = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
          const int cchunk = (col0 >> 3) + n + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_addr(vs + (cchunk >> 3) * PS * 128 + sw128(tok, cchunk & 7)), b0,
                    b1, b2, b3);
          mma_bf16_16816(oacc[n], a0, a1, a2, a3, b0, b1);
          if (n + 1 < NOT) mma_bf16_16816(oacc[n + 1], a0, a1, a2, a3, b2, b3);
          if constexpr (MODE == DEC_APPLY) {
            mma_bf16_16816(oacc[n], l0, l1, l2, l3, b0, b1);
            if (n + 1 < NOT) mma_bf16_16816(oacc[n + 1], l0, l1, l2, l3, b2, b3);
          }
        }
      }
    }
    __syncthreads();  // stage, S and P are free again
    if (tid == 0 && it + NS < count) {
      fence_proxy_async();
      issue(it + NS);
    }
  }

  if constexpr (MODE == DEC_SCORES) {
    // row maxima: over the 8 lanes sharing a row, then over the warps
    float* smax = S;  // [4 warps][16 rows]
#pragma unroll
    for (int nt = 0; nt < NTR; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v = mreg[nt][h];
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        if (gq == 0) smax[warp * 16 + nt * 8 + 2 * t4 + h] = v;
      }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = warp + 4 * k;
      if (r < R)
        m_run[k] = fmaxf(fmaxf(smax[r], smax[16 + r]), fmaxf(smax[32 + r], smax[48 + r]));
    }
  }

  // ---- partial results of this split --------------------------------------
  const size_t pbase = (((size_t)b * P.Hkv + g) * A.nsplit + s) * R;
  if constexpr (MODE == DEC_ONLINE || MODE == DEC_SCORES) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = warp + 4 * k;
      if (r >= R) break;
      if (lane == 0) {
        A.ml[(pbase + r) * 2 + 0] = m_run[k];
        A.ml[(pbase + r) * 2 + 1] = l_run[k];
      }
    }
  }
  if constexpr (MODE != DEC_SCORES) {
    const int col0 = warp * (DV / 4);
#pragma unroll
    for (int n = 0; n < NOT; ++n) {
      const int c = col0 + n * 8 + 2 * t4;
      if (gq < R)
        *reinterpret_cast<float2*>(&A.opart[(pbase + gq) * DV + c]) =
            make_float2(oacc[n][0], oacc[n][1]);
      if (gq + 8 < R)
        *reinterpret_cast<float2*>(&A.opart[(pbase + gq + 8) * DV + c]) =
            make_float2(oacc[n][2], oacc[n][3]);
    }
  }
}

// Merge the splits of every query row.  ONLINE: rescale each split's (m, l, O)
// to the common maximum; the sink (softmax1's logit 0 or a learned per-head
// logit) is added exactly once here.
// APPLY: plain sum of the partial outputs; row_stat = tau.
__global__ void decode_combine_kernel(DecodeArgs A, int mode) {
  const Problem& P = A.P;
  const int row = blockIdx.x;  // flat (b, h, i)
  const int i = row % P.Tq;
  const int h = (row / P.Tq) % P.Hq;
  const int b = row / (P.Tq * P.Hq);
  const int group = P.Hq / P.Hkv;
  const int g = h / group, r = (h % group) * P.Tq + i;
  const int Lk = P.seqlens[b];
  const bool valid = !(Lk < 1 || Lk > P.Tk || Lk > P.bt_stride * P.page_size);
  const int npages = valid ? (Lk + P.page_size - 1) / P.page_size : 0;
  const int nact = min(A.nsplit, (npages + A.pps - 1) / A.pps);
  const size_t pbase = (((size_t)b * P.Hkv + g) * A.nsplit) * A.R + r;
  if (mode == DEC_ONLINE) {
    // the sink (softmax1: logit 0; learned per-head sink) enters once, here
    const float sink2 = sink_logit(P, h) * 1.4426950408889634f;
    float M = sink2;
    for (int s = 0; s < nact; ++s) M = fmaxf(M, A.ml[(pbase + (size_t)s * A.R) * 2]);
    const float msafe = (M == -INFINITY) ? 0.f : M;
    float l = (sink2 == -INFINITY) ? 0.f : fast_exp2(sink2 - msafe);
    for (int s = 0; s < nact; ++s) {
      const float ms = A.ml[(pbase + (size_t)s * A.R) * 2];
      l += A.ml[(pbase + (size_t)s * A.R) * 2 + 1] * fast_exp2(ms - msafe);
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    for (int c = threadIdx.x; c < P.dv; c += blockDim.x) {
      float o = 0.f;
      for (int s = 0; s < nact; ++s) {
        const float ms = A.ml[(pbase + (size_t)s * A.R) * 2];
        o += A.opart[(pbase + (size_t)s * A.R) * P.dv + c] * fast_exp2(ms - msafe);
      }
      P.out[(size_t)row * P.dv + c] = __float2bfloat16_rn(o * inv);
    }
    if (threadIdx.x == 0 && P.row_stat)
      P.row_stat[row] = (l > 0.f) ? (msafe + log2f(l)) * 0.6931471805599453f : -INFINITY;
    if (threadIdx.x == 0 && P.row_nnz) {
      const RowRange rr = row_range(P, i, valid ? Lk : 0);
      P.row_nnz[row] = rr.hi >= rr.lo ? rr.hi - rr.lo + 1 : 0;
    }
  } else {
    for (int c = threadIdx.x; c < P.dv; c += blockDim.x) {
      float o = 0.f;
      for (int s = 0; s < nact; ++s) o += A.opart[(pbase + (size_t)s * A.R) * P.dv + c];
      P.out[(size_t)row * P.dv + c] = __float2bfloat16_rn(o);
    }
    if (threadIdx.x == 0 && P.row_stat) P.row_stat[row] = valid ? A.tau[row] : INFINITY;
  }
}

// Sparse pass 2: tau of every query row from its stored scores.  The row
// maximum comes from the per-split maxima; entries within one threshold unit
// of it (the only ones that can be in the support, since tau >= max - 1) are
// gathered into shared memory and the exact threshold is solved there.  Rows
// with more candidates than fit are solved over the whole stored row.
constexpr int TAU_THREADS = 256;

__global__ void __launch_bounds__(TAU_THREADS)
    decode_tau_kernel(DecodeArgs A, float* tau_out, int cap) {
  extern __shared__ float tsm[];
  float* red = tsm;
  float* cand = tsm + 64;                                     // [cap] values
  int* cidx = reinterpret_cast<int*>(cand + cap);             // [cap] key indices
  unsigned* smask = reinterpret_cast<unsigned*>(cidx + cap);  // [pm_words]
  __shared__ int s_n;
  __shared__ int s_sup;  // support size
  const Problem& P = A.P;
  const int row = blockIdx.x;
  const int i = row % P.Tq;
  const int h = (row / P.Tq) % P.Hq;
  const int b = row / (P.Tq * P.Hq);
  const int group = P.Hq / P.Hkv;
  const int g = h / group, r = (h % group) * P.Tq + i;
  const int Lk = P.seqlens[b];
  const bool valid = !(Lk < 1 || Lk > P.Tk || Lk > P.bt_stride * P.page_size);
  unsigned* prow = A.pmask + (size_t)row * A.pm_words;
  if (!valid) {
    if (threadIdx.x == 0) tau_out[row] = INFINITY;
    if (threadIdx.x == 0 && P.row_nnz) P.row_nnz[row] = 0;
    for (int w = threadIdx.x; w < A.pm_words; w += TAU_THREADS) prow[w] = 0u;
    return;
  }
  const int npages = (Lk + P.page_size - 1) / P.page_size;
  const int nact = min(A.nsplit, (npages + A.pps - 1) / A.pps);
  const size_t pbase = (((size_t)b * P.Hkv + g) * A.nsplit) * A.R + r;
  float m = -INFINITY;
  for (int s = 0; s < nact; ++s) m = fmaxf(m, A.ml[(pbase + (size_t)s * A.R) * 2]);
  if (m == -INFINITY) {  // no visible key
    if (threadIdx.x == 0) tau_out[row] = INFINITY;
    if (threadIdx.x == 0 && P.row_nnz) P.row_nnz[row] = 0;
    for (int w = threadIdx.x; w < A.pm_words; w += TAU_THREADS) prow[w] = 0u;
    return;
  }
  if (threadIdx.x == 0) {
    s_n = 0;
    s_sup = 0;
  }
  for (int w = threadIdx.x; w < A.pm_words; w += TAU_THREADS) smask[w] = 0u;
  __syncthreads();
  const float* zrow = A.scores + (size_t)row * P.Tk;
  // candidates: one shared atomic per warp and batch of keys (ballot +
  // population count), four scores per thread per load where the row is
  // 16-byte aligned
  const unsigned lt = (1u << (threadIdx.x & 31)) - 1u;
  auto put = [&](bool in, float u, int j) {
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (bal == 0u) return;
    int base = 0;
    if ((threadIdx.x & 31) == __ffs(bal) - 1) base = atomicAdd(&s_n, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, __ffs(bal) - 1);
    if (in) {
      const int k = base + __popc(bal & lt);
      if (k < cap) {
        cand[k] = u;
        cidx[k] = j;
      }
    }
  };
  const float thr = m - 1.f;
  const bool vec = (reinterpret_cast<uintptr_t>(zrow) & 15u) == 0;
  const int nvec = vec ? Lk / 4 : 0;
  // every thread of a warp runs the same number of trips (ballots above)
  const int trips = (nvec + TAU_THREADS - 1) / TAU_THREADS;
  for (int t = 0; t < trips; ++t) {
    const int q = t * TAU_THREADS + threadIdx.x;
    float4 x = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    if (q < nvec) x = reinterpret_cast<const float4*>(zrow)[q];
    put(x.x > thr, x.x, 4 * q);
    put(x.y > thr, x.y, 4 * q + 1);
    put(x.z > thr, x.z, 4 * q + 2);
    put(x.w > thr, x.w, 4 * q + 3);
  }
  const int rest = Lk - 4 * nvec;
  const int trips1 = (rest + TAU_THREADS - 1) / TAU_THREADS;
  for (int t = 0; t < trips1; ++t) {
    const int j = 4 * nvec + t * TAU_THREADS + threadIdx.x;
    const float u = (j < Lk) ? zrow[j] : -INFINITY;
    put(u > thr, u, j);
  }
  __syncthreads();
  const int n = s_n;
  float tau;
  if (n <= cap) {
    tau = block_solve_tau(cand, n, m, P.norm == NATTN_ENTMAX15, red);
    // pages of the support: the support lies among the candidates
    for (int k = threadIdx.x; k < n; k += TAU_THREADS)
      if (cand[k] > tau) {
        const int pg = cidx[k] / P.page_size;
        atomicOr(&smask[pg >> 5], 1u << (pg & 31));
        atomicAdd(&s_sup, 1);
      }
  } else {
    // every masked score is -inf and never enters {u > t}
    tau = block_solve_tau(zrow, Lk, m, P.norm == NATTN_ENTMAX15, red);
    // too many candidates to track: every page of the row is visited
    for (int pg = threadIdx.x; pg < npages; pg += TAU_THREADS)
      atomicOr(&smask[pg >> 5], 1u << (pg & 31));
    for (int j = threadIdx.x; j < Lk; j += TAU_THREADS)
      if (zrow[j] > tau) atomicAdd(&s_sup, 1);
  }
  __syncthreads();
  if (threadIdx.x == 0 && P.row_nnz) P.row_nnz[row] = s_sup;
  for (int w = threadIdx.x; w < A.pm_words; w += TAU_THREADS) prow[w] = smask[w];
  if (threadIdx.x == 0) tau_out[row] = tau;
}

}  // namespace nattn
