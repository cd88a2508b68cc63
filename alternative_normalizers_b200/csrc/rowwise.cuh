// Row-at-a-time attention on CUDA cores.
//
// One CTA owns one query row at a time: it materialises the row's allowed
// scores (in shared memory, or in a per-CTA global slot for very long rows),
// applies the row normalizer, optionally writes the dense weights, and
// accumulates O = p V.  It serves three purposes:
//   * the dense-weights request of the backend contract ("Attention",
//     factory.ai transformers wiki: output plus optional weights),
//   * small problems and head dims the tensor-core kernels do not take,
//   * the sparse prefill rows whose support overflowed the phase-1 buffer.
#pragma once

#include "common.cuh"
#include "problem.cuh"

namespace nattn {

constexpr int ROW_THREADS = 256;
constexpr int ROW_WARPS = ROW_THREADS / 32;

struct Red4 {
  float a, b, c, d;
};

// Block-wide reduction of (sum, sum, sum, min).
__device__ __forceinline__ Red4 block_red4(Red4 v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v.a = warp_sum(v.a);
  v.b = warp_sum(v.b);
  v.c = warp_sum(v.c);
  v.d = warp_min(v.d);
  __syncthreads();
  if (lane == 0) {
    red[warp * 4 + 0] = v.a;
    red[warp * 4 + 1] = v.b;
    red[warp * 4 + 2] = v.c;
    red[warp * 4 + 3] = v.d;
  }
  __syncthreads();
  Red4 r{0.f, 0.f, 0.f, INFINITY};
#pragma unroll
  for (int w = 0; w < ROW_WARPS; ++w) {
    r.a += red[w * 4 + 0];
    r.b += red[w * 4 + 1];
    r.c += red[w * 4 + 2];
    r.d = fminf(r.d, red[w * 4 + 3]);
  }
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = -INFINITY;
#pragma unroll
  for (int w = 0; w < ROW_WARPS; ++w) r = fmaxf(r, red[w]);
  return r;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < ROW_WARPS; ++w) r += red[w];
  return r;
}

// Exact threshold of sparsemax / 1.5-entmax over sc[0..n) (values already in
// threshold units u: z for sparsemax, z/2 for entmax), with u_max = m.
//
// Newton's method from the left on g(t) = sum relu(u - t)^k (k = 1 or 2),
// which is convex and decreasing, so every iterate stays at or below the root
// and the set {u > t} always contains the support.  At each iterate the
// closed-form threshold of that set is tried first and accepted as soon as
// it satisfies the optimality conditions (every member above it, every
// other entry at or below it); for sparsemax this is Michelot's projection
// algorithm.  Work is done in the shifted variable w = u - m for accuracy.
__device__ float block_solve_tau(const float* sc, int n, float m, bool entmax,
                                 float* red) {
  float t = -1.0f;  // g(-1) >= 1 since the maximum contributes 1
  for (int it = 0; it < 64; ++it) {
    Red4 acc{0.f, 0.f, 0.f, INFINITY};
    for (int j = threadIdx.x; j < n; j += ROW_THREADS) {
      const float w = sc[j] - m;
      if (w > t) {
        acc.a += 1.f;
        acc.b += w;
        acc.c += w * w;
        acc.d = fminf(acc.d, w);
      }
    }
    const Red4 r = block_red4(acc, red);
    if (tau_step(r.a, r.b, r.c, r.d, entmax, t) != 0) break;
  }
  return t + m;
}

// One CTA per query row (grid-stride over rows).  Dynamic shared memory:
// q as float [256] | reduction scratch [64] | column partials
// [ROW_WARPS * 256] | scores [cap].
__global__ void __launch_bounds__(ROW_THREADS)
    rowwise_kernel(Problem P, const int* __restrict__ row_list,
                   const int* __restrict__ row_count, int nrows_static, int cap,
                   float* __restrict__ gslots) {
  extern __shared__ float smem_f[];
  __shared__ int s_ncand;
  float* qf = smem_f;
  float* red = qf + 256;
  float* part = red + 64;
  float* sc_smem = part + ROW_WARPS * 256;
  const int tid = threadIdx.x;
  const int nrows = row_count ? *row_count : nrows_static;
  const int group = P.Hq / P.Hkv;

  for (int r = blockIdx.x; r < nrows; r += gridDim.x) {
    const int flat = row_list ? row_list[r] : r;
    int b, h, i;
    if (P.cu_q != nullptr) {
      // packed rows are [total_q][Hq]: the token's sequence by binary search
      const int tok = flat / P.Hq;
      h = flat % P.Hq;
      int lo = 0, hi = P.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.cu_q[mid] <= tok) lo = mid; else hi = mid - 1;
      }
      b = lo;
      i = tok - P.cu_q[b];
    } else {
      i = flat % P.Tq;
      h = (flat / P.Tq) % P.Hq;
      b = flat / (P.Tq * P.Hq);
    }
    const int g = h / group;
    bool bad = false;
    const SeqInfo sq = seq_info(P, b);  // out-of-range lengths: an empty row
    const RowRange rr = row_range(sq.Lq, P.causal, P.window, i, sq.Lk);
    int n = rr.hi - rr.lo + 1;
    if (n < 0) n = 0;
    float* sc = sc_smem;
    if (n > cap) {
      if (gslots == nullptr) {
        bad = true;
        n = 0;
      } else {
        sc = gslots + (size_t)blockIdx.x * P.Tk;
      }
    }
    bf16* orow = P.out + (size_t)flat * P.dv;
    for (int c = tid; c < P.d; c += ROW_THREADS)
      qf[c] = __bfloat162float(P.q[(size_t)flat * P.d + c]);
    __syncthreads();

    // scores z_j for the allowed keys, in units fixed by the normalizer.
    // Eight lanes share one key row (16-byte loads, coalesced), four keys
    // per warp and KU keys per lane group in flight.
    const float uscale = (P.norm == NATTN_ENTMAX15) ? 0.5f : 1.0f;
    int badkey = 0;
    {
      constexpr int KU = 4;
      constexpr int STEP = ROW_WARPS * 4;  // keys per pass of all warps
      const int lane = tid & 31, sub = lane & 7;
      const int nc8 = P.d / 8;  // 16-byte chunks per key row (at most 32)
      // the loop bound is the warp's first key, so every lane of a warp runs
      // the same iterations (the shuffles below need all 32 lanes)
      for (int wb = (tid >> 5) * 4; wb < n; wb += STEP * KU) {
        const int base = wb + (lane >> 3);
        uint4 x[KU][4];
#pragma unroll
        for (int u = 0; u < KU; ++u) {
          const int jj = base + u * STEP;
          bool kb = false;
          const uint4* k4 = nullptr;
          if (jj < n) {
            k4 = reinterpret_cast<const uint4*>(key_row(P, P.k, P.d, b, g, rr.lo + jj, kb));
            if (kb) {
              badkey = 1;
              k4 = nullptr;
            }
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c8 = sub + 8 * t;
            x[u][t] = (k4 != nullptr && c8 < nc8) ? k4[c8] : make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int u = 0; u < KU; ++u) {
          float s = 0.f;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c8 = sub + 8 * t;
            if (c8 < nc8) {
              const float* qq = qf + c8 * 8;
              const uint4 y = x[u][t];
              s += qq[0] * bf16lo(y.x) + qq[1] * bf16hi(y.x) + qq[2] * bf16lo(y.y) +
                   qq[3] * bf16hi(y.y) + qq[4] * bf16lo(y.z) + qq[5] * bf16hi(y.z) +
                   qq[6] * bf16lo(y.w) + qq[7] * bf16hi(y.w);
            }
          }
          s += __shfl_xor_sync(0xffffffffu, s, 1);
          s += __shfl_xor_sync(0xffffffffu, s, 2);
          s += __shfl_xor_sync(0xffffffffu, s, 4);
          const int jj = base + u * STEP;
          if (sub == 0 && jj < n) {
            float z = s * P.scale;
            if (P.softcap > 0.f) z = P.softcap * tanhf(z / P.softcap);
            // a key in a block the block mask drops is not visible
            if (!block_kept(P, b, h, i >> 7, (rr.lo + jj) >> 7)) z = -INFINITY;
            sc[jj] = z * uscale;
          }
        }
      }
    }
    if (__syncthreads_or(badkey)) bad = true;
    if (bad) {
      set_status(NATTN_EBOUNDS);
      n = 0;
    }

    // normalizer: overwrite scores with weights
    float stat;
    // softmax / softmax1: every visible key (of the blocks a block mask keeps)
    int nnz = n;
    if (P.block_mask != nullptr && n > 0) {
      nnz = 0;
      for (int kb = rr.lo >> 7; kb <= (rr.hi >> 7); ++kb)
        if (block_kept(P, b, h, i >> 7, kb))
          nnz += min(rr.hi, kb * 128 + 127) - max(rr.lo, kb * 128) + 1;
    }
    if (P.norm == NATTN_SOFTMAX || P.norm == NATTN_SOFTMAX1) {
      float mx = -INFINITY;
      for (int jj = tid; jj < n; jj += ROW_THREADS) mx = fmaxf(mx, sc[jj]);
      mx = block_max(mx, red);
      const float sink = sink_logit(P, h);  // -inf: no sink
      mx = fmaxf(mx, sink);
      const float msafe = (mx == -INFINITY) ? 0.f : mx;
      float l = 0.f;
      for (int jj = tid; jj < n; jj += ROW_THREADS) {
        const float e = expf(sc[jj] - msafe);
        sc[jj] = e;
        l += e;
      }
      l = block_sum(l, red);
      if (sink != -INFINITY) l += expf(sink - msafe);
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      for (int jj = tid; jj < n; jj += ROW_THREADS) sc[jj] *= inv;
      stat = (l > 0.f) ? msafe + logf(l) : -INFINITY;
    } else {
      const bool ent = P.norm == NATTN_ENTMAX15;
      float mx = -INFINITY;
      for (int jj = tid; jj < n; jj += ROW_THREADS) mx = fmaxf(mx, sc[jj]);
      mx = block_max(mx, red);
      // the threshold is at least max - 1 (in threshold units), so the solve
      // runs over the keys within one unit of the maximum, gathered into the
      // column-partials area (free until the PV), unless there are too many
      float tau = INFINITY;
      if (n > 0 && mx != -INFINITY) {  // -inf: every key dropped by the block mask
        float* cand = part;
        constexpr int kCandCap = ROW_WARPS * 256;
        if (tid == 0) s_ncand = 0;
        __syncthreads();
        for (int jj = tid; jj < n; jj += ROW_THREADS) {
          const float u = sc[jj];
          if (u > mx - 1.f) {
            const int k = atomicAdd(&s_ncand, 1);
            if (k < kCandCap) cand[k] = u;
          }
        }
        __syncthreads();
        const int nc = s_ncand;
        tau = (nc <= kCandCap) ? block_solve_tau(cand, nc, mx, ent, red)
                               : block_solve_tau(sc, n, mx, ent, red);
      }
      __syncthreads();
      float cnt = 0.f;
      for (int jj = tid; jj < n; jj += ROW_THREADS) {
        const float t = fmaxf(sc[jj] - tau, 0.f);
        sc[jj] = ent ? t * t : t;
        cnt += (t > 0.f) ? 1.f : 0.f;
      }
      nnz = (int)block_sum(cnt, red);
      stat = tau;
    }
    __syncthreads();

    if (P.weights) {
      float* wrow = P.weights + (size_t)flat * P.Tk;
      for (int j = tid; j < P.Tk; j += ROW_THREADS) {
        const int jj = j - rr.lo;
        wrow[j] = (jj >= 0 && jj < n) ? sc[jj] : 0.f;
      }
    }

    if (P.norm == NATTN_SOFTMAX || P.norm == NATTN_SOFTMAX1) {
      // O = p V: thread (grp, c) sums keys grp, grp + G, ... for column c
      const int G = ROW_THREADS / P.dv;
      const int c = tid % P.dv, grp = tid / P.dv;
      float acc = 0.f;
      if (grp < G) {
        for (int jj = grp; jj < n; jj += G) {
          const float p = sc[jj];
          if (p != 0.f) {
            bool kb = false;
            const bf16* vp = key_row(P, P.v, P.dv, b, g, rr.lo + jj, kb);
            acc += p * __bfloat162float(vp[c]);
          }
        }
      }
      __syncthreads();
      if (grp < G) part[grp * P.dv + c] = acc;
      __syncthreads();
      if (tid < P.dv) {
        float o = 0.f;
        for (int q2 = 0; q2 < G; ++q2) o += part[q2 * P.dv + tid];
        orow[tid] = __float2bfloat16_rn(o);
      }
    } else {
      // sparse weights: each warp scans its slice of the keys 32 at a time
      // and, for every nonzero weight a ballot finds, adds the whole V row
      // (lane c holds columns c, c + 32, ...); the warps' sums are then added
      const int lane = tid & 31, wrp = tid >> 5;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      const int per = (n + ROW_WARPS - 1) / ROW_WARPS;
      const int j0 = wrp * per, j1 = min(n, j0 + per);
      for (int jb = j0; jb < j1; jb += 32) {
        const int jj = jb + lane;
        const float p = (jj < j1) ? sc[jj] : 0.f;
        unsigned nz = __ballot_sync(0xffffffffu, p != 0.f);
        while (nz) {
          const int src = __ffs(nz) - 1;
          nz &= nz - 1;
          const float pj = __shfl_sync(0xffffffffu, p, src);
          bool kb = false;
          const bf16* vp = key_row(P, P.v, P.dv, b, g, rr.lo + jb + src, kb);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = lane + 32 * i;
            if (c < P.dv) acc[i] += pj * __bfloat162float(vp[c]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = lane + 32 * i;
        if (c < P.dv) part[wrp * 256 + c] = acc[i];
      }
      __syncthreads();
      if (tid < P.dv) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < ROW_WARPS; ++w) o += part[w * 256 + tid];
        orow[tid] = __float2bfloat16_rn(o);
      }
    }
    if (tid == 0 && P.row_stat) P.row_stat[flat] = stat;
    if (tid == 0 && P.row_nnz) P.row_nnz[flat] = nnz;
    __syncthreads();
  }
}

}  // namespace nattn
