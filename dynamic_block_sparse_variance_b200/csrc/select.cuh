// Hybrid top-k / top-p block selection (Method §3).
//
// block_scores_kernel  s_ij = scale * Qbar_i . Kbar_j for one pass of heads, a
//                      64x64-tiled fp32 SIMT product (the contraction is K = d
//                      deep and tiny next to the attention; fp32 keeps the
//                      ranking faithful).  Channels are summed in ascending
//                      order, so a score is a fixed function of its inputs.
// row_cut_kernel       one CTA per query block row: the row's keys in shared
//                      memory; max, softmax denominator, per-block masses in
//                      2^-40 fixed point (integer sums are order-free, hence
//                      deterministic); a value-binned histogram locates the bin
//                      where both "count >= min(k, nblk)" and "mass >= p" first
//                      hold; that bin's members are sorted exactly by (score
//                      desc, index asc) and walked to the cut.  A crossing
//                      bin with more members than the sort buffer is binned
//                      again over its own value range; scores packed so
//                      tightly that value bins stop separating them (many
//                      binades close to zero) are then binned by the bits of
//                      their 32-bit order keys, 10 bits a level, which ends in
//                      a single key (a run of equal scores, taken by index).
//                      The cut is stored as (key, number of equal keys taken).
// scan kernels         row counts -> CSR row_ptr and nnz (int64 checked
//                      against the column capacity).
// emit_kernel          one CTA per row: ascending indices of the selected
//                      blocks, written with block-wide scans.
#pragma once

#include "common.cuh"

namespace prism {

constexpr int kSelThreads = 512;
constexpr int kSelBins = 1024;
constexpr int kSelList = 2048;       // exact-sort buffer for the crossing bin
constexpr int kSelMaxLevels = 6;     // value-range refinements
constexpr int kSelKeyLevels = 5;     // then order-key refinements, 10 bits a level: 4 reach one key, the 5th takes a run of equal keys
constexpr double kMassOne = 1099511627776.0;  // 2^40

// Order-preserving map: ascending key <=> descending score.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~ord;
}
__device__ __forceinline__ float key_score(uint32_t key) {
  const uint32_t ord = ~key;
  const uint32_t u = (ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord;
  return __uint_as_float(u);
}
__device__ __forceinline__ unsigned long long block_mass(float s, float smax, float invZ) {
  const float P = __expf(s - smax) * invZ;
  return __double2ull_rn((double)P * kMassOne);
}

__global__ void __launch_bounds__(256) block_scores_kernel(const float *__restrict__ qb,
                                                           const float *__restrict__ kb, int D, int64_t cap,
                                                           const int32_t *__restrict__ nblk_p, int h0,
                                                           float scale, float *__restrict__ S) {
  __shared__ float Qs[32][65];
  __shared__ float Ks[32][65];
  const int n = *nblk_p;
  const int j0 = blockIdx.x * 64, i0 = blockIdx.y * 64, hl = blockIdx.z, h = h0 + hl;
  if (i0 >= n || j0 >= n) return;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float *qh = qb + (int64_t)h * cap * D;
  const float *kh = kb + (int64_t)h * cap * D;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int c0 = 0; c0 < D; c0 += 32) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = (threadIdx.x >> 3) + 32 * r, c4 = (threadIdx.x & 7) * 4;
      float4 qv = make_float4(0, 0, 0, 0), kv = make_float4(0, 0, 0, 0);
      if (i0 + row < n) qv = *reinterpret_cast<const float4 *>(qh + (int64_t)(i0 + row) * D + c0 + c4);
      if (j0 + row < n) kv = *reinterpret_cast<const float4 *>(kh + (int64_t)(j0 + row) * D + c0 + c4);
      Qs[c4 + 0][row] = qv.x; Qs[c4 + 1][row] = qv.y; Qs[c4 + 2][row] = qv.z; Qs[c4 + 3][row] = qv.w;
      Ks[c4 + 0][row] = kv.x; Ks[c4 + 1][row] = kv.y; Ks[c4 + 2][row] = kv.z; Ks[c4 + 3][row] = kv.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = Qs[c][ty * 4 + q];
        b[q] = Ks[c][tx + 16 * q];
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[q][r] = fmaf(a[q], b[r], acc[q][r]);
    }
    __syncthreads();
  }
  float *Sh = S + (int64_t)hl * cap * cap;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + ty * 4 + q;
    if (i >= n) continue;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = j0 + tx + 16 * r;
      if (j < n) Sh[(int64_t)i * cap + j] = acc[q][r] * scale;
    }
  }
}

// Block-wide reductions for kSelThreads threads (fixed order).
template <typename T, typename Op>
__device__ __forceinline__ T sel_reduce(T v, T *scratch, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = scratch[0];
  for (int w = 1; w < kSelThreads / 32; ++w) r = op(r, scratch[w]);
  __syncthreads();
  return r;
}

struct SelShared {
  unsigned int hc[kSelBins];
  unsigned long long hm[kSelBins];
  unsigned long long list[kSelList];
  float fred[kSelThreads / 32];
  unsigned long long ured[kSelThreads / 32];
  unsigned int kred[kSelThreads / 32];
  unsigned int list_n;
  unsigned int kmin, kmax;
  int bin;
  unsigned int cnt_bin;
  unsigned long long cnt_before, mass_before;
};

__global__ void __launch_bounds__(kSelThreads) row_cut_kernel(const float *__restrict__ S, int64_t cap,
                                                             const int32_t *__restrict__ nblk_p, int h0,
                                                             int top_k, float sparsity, float top_p,
                                                             int32_t *__restrict__ cnt,
                                                             uint32_t *__restrict__ cut_key,
                                                             int32_t *__restrict__ cut_q) {
  extern __shared__ uint32_t keys[];
  __shared__ SelShared sh;
  const int n = *nblk_p;
  const int i = blockIdx.x, hl = blockIdx.y;
  const int64_t row = (int64_t)(h0 + hl) * cap + i;
  if (i >= n) {
    if (threadIdx.x == 0) {
      cnt[row] = 0;
      cut_key[row] = 0u;
      cut_q[row] = 0;
    }
    return;
  }
  const float *Srow = S + ((int64_t)hl * cap + i) * cap;
  float smax = -INFINITY;
  for (int j = threadIdx.x; j < n; j += kSelThreads) {
    const float s = Srow[j];
    keys[j] = score_key(s);
    smax = fmaxf(smax, s);
  }
  smax = sel_reduce(smax, sh.fred, [](float a, float b) { return fmaxf(a, b); });
  float z = 0.f;
  for (int j = threadIdx.x; j < n; j += kSelThreads) z += __expf(key_score(keys[j]) - smax);
  z = sel_reduce(z, sh.fred, [](float a, float b) { return a + b; });
  const float invZ = 1.f / z;
  unsigned long long tot = 0;
  for (int j = threadIdx.x; j < n; j += kSelThreads) tot += block_mass(key_score(keys[j]), smax, invZ);
  tot = sel_reduce(tot, sh.ured, [](unsigned long long a, unsigned long long b) { return a + b; });
  const unsigned long long pf = __double2ull_rn((double)top_p * kMassOne);
  // k: absolute, or the ratio form ceil((1 - sparsity) * nblk), at least 1
  const int k_eff = sparsity > 0.f ? max(1, (int)ceil((1.0 - (double)sparsity) * (double)n)) : top_k;
  const unsigned long long kk = (unsigned long long)min(k_eff, n);
  // top-p never reached, or p >= 1 (every probability is positive, so only
  // the whole row has mass 1 exactly): the whole row
  if (tot < pf || top_p >= 1.f) {
    if (threadIdx.x == 0) {
      cnt[row] = n;
      cut_key[row] = 0xffffffffu;
      cut_q[row] = 0;
    }
    return;
  }
  // Members of the current level: keys in [klo, khi].
  uint32_t klo = 0u, khi = 0xfffffffeu;
  unsigned long long cnt_before = 0, mass_before = 0;
  for (int level = 0; level < kSelMaxLevels + kSelKeyLevels; ++level) {
    // value range of the members
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j = threadIdx.x; j < n; j += kSelThreads) {
      const uint32_t k = keys[j];
      if (k >= klo && k <= khi) {
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
    kmin = sel_reduce(kmin, sh.kred, [](uint32_t a, uint32_t b) { return min(a, b); });
    kmax = sel_reduce(kmax, sh.kred, [](uint32_t a, uint32_t b) { return max(a, b); });
    const float vhi = key_score(kmin), vlo = key_score(kmax);
    const bool all_equal = kmin == kmax;
    const float inv_w = all_equal ? 0.f : (float)kSelBins / (vhi - vlo);
    // bins: equal slices of the value range, or (after kSelMaxLevels) of the
    // key range; both are monotone in the key, so a bin's members are a
    // contiguous key range and bins ascend with descending score
    const bool by_key = level >= kSelMaxLevels;
    const int kshift = all_equal ? 0 : max(0, 22 - __clz(kmax - kmin));   // (kmax - kmin) >> kshift < 1024
    auto bin_of = [&](uint32_t k) -> int {
      if (all_equal) return 0;
      if (by_key) return (int)((k - kmin) >> kshift);
      return min(kSelBins - 1, (int)((vhi - key_score(k)) * inv_w));
    };
    for (int b = threadIdx.x; b < kSelBins; b += kSelThreads) {
      sh.hc[b] = 0u;
      sh.hm[b] = 0ull;
    }
    if (threadIdx.x == 0) sh.list_n = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += kSelThreads) {
      const uint32_t k = keys[j];
      if (k >= klo && k <= khi) {
        const int b = bin_of(k);
        atomicAdd(&sh.hc[b], 1u);
        atomicAdd(&sh.hm[b], block_mass(key_score(k), smax, invZ));
      }
    }
    __syncthreads();
    // first bin (ascending = descending score) where both conditions hold
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      constexpr int per = kSelBins / 32;
      unsigned long long lc = 0, lm = 0;
      for (int b = lane * per; b < (lane + 1) * per; ++b) {
        lc += sh.hc[b];
        lm += sh.hm[b];
      }
      unsigned long long ec = lc, em = lm;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long uc = __shfl_up_sync(0xffffffffu, ec, o);
        const unsigned long long um = __shfl_up_sync(0xffffffffu, em, o);
        if (lane >= o) {
          ec += uc;
          em += um;
        }
      }
      ec -= lc;
      em -= lm;
      unsigned long long cc = cnt_before + ec, mm = mass_before + em;
      int found = -1;
      unsigned long long fc = 0, fm = 0;
      for (int b = lane * per; b < (lane + 1) * per; ++b) {
        const unsigned long long c1 = cc + sh.hc[b], m1 = mm + sh.hm[b];
        if (found < 0 && sh.hc[b] && c1 >= kk && m1 >= pf) {
          found = b;
          fc = cc;
          fm = mm;
        }
        cc = c1;
        mm = m1;
      }
      const unsigned ball = __ballot_sync(0xffffffffu, found >= 0);
      const int src = ball ? __ffs(ball) - 1 : 31;
      const int fb = __shfl_sync(0xffffffffu, found, src);
      fc = __shfl_sync(0xffffffffu, fc, src);
      fm = __shfl_sync(0xffffffffu, fm, src);
      if (lane == 0) {
        sh.bin = ball ? fb : -1;
        sh.cnt_before = fc;
        sh.mass_before = fm;
        sh.cnt_bin = ball ? sh.hc[fb] : 0u;
      }
    }
    __syncthreads();
    const int fb = sh.bin;
    if (fb < 0) {  // cannot happen when tot >= pf; latch and fall back to the whole row
      if (threadIdx.x == 0) {
        set_status(PRISM_EBOUNDS);
        cnt[row] = n;
        cut_key[row] = 0xffffffffu;
        cut_q[row] = 0;
      }
      return;
    }
    cnt_before = sh.cnt_before;
    mass_before = sh.mass_before;
    const unsigned int nb = sh.cnt_bin;
    if (all_equal) {
      // every member has the same score (and mass): take q of them by index
      const unsigned long long mt = block_mass(vhi, smax, invZ);
      unsigned long long q1 = kk > cnt_before ? kk - cnt_before : 1ull;
      unsigned long long q2 = 1ull;
      if (pf > mass_before && mt > 0) q2 = (pf - mass_before + mt - 1) / mt;
      unsigned long long q = max(max(q1, q2), 1ull);
      q = min(q, (unsigned long long)nb);
      if (threadIdx.x == 0) {
        cnt[row] = (int32_t)(cnt_before + q);
        cut_key[row] = kmin;
        cut_q[row] = (int32_t)q;
      }
      return;
    }
    // key range of the crossing bin's members
    uint32_t bmin = 0xffffffffu, bmax = 0u;
    for (int j = threadIdx.x; j < n; j += kSelThreads) {
      const uint32_t k = keys[j];
      if (k >= klo && k <= khi) {
        const int b = bin_of(k);
        if (b == fb) {
          bmin = min(bmin, k);
          bmax = max(bmax, k);
        }
      }
    }
    bmin = sel_reduce(bmin, sh.kred, [](uint32_t a, uint32_t b) { return min(a, b); });
    bmax = sel_reduce(bmax, sh.kred, [](uint32_t a, uint32_t b) { return max(a, b); });
    if (nb <= (unsigned)kSelList) {
      // collect (key, index), sort ascending, walk to the cut
      for (int j = threadIdx.x; j < n; j += kSelThreads) {
        const uint32_t k = keys[j];
        if (k >= bmin && k <= bmax) {
          const unsigned int pos = atomicAdd(&sh.list_n, 1u);
          sh.list[pos] = ((unsigned long long)k << 32) | (unsigned)j;
        }
      }
      __syncthreads();
      int len = 1;
      while (len < (int)nb) len <<= 1;
      for (int t = nb + threadIdx.x; t < len; t += kSelThreads) sh.list[t] = ~0ull;
      __syncthreads();
      for (int size = 2; size <= len; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int t = threadIdx.x; t < len; t += kSelThreads) {
            const int u = t ^ stride;
            if (u > t) {
              const bool up = (t & size) == 0;
              const unsigned long long a = sh.list[t], b = sh.list[u];
              if ((a > b) == up) {
                sh.list[t] = b;
                sh.list[u] = a;
              }
            }
          }
          __syncthreads();
        }
      }
      if (threadIdx.x == 0) {
        unsigned long long cc = cnt_before, mm = mass_before;
        unsigned int pos = 0;
        for (; pos < nb; ++pos) {
          const uint32_t k = (uint32_t)(sh.list[pos] >> 32);
          cc += 1;
          mm += block_mass(key_score(k), smax, invZ);
          if (cc >= kk && mm >= pf) break;
        }
        if (pos >= nb) pos = nb - 1;  // unreachable: the bin satisfies both conditions
        const uint32_t ck = (uint32_t)(sh.list[pos] >> 32);
        int q = 0;
        for (unsigned int t = 0; t <= pos; ++t) q += ((uint32_t)(sh.list[t] >> 32) == ck);
        cnt[row] = (int32_t)(cnt_before + pos + 1);
        cut_key[row] = ck;
        cut_q[row] = q;
      }
      return;
    }
    // too many members: refine inside the crossing bin
    klo = bmin;
    khi = bmax;
    __syncthreads();
  }
  if (threadIdx.x == 0) {  // unreachable (the key levels end in one key): latch, keep the whole row
    set_status(PRISM_EBOUNDS);
    cnt[row] = n;
    cut_key[row] = 0xffffffffu;
    cut_q[row] = 0;
  }
}

// ---- row counts -> row_ptr ------------------------------------------------
constexpr int kScanThreads = 1024, kScanPer = 4, kScanChunk = kScanThreads * kScanPer;

template <typename T>
__device__ __forceinline__ T block_excl_scan(T v, T *warp_tot, T *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T u = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += u;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    T w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : (T)0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const T u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  const T excl = x - v + (warp > 0 ? warp_tot[warp - 1] : (T)0);
  if (total) *total = warp_tot[(blockDim.x >> 5) - 1];
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kScanThreads) scan_partial_kernel(const int32_t *__restrict__ cnt, int64_t R,
                                                                   long long *__restrict__ part) {
  __shared__ long long wt[32];
  long long s = 0;
  const int64_t base = (int64_t)blockIdx.x * kScanChunk + (int64_t)threadIdx.x * kScanPer;
#pragma unroll
  for (int e = 0; e < kScanPer; ++e)
    if (base + e < R) s += cnt[base + e];
  long long tot;
  block_excl_scan<long long>(s, wt, &tot);
  if (threadIdx.x == 0) part[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(kScanThreads) scan_top_kernel(long long *__restrict__ part, int nchunk,
                                                               int64_t col_capacity,
                                                               int64_t *__restrict__ nnz) {
  __shared__ long long wt[32];
  __shared__ long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int c0 = 0; c0 < nchunk; c0 += kScanThreads) {
    const int c = c0 + threadIdx.x;
    const long long v = c < nchunk ? part[c] : 0;
    long long tot;
    const long long ex = block_excl_scan<long long>(v, wt, &tot);
    if (c < nchunk) part[c] = carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *nnz = carry;
    if (carry > col_capacity || carry > 0x7fffffffLL) set_status(PRISM_ECAPACITY);
  }
}

// On overflow (nnz > capacity) every row is left empty, so that no consumer
// indexes past the column array; the latched status reports the overflow.
__global__ void __launch_bounds__(kScanThreads) scan_final_kernel(const int32_t *__restrict__ cnt, int64_t R,
                                                                 const long long *__restrict__ part,
                                                                 const int64_t *__restrict__ nnz,
                                                                 int64_t capacity,
                                                                 int32_t *__restrict__ row_ptr) {
  __shared__ long long wt[32];
  const int64_t base = (int64_t)blockIdx.x * kScanChunk + (int64_t)threadIdx.x * kScanPer;
  const bool overflow = *nnz > capacity || *nnz > 0x7fffffffLL;
  long long v[kScanPer], s = 0;
#pragma unroll
  for (int e = 0; e < kScanPer; ++e) {
    v[e] = (base + e < R && !overflow) ? cnt[base + e] : 0;
    s += v[e];
  }
  long long tot;
  long long ex = block_excl_scan<long long>(s, wt, &tot) + (overflow ? 0 : part[blockIdx.x]);
#pragma unroll
  for (int e = 0; e < kScanPer; ++e) {
    if (base + e < R) row_ptr[base + e] = (int32_t)ex;
    ex += v[e];
  }
  if (base + kScanPer >= R && base < R) row_ptr[R] = (int32_t)ex;
}

__global__ void __launch_bounds__(kSelThreads) emit_kernel(const float *__restrict__ S, int64_t cap,
                                                          const int32_t *__restrict__ nblk_p, int h0,
                                                          const uint32_t *__restrict__ cut_key,
                                                          const int32_t *__restrict__ cut_q,
                                                          const int32_t *__restrict__ row_ptr,
                                                          const int64_t *__restrict__ nnz,
                                                          int64_t col_capacity, int32_t *__restrict__ col) {
  __shared__ int wt[32];
  __shared__ int s_tie, s_out;
  const int n = *nblk_p;
  const int i = blockIdx.x, hl = blockIdx.y;
  if (i >= n || *nnz > col_capacity || *nnz > 0x7fffffffLL) return;
  const int64_t row = (int64_t)(h0 + hl) * cap + i;
  const uint32_t ck = cut_key[row];
  const int q = cut_q[row];
  const float *Srow = S + ((int64_t)hl * cap + i) * cap;
  int32_t *out = col + row_ptr[row];
  if (threadIdx.x == 0) {
    s_tie = 0;
    s_out = 0;
  }
  __syncthreads();
  for (int j0 = 0; j0 < n; j0 += kSelThreads) {
    const int j = j0 + threadIdx.x;
    uint32_t k = 0xffffffffu;
    if (j < n) k = score_key(Srow[j]);
    const int tie = (j < n && k == ck) ? 1 : 0;
    int tie_tot;
    const int tie_rank = block_excl_scan<int>(tie, wt, &tie_tot) + s_tie;
    const int sel = (j < n && (k < ck || (tie && tie_rank < q))) ? 1 : 0;
    int sel_tot;
    const int pos = block_excl_scan<int>(sel, wt, &sel_tot) + s_out;
    if (sel) out[pos] = j;
    __syncthreads();
    if (threadIdx.x == 0) {
      s_tie += tie_tot;
      s_out += sel_tot;
    }
    __syncthreads();
  }
}

}  // namespace prism
