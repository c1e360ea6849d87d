// Variation indicator (Method §1), density and block assignment (Method §2).
//
// zone_stats_kernel   one CTA per (zone, 128-channel slab): eight warps, one per
//                     time slice of the zone, stream the slab's 512 tokens once
//                     (coalesced 8/16-byte lane loads), accumulate the three
//                     axis-pooled sums in registers, combine them in shared
//                     memory and write the slab's sum over channels of the
//                     per-axis population variance.  HBM-bound: reads V once.
// zone_finish_kernel  one CTA per zone: sums the slab partials in a fixed
//                     order and pools the audio norms of the zone (double).
// zone_final_kernel   one CTA: grid maxima, then r, abar, vhat, g and rho.
// assign_blocks_kernel one CTA: B(m), l*, nearest candidate (double), block
//                     table via a block-wide scan.
#pragma once

#include "common.cuh"

namespace prism {

constexpr int kSlab = 128;  // channels per zone_stats CTA (32 lanes x 4)

template <typename Tin>
struct Load4;
template <>
struct Load4<__nv_bfloat16> {
  static __device__ __forceinline__ void run(const __nv_bfloat16 *p, float v[4]) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  }
};
template <>
struct Load4<float> {
  static __device__ __forceinline__ void run(const float *p, float v[4]) {
    const float4 u = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
};

// part[(m * nslab + slab) * 3 + d] = sum over the slab's channels c of
// (1/8) sum_i (Vbar^{(d)}_{i,c} - mu_c)^2.
// Each warp streams its time slice row by row with the next row's eight loads
// issued before the current row is summed (two rows in flight).  Its row sums
// (the H pool of the slice) go to shared memory as soon as a row is done, so
// only the T and W sums stay in registers; the cross-warp combines then run in
// warp order 0..7, the same order of float additions as a sequential sum.
template <typename Tin>
__global__ void __launch_bounds__(256, 2) zone_stats_kernel(const Tin *__restrict__ V, int C, int H, int W,
                                                         int ZY, int ZX, float *__restrict__ part) {
  __shared__ float sT[8][kSlab];      // [t][c]: slice sums, one warp per t
  __shared__ float sHw[8][8][kSlab];  // [t][y][c]: row sums of each slice
  __shared__ float sH[8][kSlab];      // [y][c]: summed over the eight warps in order
  __shared__ float sW[8][kSlab];      // [x][c]
  __shared__ float red[8][3];
  const int slab = blockIdx.x, m = blockIdx.y, nslab = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int zt = m / (ZY * ZX), zy = (m / ZX) % ZY, zx = m % ZX;
  const int c0 = slab * kSlab + lane * 4;
  const bool active = c0 < C;
  float accT[4] = {0, 0, 0, 0}, accW[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) accW[i][c] = 0.f;
  if (active) {
    const int64_t t = zt * kZone + warp;
    const Tin *base = V + ((t * H + zy * kZone) * W + zx * kZone) * (int64_t)C + c0;
    const int64_t row_stride = (int64_t)W * C;
    float v[2][8][4];
#pragma unroll
    for (int x = 0; x < 8; ++x) Load4<Tin>::run(base + x * (int64_t)C, v[0][x]);
#pragma unroll
    for (int y = 0; y < 8; ++y) {
      const int cur = y & 1;
      if (y + 1 < 8) {
#pragma unroll
        for (int x = 0; x < 8; ++x) Load4<Tin>::run(base + (y + 1) * row_stride + x * (int64_t)C, v[cur ^ 1][x]);
      }
      float accH[4] = {0, 0, 0, 0};
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          accT[c] += v[cur][x][c];
          accH[c] += v[cur][x][c];
          accW[x][c] += v[cur][x][c];
        }
#pragma unroll
      for (int c = 0; c < 4; ++c) sHw[warp][y][lane * 4 + c] = accH[c];
    }
  } else {
#pragma unroll
    for (int y = 0; y < 8; ++y)
#pragma unroll
      for (int c = 0; c < 4; ++c) sHw[warp][y][lane * 4 + c] = 0.f;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) sT[warp][lane * 4 + c] = accT[c];
  // fixed-order (warp 0, 1, ..., 7) accumulation of the W pools
  for (int w = 0; w < 8; ++w) {
    if (warp == w) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float w0 = w ? sW[i][lane * 4 + c] : 0.f;
          sW[i][lane * 4 + c] = w0 + accW[i][c];
        }
    }
    __syncthreads();
  }
  // H pools: row y summed over the warps in order 0..7
  for (int e = threadIdx.x; e < 8 * kSlab; e += blockDim.x) {
    const int y = e / kSlab, c = e % kSlab;
    float h = sHw[0][y][c];
#pragma unroll
    for (int w = 1; w < 8; ++w) h += sHw[w][y][c];
    sH[y][c] = h;
  }
  __syncthreads();
  // threads 0..127: channel c of the slab, all three axes
  float var[3] = {0, 0, 0};
  if (threadIdx.x < kSlab && slab * kSlab + (int)threadIdx.x < C) {
    const int c = threadIdx.x;
    float pt[8], ph[8], pw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pt[i] = sT[i][c] * (1.f / 64.f);
      ph[i] = sH[i][c] * (1.f / 64.f);
      pw[i] = sW[i][c] * (1.f / 64.f);
    }
    float mt = 0.f, mh = 0.f, mw = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) { mt += pt[i]; mh += ph[i]; mw += pw[i]; }
    mt *= 0.125f; mh *= 0.125f; mw *= 0.125f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      var[0] += (pt[i] - mt) * (pt[i] - mt);
      var[1] += (ph[i] - mh) * (ph[i] - mh);
      var[2] += (pw[i] - mw) * (pw[i] - mw);
    }
#pragma unroll
    for (int d = 0; d < 3; ++d) var[d] *= 0.125f;
  }
#pragma unroll
  for (int d = 0; d < 3; ++d) var[d] = warp_sum(var[d]);
  if (lane == 0)
#pragma unroll
    for (int d = 0; d < 3; ++d) red[warp][d] = var[d];
  __syncthreads();
  if (threadIdx.x < 3) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += red[w][threadIdx.x];
    part[((int64_t)m * nslab + slab) * 3 + threadIdx.x] = s;
  }
}

// Per-zone record (double): sigma2_v[3], info, amean, sigma2_a[3], amax.
constexpr int kZoneRec = 9;

__global__ void __launch_bounds__(64) zone_finish_kernel(const float *__restrict__ part, int nslab, int C,
                                                         const float *__restrict__ audio, int H, int W,
                                                         int ZY, int ZX, double *__restrict__ rec) {
  __shared__ double av[8][8][8];  // [t][y][x]
  const int m = blockIdx.x;
  const int zt = m / (ZY * ZX), zy = (m / ZX) % ZY, zx = m % ZX;
  if (audio) {
    const int t = threadIdx.x >> 3, y = threadIdx.x & 7;
    const int64_t row = ((int64_t)(zt * kZone + t) * H + zy * kZone + y) * W + zx * kZone;
#pragma unroll
    for (int x = 0; x < 8; ++x) av[t][y][x] = (double)audio[row + x];
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  double *r = rec + (int64_t)m * kZoneRec;
  double info = 0.0;
  for (int d = 0; d < 3; ++d) {
    double s = 0.0;
    for (int k = 0; k < nslab; ++k) s += (double)part[((int64_t)m * nslab + k) * 3 + d];
    r[d] = s / (double)C;
    info += r[d];
  }
  r[3] = info;
  double amean = 0.0, amax = 0.0, va[3] = {0.0, 0.0, 0.0};
  if (audio) {
    double pool[3][8];
    for (int i = 0; i < 8; ++i) pool[0][i] = pool[1][i] = pool[2][i] = 0.0;
    amax = av[0][0][0];
    for (int t = 0; t < 8; ++t)
      for (int y = 0; y < 8; ++y)
        for (int x = 0; x < 8; ++x) {
          const double a = av[t][y][x];
          pool[0][t] += a;
          pool[1][y] += a;
          pool[2][x] += a;
          amax = fmax(amax, a);
        }
    for (int i = 0; i < 8; ++i) amean += pool[0][i];
    amean /= 512.0;
    for (int d = 0; d < 3; ++d) {
      double s = 0.0;
      for (int i = 0; i < 8; ++i) {
        const double e = pool[d][i] / 64.0 - amean;
        s += e * e;
      }
      va[d] = s / 8.0;
    }
  }
  r[4] = amean;
  r[5] = va[0]; r[6] = va[1]; r[7] = va[2];
  r[8] = amax;
}

__global__ void __launch_bounds__(1024) zone_final_kernel(const double *__restrict__ rec, int Z, int has_audio,
                                                          float eps, float *__restrict__ g,
                                                          float *__restrict__ rho, float *__restrict__ debug) {
  __shared__ double s_imax[32], s_amax[32];
  double imax = 0.0, amax = 0.0;
  for (int m = threadIdx.x; m < Z; m += blockDim.x) {
    imax = fmax(imax, rec[(int64_t)m * kZoneRec + 3]);
    amax = fmax(amax, rec[(int64_t)m * kZoneRec + 8]);
  }
  imax = warp_max(imax);
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) {
    s_imax[threadIdx.x >> 5] = imax;
    s_amax[threadIdx.x >> 5] = amax;
  }
  __syncthreads();
  imax = 0.0;
  amax = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    imax = fmax(imax, s_imax[w]);
    amax = fmax(amax, s_amax[w]);
  }
  const bool audio_on = has_audio && amax > 0.0;
  for (int m = threadIdx.x; m < Z; m += blockDim.x) {
    const double *r = rec + (int64_t)m * kZoneRec;
    const double sv = r[0] + r[1] + r[2];
    const double sa = r[5] + r[6] + r[7];
    const double abar = audio_on ? r[4] / amax : 0.0;
    double gd[3], rv[3], vh[3];
    for (int d = 0; d < 3; ++d) {
      rv[d] = sv > 0.0 ? r[d] / sv : 0.0;
      vh[d] = (audio_on && sa > 0.0) ? r[5 + d] / sa : 0.0;
      gd[d] = rv[d] + abar * vh[d] + (double)eps;
      g[(int64_t)m * 3 + d] = (float)gd[d];
    }
    rho[m] = (float)(0.5 * ((imax > 0.0 ? r[3] / imax : 0.0) + abar));
    if (debug) {
      float *o = debug + (int64_t)m * 8;
      o[0] = (float)r[0]; o[1] = (float)r[1]; o[2] = (float)r[2];
      o[3] = (float)r[3]; o[4] = (float)abar;
      o[5] = (float)vh[0]; o[6] = (float)vh[1]; o[7] = (float)vh[2];
    }
  }
}

// Nearest candidate of volume B to l* (squared log2 distance, double); ties
// within 1e-9 resolve to the lowest canonical index.
__device__ __forceinline__ int quantise_shape(const double ell[3], int B) {
  const int first = shape_first(B), count = shape_count(B);
  double dist[7];
  double best = 1e300;
  for (int s = 0; s < count; ++s) {
    double d2 = 0.0;
    for (int a = 0; a < 3; ++a) {
      const double e = ell[a] - log2((double)shape_edge(first + s, a));
      d2 += e * e;
    }
    dist[s] = d2;
    best = fmin(best, d2);
  }
  for (int s = 0; s < count; ++s)
    if (dist[s] <= best + 1e-9) return first + s;
  return first;
}

// fixed > 0: every zone takes canonical shape fixed - 1 (g and rho unread).
__global__ void __launch_bounds__(1024) assign_blocks_kernel(const float *__restrict__ g,
                                                             const float *__restrict__ rho, int Z,
                                                             float tau128, float tau256, int fixed,
                                                             uint8_t *__restrict__ shape_id,
                                                             int32_t *__restrict__ zone_blk_base,
                                                             prism_block *__restrict__ blocks,
                                                             int32_t *__restrict__ nblk) {
  __shared__ int s_warp[32];
  __shared__ int s_carry;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  for (int m0 = 0; m0 < Z; m0 += blockDim.x) {
    const int m = m0 + threadIdx.x;
    int sid = 0, B = 0, nb = 0;
    if (m < Z && fixed > 0) {
      sid = fixed - 1;
      B = shape_volume(sid);
      nb = kZoneTokens / B;
    } else if (m < Z) {
      const float r = rho[m];
      B = r >= tau128 ? 64 : (r >= tau256 ? 128 : 256);
      const double S = log2((double)B);
      double lg[3], ell[3];
      for (int a = 0; a < 3; ++a) lg[a] = log2((double)g[(int64_t)m * 3 + a]);
      const double mean = (1.0 / 3.0) * (S + 0.5 * (lg[0] + lg[1] + lg[2]));
      for (int a = 0; a < 3; ++a) ell[a] = -0.5 * lg[a] + mean;
      sid = quantise_shape(ell, B);
      nb = kZoneTokens / B;
    }
    // block-wide inclusive scan of nb
    int v = nb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = lane < nwarp ? s_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += u;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const int incl = v + (warp > 0 ? s_warp[warp - 1] : 0) + s_carry;
    const int base = incl - nb;
    if (m < Z) {
      shape_id[m] = (uint8_t)sid;
      zone_blk_base[m] = base;
      for (int b = 0; b < nb; ++b) {
        prism_block blk;
        blk.start = m * kZoneTokens + b * B;
        blk.size = B;
        blk.zone = m;
        blk.shape = sid;
        blocks[base + b] = blk;
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    zone_blk_base[Z] = s_carry;
    *nblk = s_carry;
  }
}

}  // namespace prism
