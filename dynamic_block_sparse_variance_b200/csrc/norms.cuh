// Per-token Euclidean norms of the audio-to-video cross-attention output
// (Method §1: a = ||h_hat||_2, the indicator's audio input).  HBM-bound: each
// row is read once with 16-byte streaming loads, one warp per row, several
// loads in flight per lane; squares are summed in float in a fixed order
// (lane-strided, then a butterfly), so the result is deterministic.
#pragma once

#include "common.cuh"

namespace prism {

constexpr int kNormThreads = 256;

__device__ __forceinline__ float sum_sq(uint4 v, const __nv_bfloat16 *) {
  float s = 0.f;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = bf16_lo(w[i]), hi = bf16_hi(w[i]);
    s = fmaf(lo, lo, s);
    s = fmaf(hi, hi, s);
  }
  return s;
}
__device__ __forceinline__ float sum_sq(uint4 v, const float *) {
  const float a = __uint_as_float(v.x), b = __uint_as_float(v.y), c = __uint_as_float(v.z),
              d = __uint_as_float(v.w);
  return fmaf(d, d, fmaf(c, c, fmaf(b, b, a * a)));
}

template <typename T>
__global__ void __launch_bounds__(kNormThreads) audio_norms_kernel(const T *__restrict__ h, int64_t N, int C,
                                                                   float *__restrict__ a) {
  constexpr int kUnroll = 4;
  const int lane = threadIdx.x & 31;
  const int nvec = C / (16 / (int)sizeof(T));
  const int64_t wpb = kNormThreads / 32;
  const int64_t stride = (int64_t)gridDim.x * wpb;
  for (int64_t n = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); n < N; n += stride) {
    const uint4 *row = reinterpret_cast<const uint4 *>(h + n * (int64_t)C);
    float acc[kUnroll] = {0.f, 0.f, 0.f, 0.f};
    int v = lane;
    for (; v + 32 * (kUnroll - 1) < nvec; v += 32 * kUnroll) {
      uint4 x[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) x[u] = __ldcs(row + v + 32 * u);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) acc[u] += sum_sq(x[u], h);
    }
    for (; v < nvec; v += 32) acc[0] += sum_sq(__ldcs(row + v), h);
    const float s = warp_sum((acc[0] + acc[1]) + (acc[2] + acc[3]));
    if (lane == 0) a[n] = sqrtf(s);
  }
}

}  // namespace prism
