// V as fp16 with one power-of-two scale per head, for the forward's O += P V.
//
// The forward's second product takes P in fp16 (11 significant bits) rather
// than bf16 (8): the backward's row sums D = rowsum(dO o O) need O to more
// bits than one bf16 rounding of every probability leaves, and the
// tensor cores want both operands of one product in the same type.  bf16 V
// maps into fp16 exactly once it is scaled by 2^e_h so that the head's
// largest |v| lands in [2^14, 2^15): the bf16 significand fits in fp16's,
// the range cannot overflow, and only values under 2^-28 of the head maximum
// (fp16 subnormals) round.  The forward's epilogue multiplies by 2^-e_h,
// which is exact.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace prism {

// e_h from the bf16 bit pattern of max |v| over head h (sign cleared).  Zero,
// infinite and NaN maxima keep e = 0 (NaN and Inf propagate unscaled).
__host__ __device__ __forceinline__ int v16_exponent(uint32_t maxbits) {
  const int E = (int)((maxbits >> 7) & 0xffu);   // biased exponent of the bf16 maximum
  if (maxbits == 0u || E == 0xff) return 0;
  int e = 141 - (E == 0 ? 1 : E);                 // max in [2^(E-127), 2^(E-126)) -> [2^14, 2^15)
  return e < -125 ? -125 : (e > 125 ? 125 : e);
}
// 2^e as a float, for |e| <= 126.
__device__ __forceinline__ float pow2f(int e) {
  return __uint_as_float((uint32_t)(e + 127) << 23);
}
// 2^d exactly for an integer-valued d <= 0 (d = -inf or d < -126 give 0).
__device__ __forceinline__ float pow2_or_zero(float d) {
  return d >= -126.f ? pow2f((int)d) : 0.f;
}

// Per-head max |v| of a permuted [heads, N*128] bf16 tensor, as the bf16 bit
// pattern (abs values of finite bf16 order like their bits).  vmax must be
// zeroed first.  Grid (x, heads); each thread strides over 16-byte words.
__global__ void __launch_bounds__(256) head_absmax_kernel(const uint4 *__restrict__ v, int64_t words_per_head,
                                                          uint32_t *__restrict__ vmax) {
  const uint4 *src = v + (int64_t)blockIdx.y * words_per_head;
  uint32_t m = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < words_per_head; i += 4 * stride) {
    uint4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) w[u] = __ldg(src + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      m = __vmaxu2(m, __vmaxu2(__vmaxu2(w[u].x & 0x7fff7fffu, w[u].y & 0x7fff7fffu),
                               __vmaxu2(w[u].z & 0x7fff7fffu, w[u].w & 0x7fff7fffu)));
  }
  for (; i < words_per_head; i += stride) {
    const uint4 w = __ldg(src + i);
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(w.x & 0x7fff7fffu, w.y & 0x7fff7fffu),
                             __vmaxu2(w.z & 0x7fff7fffu, w.w & 0x7fff7fffu)));
  }
  m = max(m & 0xffffu, m >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = max(m, red[w]);
    atomicMax(vmax + blockIdx.y, m);
  }
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
// The two fp16 halves of a packed pair, as floats.
__device__ __forceinline__ float f16_lo(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u & 0xffffu))); }
__device__ __forceinline__ float f16_hi(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u >> 16))); }

// x with its 13 low significand bits cleared (rounded toward zero to 11
// significant bits): exactly an fp16 value when in fp16's normal range.
__device__ __forceinline__ float trunc11(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }

// out = fp16(v * 2^e_h), same layout.  Grid (x, heads).
__global__ void __launch_bounds__(256) v_to_f16_kernel(const uint4 *__restrict__ v, int64_t words_per_head,
                                                       const uint32_t *__restrict__ vmax, uint4 *__restrict__ out) {
  const int64_t base = (int64_t)blockIdx.y * words_per_head;
  const float s = pow2f(v16_exponent(vmax[blockIdx.y]));
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words_per_head; i += stride) {
    const uint4 w = __ldg(v + base + i);
    uint4 r;
    r.x = pack_f16(bf16_lo(w.x) * s, bf16_hi(w.x) * s);
    r.y = pack_f16(bf16_lo(w.y) * s, bf16_hi(w.y) * s);
    r.z = pack_f16(bf16_lo(w.z) * s, bf16_hi(w.z) * s);
    r.w = pack_f16(bf16_lo(w.w) * s, bf16_hi(w.w) * s);
    out[base + i] = r;
  }
}

}  // namespace prism
