// Zone-local token permutation with fused block mean-pooling, and its inverse.
//
// One CTA per (head, zone).  VL = D/8 lanes each own 8 channels (one 16-byte
// bf16 vector) of a token; TL = 256/VL token lanes walk the zone's 512
// permuted positions block by block.  Every token row of a head is a
// contiguous D-wide segment on both sides, so loads and stores are full
// 16-byte vectors covering whole 128-byte lines.  The block sums stay in
// registers and are combined over the token lanes in shared memory, in a
// fixed order, at each block boundary.
#pragma once

#include "common.cuh"

namespace prism {

template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float v[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float v[8]) {
    uint4 u;
    u.x = pack_bf16(v[0], v[1]); u.y = pack_bf16(v[2], v[3]);
    u.z = pack_bf16(v[4], v[5]); u.w = pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4 *>(p) = u;
  }
};
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float *p, float v[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float *p, const float v[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

// Exact bf16 copy (no float round trip) for the bf16 -> bf16 fast path.
__device__ __forceinline__ void copy16(const void *src, void *dst) {
  *reinterpret_cast<uint4 *>(dst) = __ldg(reinterpret_cast<const uint4 *>(src));
}

template <typename Tin, int D>
__global__ void __launch_bounds__(256) permute_kernel(const Tin *__restrict__ x, int heads, int64_t N, int H,
                                                      int W, int ZY, int ZX, const uint8_t *__restrict__ shape_id,
                                                      const int32_t *__restrict__ zone_blk_base, int64_t cap,
                                                      __nv_bfloat16 *__restrict__ xp, float *__restrict__ pooled) {
  constexpr int VL = D / 8, TL = 256 / VL;
  __shared__ float red[TL][D];
  const int h = blockIdx.x, m = blockIdx.y;
  const int vl = threadIdx.x % VL, tl = threadIdx.x / VL;
  const int zt = m / (ZY * ZX), zy = (m / ZX) % ZY, zx = m % ZX;
  const int sid = shape_id[m];
  const int B = shape_volume(sid), nb = kZoneTokens / B;
  const int64_t blk0 = pooled ? zone_blk_base[m] : 0;
  const int64_t C = (int64_t)heads * D;
  for (int b = 0; b < nb; ++b) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int p = b * B + tl; p < (b + 1) * B; p += TL) {
      const int64_t n = zone_token(p, sid, zt, zy, zx, H, W);
      const Tin *src = x + n * C + (int64_t)h * D + vl * 8;
      __nv_bfloat16 *dst = xp + ((int64_t)h * N + (int64_t)m * kZoneTokens + p) * D + vl * 8;
      float v[8];
      Vec8<Tin>::load(src, v);
      Vec8<__nv_bfloat16>::store(dst, v);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += v[c];
    }
    if (pooled) {
#pragma unroll
      for (int c = 0; c < 8; ++c) red[tl][vl * 8 + c] = acc[c];
      __syncthreads();
      if (threadIdx.x < D) {
        float s = 0.f;
        for (int t = 0; t < TL; ++t) s += red[t][threadIdx.x];
        pooled[((int64_t)h * cap + blk0 + b) * D + threadIdx.x] = s / (float)B;
      }
      __syncthreads();
    }
  }
}

template <typename Tin, typename Tout, int D>
__global__ void __launch_bounds__(256) unpermute_kernel(const Tin *__restrict__ xp, int heads, int64_t N, int H,
                                                        int W, int ZY, int ZX,
                                                        const uint8_t *__restrict__ shape_id,
                                                        Tout *__restrict__ x) {
  constexpr int VL = D / 8, TL = 256 / VL;
  const int h = blockIdx.x, m = blockIdx.y;
  const int vl = threadIdx.x % VL, tl = threadIdx.x / VL;
  const int zt = m / (ZY * ZX), zy = (m / ZX) % ZY, zx = m % ZX;
  const int sid = shape_id[m];
  const int64_t C = (int64_t)heads * D;
  for (int p = tl; p < kZoneTokens; p += TL) {
    const int64_t n = zone_token(p, sid, zt, zy, zx, H, W);
    const Tin *src = xp + ((int64_t)h * N + (int64_t)m * kZoneTokens + p) * D + vl * 8;
    Tout *dst = x + n * C + (int64_t)h * D + vl * 8;
    float v[8];
    Vec8<Tin>::load(src, v);
    Vec8<Tout>::store(dst, v);
  }
}

}  // namespace prism
