// Shared device helpers of the Prism sm_100a library: the latched status word,
// the candidate-shape table and small vector/reduction utilities.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "prism.h"

namespace prism {

constexpr int kZone = 8;            // macro-zone edge (Key ideas: 8x8x8)
constexpr int kZoneTokens = 512;    // tokens per zone
constexpr int kMaxBlocksPerZone = 8;

// Latched device status (first error wins); read and cleared by
// prism_device_status().  The library is one translation unit, so this is
// the only definition.
__device__ int g_status = 0;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

// The 16 candidate block shapes (bT, bH, bW): edges in {2,4,8} with volume
// 64, 128 or 256, ordered by volume then lexicographically.
struct ShapeTable {
  int8_t e[16][3];
};
constexpr ShapeTable kShapes = {{{2, 4, 8}, {2, 8, 4}, {4, 2, 8}, {4, 4, 4}, {4, 8, 2}, {8, 2, 4},
                                 {8, 4, 2}, {2, 8, 8}, {4, 4, 8}, {4, 8, 4}, {8, 2, 8}, {8, 4, 4},
                                 {8, 8, 2}, {4, 8, 8}, {8, 4, 8}, {8, 8, 4}}};
// log2 of each edge packed two bits per shape, one word per axis, so that
// device code reads an edge from an immediate instead of a local array.
constexpr uint32_t pack_axis(int axis) {
  uint32_t w = 0;
  for (int s = 0; s < 16; ++s) {
    const int e = kShapes.e[s][axis];
    const uint32_t l = e == 2 ? 1u : (e == 4 ? 2u : 3u);
    w |= l << (2 * s);
  }
  return w;
}
constexpr uint32_t kShapeLog2T = pack_axis(0), kShapeLog2H = pack_axis(1), kShapeLog2W = pack_axis(2);
__host__ __device__ __forceinline__ constexpr int shape_edge(int sid, int axis) {
  return 1 << (((axis == 0 ? kShapeLog2T : (axis == 1 ? kShapeLog2H : kShapeLog2W)) >> (2 * sid)) & 3u);
}
__host__ __device__ constexpr int shape_volume(int sid) {
  return shape_edge(sid, 0) * shape_edge(sid, 1) * shape_edge(sid, 2);
}
__host__ __device__ constexpr int shape_first(int volume) {
  return volume == 64 ? 0 : (volume == 128 ? 7 : 13);
}
__host__ __device__ constexpr int shape_count(int volume) {
  return volume == 64 ? 7 : (volume == 128 ? 6 : 3);
}

// Natural token index of permuted position p (0..511) of zone (zt, zy, zx)
// whose blocks have shape sid.
__device__ __forceinline__ int64_t zone_token(int p, int sid, int zt, int zy, int zx, int H, int W) {
  const int bT = shape_edge(sid, 0), bH = shape_edge(sid, 1), bW = shape_edge(sid, 2);
  const int B = bT * bH * bW;
  const int b = p / B, l = p - b * B;
  const int nH = kZone / bH, nW = kZone / bW;
  const int it = b / (nH * nW), iy = (b / nW) % nH, ix = b % nW;
  const int lt = l / (bH * bW), ly = (l / bW) % bH, lx = l % bW;
  const int64_t t = zt * kZone + it * bT + lt;
  const int64_t y = zy * kZone + iy * bH + ly;
  const int64_t x = zx * kZone + ix * bW + lx;
  return (t * H + y) * W + x;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
template <typename T>
__device__ __forceinline__ T warp_max(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace prism

#define PRISM_CUDA_CHECK_LAUNCH()                                        \
  do {                                                                   \
    cudaError_t _e = cudaGetLastError();                                 \
    if (_e != cudaSuccess) return prism::fail(PRISM_ECUDA, cudaGetErrorString(_e)); \
  } while (0)

namespace prism {
int fail(int code, const char *msg);
}
