// Building blocks shared by the block-sparse attention kernels: swizzled
// shared-memory tiles, cp.async loaders, ldmatrix and the bf16 m16n8k16 MMA.
#pragma once

#include "common.cuh"

namespace prism {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of 16-byte chunk `ch` of row `row` in a [rows][D] bf16 tile.
// Chunks are XOR-swizzled by the row's low three bits so that the eight rows an
// ldmatrix phase reads fall in distinct bank groups.
template <int D>
__device__ __forceinline__ uint32_t tile_off(int row, int ch) {
  return (uint32_t)(row * (D * 2) + ((ch ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Load a [ROWS][D] bf16 tile (global row stride D) into a swizzled tile.
template <int D, int ROWS, int NT>
__device__ __forceinline__ void load_tile_async(uint32_t sbase, const __nv_bfloat16 *g) {
  constexpr int CH = D / 8;
#pragma unroll
  for (int c = threadIdx.x; c < ROWS * CH; c += NT) {
    const int row = c / CH, ch = c % CH;
    cp_async16(sbase + tile_off<D>(row, ch), g + (int64_t)row * D + ch * 8);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (16 rows x 16 k) at (r0, k0) of a row-major swizzled tile.
template <int D>
__device__ __forceinline__ void load_a_frag(uint32_t a[4], uint32_t tile, int r0, int k0) {
  const int lane = threadIdx.x & 31;
  ldsm_x4(a, tile + tile_off<D>(r0 + (lane & 15), (k0 >> 3) + (lane >> 4)));
}
// B fragments for two n-tiles (n0..n0+15) x one k-step (k0..k0+15) where the
// tile is stored [n][k] (k contiguous): b[0],b[1] -> n-tile 0; b[2],b[3] -> n-tile 1.
template <int D>
__device__ __forceinline__ void load_b_nk(uint32_t b[4], uint32_t tile, int n0, int k0) {
  const int lane = threadIdx.x & 31;
  ldsm_x4(b, tile + tile_off<D>(n0 + (lane & 7) + ((lane >> 4) << 3), (k0 >> 3) + ((lane >> 3) & 1)));
}
// B fragments for two n-tiles (n0..n0+15) x one k-step (k0..k0+15) where the
// tile is stored [k][n] (n contiguous), via the transposing ldmatrix.
template <int D>
__device__ __forceinline__ void load_b_kn(uint32_t b[4], uint32_t tile, int k0, int n0) {
  const int lane = threadIdx.x & 31;
  ldsm_x4_t(b, tile + tile_off<D>(k0 + (lane & 7) + (((lane >> 3) & 1) << 3), (n0 >> 3) + (lane >> 4)));
}

// Query/key tile of 64 rows starting at permuted row r0: the block it lies in.
__device__ __forceinline__ int block_of_row(int64_t r0, const prism_block *__restrict__ blocks,
                                           const int32_t *__restrict__ zone_blk_base) {
  const int m = (int)(r0 / kZoneTokens);
  const int b0 = zone_blk_base[m];
  const int B = blocks[b0].size;
  return b0 + (int)((r0 - (int64_t)m * kZoneTokens) / B);
}

}  // namespace prism
