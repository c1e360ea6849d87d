// Block-sparse flash attention forward and backward on the warp-level bf16
// tensor-core MMA (m16n8k16).  64-row query or key tiles, four warps, K/V
// (or Q/dO) tiles double-buffered through cp.async, online softmax in
// registers.  These kernels are the portable reference path of the library;
// the tcgen05/TMEM kernels replace them where they apply.
#pragma once

#include "attn_common.cuh"

namespace prism {

// Sequence of 64-row sub-tiles of the key blocks listed in col[e0..e1).
struct SubtileCursor {
  const int32_t *col;
  const prism_block *blocks;
  int e, e1, sub, nsub;
  int64_t start;
  __device__ __forceinline__ void init(const int32_t *c, const prism_block *b, int e0, int e1_) {
    col = c; blocks = b; e = e0; e1 = e1_; sub = 0;
    if (e < e1) {
      const prism_block blk = blocks[col[e]];
      start = blk.start;
      nsub = blk.size >> 6;
    }
  }
  __device__ __forceinline__ bool valid() const { return e < e1; }
  __device__ __forceinline__ int64_t row() const { return start + ((int64_t)sub << 6); }
  __device__ __forceinline__ void next() {
    if (++sub >= nsub) {
      sub = 0;
      if (++e < e1) {
        const prism_block blk = blocks[col[e]];
        start = blk.start;
        nsub = blk.size >> 6;
      }
    }
  }
};

template <int D>
__global__ void __launch_bounds__(128) bsa_fwd_mma_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, const prism_block *__restrict__ blocks,
    const int32_t *__restrict__ zone_blk_base, const int32_t *__restrict__ row_ptr,
    const int32_t *__restrict__ col, int64_t N, int64_t cap, float scale_log2,
    __nv_bfloat16 *__restrict__ o, __nv_bfloat16 *__restrict__ o_res, float *__restrict__ lse) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TILE = 64 * D * 2;
  const uint32_t sQ = smem_u32(smem), sK = sQ + TILE, sV = sQ + 3 * TILE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t r0 = (int64_t)blockIdx.x * 64;
  const int i = block_of_row(r0, blocks, zone_blk_base);
  const int64_t hoff = (int64_t)h * N * D;
  SubtileCursor cur;
  cur.init(col, blocks, row_ptr[h * cap + i], row_ptr[h * cap + i + 1]);

  load_tile_async<D, 64, 128>(sQ, q + hoff + r0 * D);
  if (cur.valid()) {
    load_tile_async<D, 64, 128>(sK, k + hoff + cur.row() * D);
    load_tile_async<D, 64, 128>(sV, v + hoff + cur.row() * D);
  }
  cp_async_commit();

  float acc[D / 8][4];
#pragma unroll
  for (int t = 0; t < D / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];
  int buf = 0;
  bool first = true;
  while (cur.valid()) {
    SubtileCursor nxt = cur;
    nxt.next();
    if (nxt.valid()) {
      load_tile_async<D, 64, 128>(sK + (buf ^ 1) * TILE, k + hoff + nxt.row() * D);
      load_tile_async<D, 64, 128>(sV + (buf ^ 1) * TILE, v + hoff + nxt.row() * D);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (first) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) load_a_frag<D>(qf[ks], sQ, warp * 16, ks * 16);
      first = false;
    }
    const uint32_t tK = sK + buf * TILE, tV = sV + buf * TILE;
    float s[8][4];
#pragma unroll
    for (int t = 0; t < 8; ++t) s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        load_b_nk<D>(b, tK, np * 16, ks * 16);
        mma16816(s[2 * np], qf[ks], b[0], b[1]);
        mma16816(s[2 * np + 1], qf[ks], b[2], b[3]);
      }
    }
    // online softmax (log2 domain), rows lane/4 and lane/4 + 8
    float mx[2] = {mrow[0], mrow[1]};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      mx[0] = fmaxf(mx[0], fmaxf(s[t][0], s[t][1]) * scale_log2);
      mx[1] = fmaxf(mx[1], fmaxf(s[t][2], s[t][3]) * scale_log2);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2], rs[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      corr[r] = exp2f(mrow[r] - mx[r]);
      mrow[r] = mx[r];
    }
    uint32_t pa[4][4];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float p0 = exp2f(s[t][0] * scale_log2 - mx[0]);
      const float p1 = exp2f(s[t][1] * scale_log2 - mx[0]);
      const float p2 = exp2f(s[t][2] * scale_log2 - mx[1]);
      const float p3 = exp2f(s[t][3] * scale_log2 - mx[1]);
      rs[0] += p0 + p1;
      rs[1] += p2 + p3;
      pa[t >> 1][(t & 1) * 2 + 0] = pack_bf16(p0, p1);
      pa[t >> 1][(t & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) lrow[r] = lrow[r] * corr[r] + rs[r];
#pragma unroll
    for (int t = 0; t < D / 8; ++t) {
      acc[t][0] *= corr[0]; acc[t][1] *= corr[0];
      acc[t][2] *= corr[1]; acc[t][3] *= corr[1];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int cp = 0; cp < D / 16; ++cp) {
        uint32_t b[4];
        load_b_kn<D>(b, tV, kk * 16, cp * 16);
        mma16816(acc[2 * cp], pa[kk], b[0], b[1]);
        mma16816(acc[2 * cp + 1], pa[kk], b[2], b[3]);
      }
    }
    __syncthreads();
    buf ^= 1;
    cur = nxt;
  }
  cp_async_wait<0>();
  // finish: quad-reduce the row sums, normalise, store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  const float inv0 = lrow[0] > 0.f ? 1.f / lrow[0] : 0.f;
  const float inv1 = lrow[1] > 0.f ? 1.f / lrow[1] : 0.f;
  const int64_t ra = r0 + warp * 16 + (lane >> 2), rb = ra + 8;
  __nv_bfloat16 *oa = o + hoff + ra * D, *ob = o + hoff + rb * D;
#pragma unroll
  for (int t = 0; t < D / 8; ++t) {
    const int c = t * 8 + (lane & 3) * 2;
    const float x0 = acc[t][0] * inv0, x1 = acc[t][1] * inv0, x2 = acc[t][2] * inv1, x3 = acc[t][3] * inv1;
    const uint32_t ua = pack_bf16(x0, x1), ub = pack_bf16(x2, x3);
    *reinterpret_cast<uint32_t *>(oa + c) = ua;
    *reinterpret_cast<uint32_t *>(ob + c) = ub;
    if (o_res) {
      *reinterpret_cast<uint32_t *>(o_res + hoff + ra * D + c) = pack_bf16(x0 - bf16_lo(ua), x1 - bf16_hi(ua));
      *reinterpret_cast<uint32_t *>(o_res + hoff + rb * D + c) = pack_bf16(x2 - bf16_lo(ub), x3 - bf16_hi(ub));
    }
  }
  if ((lane & 3) == 0) {
    lse[(int64_t)h * N + ra] = lrow[0] > 0.f ? (mrow[0] + log2f(lrow[0])) * kLn2 : -INFINITY;
    lse[(int64_t)h * N + rb] = lrow[1] > 0.f ? (mrow[1] + log2f(lrow[1])) * kLn2 : -INFINITY;
  }
}

}  // namespace prism
