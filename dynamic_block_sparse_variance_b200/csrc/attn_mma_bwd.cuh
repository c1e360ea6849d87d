// Backward of the block-sparse attention on the warp-level bf16 MMA.
//
// bwd_delta_kernel   D_r = sum_c dO_rc O_rc (fp32), one warp per row; O is the
//                    bf16 output plus, when given, its rounding residual.
// csc kernels        transpose of the selection (per head, key block ->
//                    ascending query blocks), so dK/dV are owned by one CTA.
// bsa_dkdv_mma_kernel  one CTA per (64-key tile, head): walks the query blocks
//                    that selected its key block; dV += P^T dO, dK += dS^T Q.
// bsa_dq_mma_kernel  one CTA per (64-query tile, head): walks S_i;
//                    dQ += dS K.  Both accumulate in registers in a fixed
//                    order, so the gradients are bit-reproducible.
#pragma once

#include "attn_mma.cuh"

namespace prism {

template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16 *__restrict__ o,
                                                        const __nv_bfloat16 *__restrict__ o_res,
                                                        const __nv_bfloat16 *__restrict__ dout,
                                                        const float *__restrict__ lse, int64_t rows,
                                                        float *__restrict__ delta, float *__restrict__ lse2) {
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  constexpr int PER = D / 32;  // 2 or 4 elements per lane
  float s = 0.f;
  const __nv_bfloat16 *a = o + r * D + lane * PER, *b = dout + r * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const uint32_t ua = *reinterpret_cast<const uint32_t *>(a + e);
    const uint32_t ub = *reinterpret_cast<const uint32_t *>(b + e);
    float o0 = bf16_lo(ua), o1 = bf16_hi(ua);
    if (o_res) {
      const uint32_t ur = *reinterpret_cast<const uint32_t *>(o_res + r * D + lane * PER + e);
      o0 += bf16_lo(ur);
      o1 += bf16_hi(ur);
    }
    s += o0 * bf16_lo(ub) + o1 * bf16_hi(ub);
  }
  s = warp_sum(s);
  if (lane == 0) {
    delta[r] = s;
    lse2[r] = -(lse[r] * 1.4426950408889634f);   // -LSE in log2 units: the key-side kernel's FMA addend
  }
}

// ---- CSR -> CSC per head -------------------------------------------------
__global__ void __launch_bounds__(256) csc_count_kernel(const int32_t *__restrict__ row_ptr,
                                                        const int32_t *__restrict__ col, int64_t cap,
                                                        const int32_t *__restrict__ nblk_p,
                                                        int32_t *__restrict__ ccnt) {
  const int n = *nblk_p;
  const int i = blockIdx.x, h = blockIdx.y;
  if (i >= n) return;
  const int64_t row = (int64_t)h * cap + i;
  for (int e = row_ptr[row] + threadIdx.x; e < row_ptr[row + 1]; e += blockDim.x)
    atomicAdd(&ccnt[(int64_t)h * cap + col[e]], 1);
}

__global__ void __launch_bounds__(256) csc_fill_kernel(const int32_t *__restrict__ row_ptr,
                                                       const int32_t *__restrict__ col, int64_t cap,
                                                       const int32_t *__restrict__ nblk_p,
                                                       const int32_t *__restrict__ col_ptr,
                                                       int32_t *__restrict__ fill,
                                                       int32_t *__restrict__ row_idx) {
  const int n = *nblk_p;
  const int i = blockIdx.x, h = blockIdx.y;
  if (i >= n) return;
  const int64_t row = (int64_t)h * cap + i;
  for (int e = row_ptr[row] + threadIdx.x; e < row_ptr[row + 1]; e += blockDim.x) {
    const int64_t c = (int64_t)h * cap + col[e];
    const int pos = atomicAdd(&fill[c], 1);
    row_idx[col_ptr[c] + pos] = i;
  }
}

// Sort each column's query-block list ascending (bitonic, in shared memory).
__global__ void __launch_bounds__(512) csc_sort_kernel(const int32_t *__restrict__ col_ptr, int64_t cap,
                                                       const int32_t *__restrict__ nblk_p,
                                                       int32_t *__restrict__ row_idx) {
  extern __shared__ int32_t buf[];
  const int n = *nblk_p;
  const int j = blockIdx.x, h = blockIdx.y;
  if (j >= n) return;
  const int64_t c = (int64_t)h * cap + j;
  const int b = col_ptr[c], len = col_ptr[c + 1] - b;
  if (len <= 1) return;
  int p2 = 1;
  while (p2 < len) p2 <<= 1;
  for (int t = threadIdx.x; t < p2; t += blockDim.x) buf[t] = t < len ? row_idx[b + t] : 0x7fffffff;
  __syncthreads();
  for (int size = 2; size <= p2; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < p2; t += blockDim.x) {
        const int u = t ^ stride;
        if (u > t) {
          const bool up = (t & size) == 0;
          const int a = buf[t], bb = buf[u];
          if ((a > bb) == up) {
            buf[t] = bb;
            buf[u] = a;
          }
        }
      }
      __syncthreads();
    }
  for (int t = threadIdx.x; t < len; t += blockDim.x) row_idx[b + t] = buf[t];
}

// ---- dK, dV ---------------------------------------------------------------
// Shared memory: K tile, V tile (64 keys), then double-buffered Q and dO tiles
// (64 queries) with their LSE*log2e and D values.
template <int D>
__global__ void __launch_bounds__(128) bsa_dkdv_mma_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dout,
    const float *__restrict__ lse, const float *__restrict__ delta,
    const prism_block *__restrict__ blocks, const int32_t *__restrict__ zone_blk_base,
    const int32_t *__restrict__ col_ptr, const int32_t *__restrict__ row_idx, int64_t N, int64_t cap,
    float scale, __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TILE = 64 * D * 2;
  const uint32_t sK = smem_u32(smem), sV = sK + TILE, sQ = sK + 2 * TILE, sO = sK + 4 * TILE;
  float *sL = reinterpret_cast<float *>(smem + 6 * TILE);  // [2][64] lse*log2e
  float *sD = sL + 128;                                     // [2][64] delta
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t k0 = (int64_t)blockIdx.x * 64;
  const int j = block_of_row(k0, blocks, zone_blk_base);
  const int64_t hoff = (int64_t)h * N * D;
  const float scale_log2 = scale * kLog2e;
  SubtileCursor cur;  // walks the query blocks that selected key block j
  cur.init(row_idx, blocks, col_ptr[h * cap + j], col_ptr[h * cap + j + 1]);

  auto load_q = [&](int b, int64_t qr) {
    load_tile_async<D, 64, 128>(sQ + b * TILE, q + hoff + qr * D);
    load_tile_async<D, 64, 128>(sO + b * TILE, dout + hoff + qr * D);
    if (threadIdx.x < 16) {
      cp_async16(smem_u32(sL + b * 64 + threadIdx.x * 4), lse + (int64_t)h * N + qr + threadIdx.x * 4);
    } else if (threadIdx.x < 32) {
      const int t = threadIdx.x - 16;
      cp_async16(smem_u32(sD + b * 64 + t * 4), delta + (int64_t)h * N + qr + t * 4);
    }
  };
  load_tile_async<D, 64, 128>(sK, k + hoff + k0 * D);
  load_tile_async<D, 64, 128>(sV, v + hoff + k0 * D);
  if (cur.valid()) load_q(0, cur.row());
  cp_async_commit();

  float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
  for (int t = 0; t < D / 8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) dka[t][e] = dva[t][e] = 0.f;
  int buf = 0;
  while (cur.valid()) {
    SubtileCursor nxt = cur;
    nxt.next();
    if (nxt.valid()) load_q(buf ^ 1, nxt.row());
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t tQ = sQ + buf * TILE, tO = sO + buf * TILE;
    const float *L = sL + buf * 64, *Dl = sD + buf * 64;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int qb = half * 32;  // 32 queries per half
      // S^T (16 keys x 32 queries) = K_w Q^T; dP^T = V_w dO^T
      float st[4][4], dpt[4][4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[t][e] = dpt[t][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t ka[4], va[4];
        load_a_frag<D>(ka, sK, warp * 16, ks * 16);
        load_a_frag<D>(va, sV, warp * 16, ks * 16);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t b[4];
          load_b_nk<D>(b, tQ, qb + np * 16, ks * 16);
          mma16816(st[2 * np], ka, b[0], b[1]);
          mma16816(st[2 * np + 1], ka, b[2], b[3]);
          load_b_nk<D>(b, tO, qb + np * 16, ks * 16);
          mma16816(dpt[2 * np], va, b[0], b[1]);
          mma16816(dpt[2 * np + 1], va, b[2], b[3]);
        }
      }
      // P^T and dS^T; columns are queries qb + t*8 + (lane&3)*2 + {0,1}
      uint32_t pa[2][4], sa[2][4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int qc = qb + t * 8 + (lane & 3) * 2;
        const float l0 = L[qc] * kLog2e, l1 = L[qc + 1] * kLog2e, d0 = Dl[qc], d1 = Dl[qc + 1];
        const float p0 = exp2f(st[t][0] * scale_log2 - l0), p1 = exp2f(st[t][1] * scale_log2 - l1);
        const float p2 = exp2f(st[t][2] * scale_log2 - l0), p3 = exp2f(st[t][3] * scale_log2 - l1);
        pa[t >> 1][(t & 1) * 2 + 0] = pack_bf16(p0, p1);
        pa[t >> 1][(t & 1) * 2 + 1] = pack_bf16(p2, p3);
        sa[t >> 1][(t & 1) * 2 + 0] = pack_bf16(p0 * (dpt[t][0] - d0), p1 * (dpt[t][1] - d1));
        sa[t >> 1][(t & 1) * 2 + 1] = pack_bf16(p2 * (dpt[t][2] - d0), p3 * (dpt[t][3] - d1));
      }
      // dV += P^T dO ; dK += dS^T Q   (k = queries)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
        for (int cp = 0; cp < D / 16; ++cp) {
          uint32_t b[4];
          load_b_kn<D>(b, tO, qb + kk * 16, cp * 16);
          mma16816(dva[2 * cp], pa[kk], b[0], b[1]);
          mma16816(dva[2 * cp + 1], pa[kk], b[2], b[3]);
          load_b_kn<D>(b, tQ, qb + kk * 16, cp * 16);
          mma16816(dka[2 * cp], sa[kk], b[0], b[1]);
          mma16816(dka[2 * cp + 1], sa[kk], b[2], b[3]);
        }
      }
    }
    __syncthreads();
    buf ^= 1;
    cur = nxt;
  }
  cp_async_wait<0>();
  const int64_t ra = k0 + warp * 16 + (lane >> 2), rb = ra + 8;
#pragma unroll
  for (int t = 0; t < D / 8; ++t) {
    const int c = t * 8 + (lane & 3) * 2;
    *reinterpret_cast<uint32_t *>(dk + hoff + ra * D + c) = pack_bf16(dka[t][0] * scale, dka[t][1] * scale);
    *reinterpret_cast<uint32_t *>(dk + hoff + rb * D + c) = pack_bf16(dka[t][2] * scale, dka[t][3] * scale);
    *reinterpret_cast<uint32_t *>(dv + hoff + ra * D + c) = pack_bf16(dva[t][0], dva[t][1]);
    *reinterpret_cast<uint32_t *>(dv + hoff + rb * D + c) = pack_bf16(dva[t][2], dva[t][3]);
  }
}

// ---- dQ -------------------------------------------------------------------
// Shared memory: Q and dO tiles (64 queries), then double-buffered K and V tiles.
template <int D>
__global__ void __launch_bounds__(128) bsa_dq_mma_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dout,
    const float *__restrict__ lse, const float *__restrict__ delta,
    const prism_block *__restrict__ blocks, const int32_t *__restrict__ zone_blk_base,
    const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col, int64_t N, int64_t cap,
    float scale, __nv_bfloat16 *__restrict__ dq) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TILE = 64 * D * 2;
  const uint32_t sQ = smem_u32(smem), sO = sQ + TILE, sK = sQ + 2 * TILE, sV = sQ + 4 * TILE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t r0 = (int64_t)blockIdx.x * 64;
  const int i = block_of_row(r0, blocks, zone_blk_base);
  const int64_t hoff = (int64_t)h * N * D;
  const float scale_log2 = scale * kLog2e;
  SubtileCursor cur;
  cur.init(col, blocks, row_ptr[h * cap + i], row_ptr[h * cap + i + 1]);
  const int64_t ra = r0 + warp * 16 + (lane >> 2), rb = ra + 8;
  const float la = lse[(int64_t)h * N + ra] * kLog2e, lb = lse[(int64_t)h * N + rb] * kLog2e;
  const float da = delta[(int64_t)h * N + ra], db = delta[(int64_t)h * N + rb];

  load_tile_async<D, 64, 128>(sQ, q + hoff + r0 * D);
  load_tile_async<D, 64, 128>(sO, dout + hoff + r0 * D);
  if (cur.valid()) {
    load_tile_async<D, 64, 128>(sK, k + hoff + cur.row() * D);
    load_tile_async<D, 64, 128>(sV, v + hoff + cur.row() * D);
  }
  cp_async_commit();
  float acc[D / 8][4];
#pragma unroll
  for (int t = 0; t < D / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  int buf = 0;
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
    const uint32_t tK = sK + buf * TILE, tV = sV + buf * TILE;
    float s[8][4], dp[8][4];
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[t][e] = dp[t][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t qa[4], oa[4];
      load_a_frag<D>(qa, sQ, warp * 16, ks * 16);
      load_a_frag<D>(oa, sO, warp * 16, ks * 16);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        load_b_nk<D>(b, tK, np * 16, ks * 16);
        mma16816(s[2 * np], qa, b[0], b[1]);
        mma16816(s[2 * np + 1], qa, b[2], b[3]);
        load_b_nk<D>(b, tV, np * 16, ks * 16);
        mma16816(dp[2 * np], oa, b[0], b[1]);
        mma16816(dp[2 * np + 1], oa, b[2], b[3]);
      }
    }
    uint32_t sa[4][4];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float p0 = exp2f(s[t][0] * scale_log2 - la), p1 = exp2f(s[t][1] * scale_log2 - la);
      const float p2 = exp2f(s[t][2] * scale_log2 - lb), p3 = exp2f(s[t][3] * scale_log2 - lb);
      sa[t >> 1][(t & 1) * 2 + 0] = pack_bf16(p0 * (dp[t][0] - da), p1 * (dp[t][1] - da));
      sa[t >> 1][(t & 1) * 2 + 1] = pack_bf16(p2 * (dp[t][2] - db), p3 * (dp[t][3] - db));
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int cp = 0; cp < D / 16; ++cp) {
        uint32_t b[4];
        load_b_kn<D>(b, tK, kk * 16, cp * 16);
        mma16816(acc[2 * cp], sa[kk], b[0], b[1]);
        mma16816(acc[2 * cp + 1], sa[kk], b[2], b[3]);
      }
    }
    __syncthreads();
    buf ^= 1;
    cur = nxt;
  }
  cp_async_wait<0>();
#pragma unroll
  for (int t = 0; t < D / 8; ++t) {
    const int c = t * 8 + (lane & 3) * 2;
    *reinterpret_cast<uint32_t *>(dq + hoff + ra * D + c) = pack_bf16(acc[t][0] * scale, acc[t][1] * scale);
    *reinterpret_cast<uint32_t *>(dq + hoff + rb * D + c) = pack_bf16(acc[t][2] * scale, acc[t][3] * scale);
  }
}

}  // namespace prism
