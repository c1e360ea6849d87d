// Block-sparse attention backward on the tcgen05 tensor cores (head_dim 128):
// dK, dV and dQ from one pass over the transposed selection.
//
// bsa_bwd_tc_kernel  one CTA per (128-key tile, head), walking the query tiles
//   of the query blocks that selected its key block.  Per query tile n:
//     S^T_n  = K Q_n^T          (both operands in shared memory)
//     dP^T_n = V dO_n^T
//     P^T_n  -> A operand of dV += P^T_n dO_n   (fp16, from tensor memory)
//     dS^T_n = P^T (dP^T - D)  -> A operand of dK += dS^T_n Q_n (a bf16 pair
//                                 dS_hi + dS_lo in tensor memory, two products)
//                                 and, through shared memory, of
//     dQ_n   = dS_n K           (the same pair, two products, written over the
//                                 dP^T columns once dK_n has read dS^T)
//   and four drain warps move dQ_n out of tensor memory into an fp32
//   accumulator in global memory with vector reductions (red.global.add.v4).
//   Seven products and one exponential per score.  dQ is summed in fp32 in
//   the order the reductions reach L2, so its last bits may differ run to run.
//
// Precision.  Every product accumulates in fp32 and takes its operands at the
// precision the errors they carry allow:
//   * P, the forward's: P_c = t(2^(x_c - m)) 2^(m - L), x_c the score and
//     L = LSE log2e in log2 units, m = ceil(L) - 15 an integer and t()
//     truncation to 11 significant bits, which is what the forward used for
//     O = sum_c P_c v_c
//     (it truncates the same way, with an integer running max, and normalises
//     by the sum of the truncated values).  So D = rowsum(dO o O) equals
//     sum_c P_c dP_c and every row of dS = P (dP - D) sums to zero, as it must:
//     otherwise dQ_r = scale sum_c dS_rc k_c keeps an error times the keys'
//     common component.  It is kept in fp32, scaled by 2^15.
//   * dV += P^T dO in fp16 x fp16: 2^15 P as fp16 (probabilities down to
//     2^-29 stay normal) and dO as fp16 scaled per head by a power of two
//     (exact for bf16 input, see v16.cuh).  dV sums P over every selecting
//     query row; fp16's 11 bits keep that sum's error near 2^-11 of sum |P dO|.
//   * dP^T = V dO^T in fp16 x fp16, V likewise scaled (exact).
//   * S^T = K Q^T, dK += dS^T Q and dQ = dS K in bf16 x bf16, the inputs
//     themselves, with dS as the pair dS_hi = dS truncated to bf16 and
//     dS_lo = bf16(dS - dS_hi) (about 16 bits together, and bf16's exponent
//     range, which the dS of key blocks that few
//     queries attend to need: their dS lies far below the head's largest).
//     One rounding of dS would leave dK of heavily selected key blocks (sums
//     over thousands of query rows) and dQ (the rows of dS sum to zero, so
//     its error would carry the keys' common component) outside the bounds.
//
// Tensor-pipe order per tile: dV_n, S^T_{n+1}, dK_n (2), dQ_n (2), dP^T_{n+1}; the
// last waits until the drain warps have read dQ_n (they load all of it
// before they start the reductions).  Shared memory holds Q in two stages
// and dO in one (dO_{n+1} is loaded while S^T_{n+1}, dK_n and dQ_n run).
// TMEM: dK | dV | S^T (P^T) | dP^T (dS^T, then dQ).  A half of the
// elementwise warps writes its 16-bit P^T or dS_hi^T into the first 32 columns
// of its own 64-column range (dS_lo^T into the next 32), so operand k-step k
// (16 queries) sits at column 8k + (k >= 4 ? 32 : 0) (+32 for dS_lo^T).
//
// dQ accumulator layout (fp32): [head][row group of 64][32 column quads][64
// rows][4 columns], so that the 32 lanes of a drain warp (32 consecutive rows)
// reducing one column quad touch 512 contiguous bytes.
// dq_convert_kernel  one CTA per (row group, head): 64 rows x 128 columns of
//   the accumulator (32 KB, contiguous) -> scaled bf16 rows of dQ.
//
// Warps: 0-3 drain (TMEM lane quadrant = warp), 4-11 elementwise (quadrant
// warp & 3; warps w and w+4 take query columns [0,64) and [64,128)), 12 MMA
// issuer and TMEM owner, 13 TMA producer, 14-15 idle.  Registers: launched at
// 128 per thread; the drain warpgroup takes 152 (a whole dQ row, 128 values),
// the elementwise warpgroups 128 each (P of the row half kept for dS) and the
// MMA/producer warpgroup 104 (152 + 2 x 128 + 104 = 4 x 128).
// Every wait is bounded: a wait that runs out raises a CTA-wide abort,
// latches PRISM_ETIMEOUT, and the CTA drains its copies and products and
// frees its tensor memory.
#pragma once

#include "attn_tc_fwd.cuh"

namespace prism {

__device__ __forceinline__ uint32_t half_col(int k) { return 8u * (uint32_t)k + (k >= 4 ? 32u : 0u); }

struct TcBwdArgs {
  const prism_block *blocks;
  const int32_t *zone_blk_base;
  const int32_t *col_ptr;   // transposed selection: the query blocks of each key block
  const int32_t *row_idx;
  const float *stat_m;      // per query row: -(ceil(LSE log2e) - 15), -inf for rows without keys; +128 padding
  const float *stat_inv;    // per query row: 2^(ceil(LSE log2e) - LSE log2e), in [1, 2); +128 padding
  const float *delta_pad;   // per query row: D; +128 padding
  const uint32_t *amax;     // [2][heads] bf16 bits of max |x| of V and dO per head
  int heads;
  int64_t N, cap;
  float scale_log2, scale;
  __nv_bfloat16 *dk, *dv;
  uint32_t wait_limit;
  int debug_stall;   // test knob: P^T_0 is never signalled, so the MMA wait times out
};

// Tile of a zone: 128 rows (blocks of 128/256) or 64 rows (blocks of 64).
struct ZoneTile {
  int blk, r0, rows;
  __device__ __forceinline__ bool init(const prism_block *blocks, const int32_t *zbb, int m, int t) {
    const int b0 = zbb[m];
    const int B = blocks[b0].size;
    if (B >= 128 && t >= 4) return false;
    if (B == 64) {
      blk = b0 + t;
      r0 = m * kZoneTokens + 64 * t;
      rows = 64;
    } else {
      r0 = m * kZoneTokens + 128 * t;
      blk = b0 + (128 * t) / B;
      rows = 128;
    }
    return true;
  }
};

// Per-head power-of-two exponents of the backward's fp16 operands V and dO:
// the v16 exponent of their maximum (largest |x| in [2^14, 2^15)), kept in
// [-60, 60] so that their sum is a normal float's exponent (maxima of 2^75
// and more are outside the fp16 range).
struct BwdScales {
  int ev, edo;
  __device__ __forceinline__ BwdScales(const uint32_t *amax, int heads, int h) {
    ev = clampe(v16_exponent(amax[h]));
    edo = clampe(v16_exponent(amax[heads + h]));
  }
  __device__ __forceinline__ static int clampe(int e) { return max(-60, min(60, e)); }
};

// Per-head maxima of two permuted [heads, N*128] bf16 tensors (grid z picks
// the tensor: V, dO), as bf16 bit patterns; amax[2][heads] must be zeroed first.
struct Tensors2 {
  const uint4 *src[2];
  uint4 *dst[2];
};
__global__ void __launch_bounds__(256) head_absmax2_kernel(const Tensors2 t, int64_t words_per_head, int heads,
                                                           uint32_t *__restrict__ amax) {
  const uint4 *src = t.src[blockIdx.z] + (int64_t)blockIdx.y * words_per_head;
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
    atomicMax(amax + blockIdx.z * heads + blockIdx.y, m);
  }
}

// dst[z] = fp16(src[z] * 2^e) with the tensor's BwdScales exponent.
__global__ void __launch_bounds__(256) to_f16x2_kernel(const Tensors2 t, int64_t words_per_head, int heads,
                                                       const uint32_t *__restrict__ amax) {
  const int z = blockIdx.z;
  const int64_t base = (int64_t)blockIdx.y * words_per_head;
  const BwdScales sc(amax, heads, blockIdx.y);
  const float s = pow2f(z == 0 ? sc.ev : sc.edo);
  const uint4 *src = t.src[z];
  uint4 *dst = t.dst[z];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words_per_head; i += stride) {
    const uint4 w = __ldg(src + base + i);
    uint4 r;
    r.x = pack_f16(bf16_lo(w.x) * s, bf16_hi(w.x) * s);
    r.y = pack_f16(bf16_lo(w.y) * s, bf16_hi(w.y) * s);
    r.z = pack_f16(bf16_lo(w.z) * s, bf16_hi(w.z) * s);
    r.w = pack_f16(bf16_lo(w.w) * s, bf16_hi(w.w) * s);
    dst[base + i] = r;
  }
}

// Per query row (one warp each): D = rowsum(dO o (O + residual)), and the
// two factors that turn the row's scores into 2^15 P:
// m = -(ceil(LSE log2e) - 15) and inv = 2^(ceil(LSE log2e) - LSE log2e), so
// that 2^(x - (ceil(LSE log2e) - 15)) inv = 2^15 P.  Rows whose LSE is not
// finite (no selected keys) get m = -inf, inv = 0.
__global__ void __launch_bounds__(256) bwd_stats_tc_kernel(const __nv_bfloat16 *__restrict__ o,
                                                           const __nv_bfloat16 *__restrict__ o_res,
                                                           const __nv_bfloat16 *__restrict__ dout,
                                                           const float *__restrict__ lse, int64_t rows,
                                                           float *__restrict__ delta, float *__restrict__ stat_m,
                                                           float *__restrict__ stat_inv) {
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const uint2 ua = *reinterpret_cast<const uint2 *>(o + r * 128 + lane * 4);
  const uint2 ub = *reinterpret_cast<const uint2 *>(dout + r * 128 + lane * 4);
  float o0 = bf16_lo(ua.x), o1 = bf16_hi(ua.x), o2 = bf16_lo(ua.y), o3 = bf16_hi(ua.y);
  if (o_res) {
    const uint2 ur = *reinterpret_cast<const uint2 *>(o_res + r * 128 + lane * 4);
    o0 += bf16_lo(ur.x);
    o1 += bf16_hi(ur.x);
    o2 += bf16_lo(ur.y);
    o3 += bf16_hi(ur.y);
  }
  float s = (o0 * bf16_lo(ub.x) + o1 * bf16_hi(ub.x)) + (o2 * bf16_lo(ub.y) + o3 * bf16_hi(ub.y));
  s = warp_sum(s);
  if (lane == 0) {
    delta[r] = s;
    const float L2 = lse[r] * 1.4426950408889634f;
    if (isfinite(L2)) {
      const float c = ceilf(L2);
      stat_m[r] = 15.f - c;
      stat_inv[r] = exp2f(c - L2);
    } else {
      stat_m[r] = -INFINITY;
      stat_inv[r] = 0.f;
    }
  }
}

constexpr int kFbThreads = 512;
constexpr int kFbQStages = 2;
// K, V, dS_hi, dS_lo, 2 x Q, dO tiles (fp16); D of the query tile in two
// stages (with Q), m and inv in one (with dO: they are read only before dV,
// which frees dO); barriers.  The dynamic shared window starts 1024-byte
// aligned (no static shared memory here); the kernel checks it.
constexpr int kFbSmemBytes = kTcTileBytes * (5 + kFbQStages) + kFbQStages * 512 + 1024 + 256;
static_assert(kFbSmemBytes <= 232448, "backward shared memory");

// Float offset of (row, column quad j) of head h in the dQ accumulator.
__device__ __forceinline__ int64_t dqacc_off(int64_t N, int h, int64_t row, int j) {
  return (((int64_t)h * (N >> 6) + (row >> 6)) * 32 + j) * 256 + (row & 63) * 4;
}

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
template <int R>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
constexpr int kFbRegsDrain = 152, kFbRegsMath = 128, kFbRegsIssue = 104;
static_assert(kFbRegsDrain + 2 * kFbRegsMath + kFbRegsIssue <= 4 * 128, "register split above the launch budget");

__global__ void __launch_bounds__(kFbThreads, 1) bsa_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                  const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const __grid_constant__ CUtensorMap tmO,
                                                                  const TcBwdArgs args, float *dqacc) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t *sgen = smem_raw + (sbase - smem_u32(smem_raw));
  if (sbase != smem_u32(smem_raw)) {   // the layout has no alignment slack
    if (threadIdx.x == 0) set_status(PRISM_EBOUNDS);
    return;
  }
  const uint32_t sK = sbase, sV = sbase + kTcTileBytes;
  const uint32_t sDS = sbase + 2 * kTcTileBytes, sDSlo = sbase + 3 * kTcTileBytes;
  auto sQ = [&](int s) { return sbase + (uint32_t)(4 + s) * kTcTileBytes; };
  const uint32_t sO = sbase + (uint32_t)(4 + kFbQStages) * kTcTileBytes;
  const uint32_t sStat0 = sbase + (uint32_t)(5 + kFbQStages) * kTcTileBytes;
  auto sD = [&](int s) { return sStat0 + 512u * (uint32_t)s; };   // [stage][128] D 2^e_dS
  const uint32_t sMI = sStat0 + 512u * kFbQStages;                 // [m | inv][128]
  const uint32_t sBar = sMI + 1024;
  const uint32_t b_kv = sBar;
  auto b_qfull = [&](int s) { return sBar + 8u * (1 + s); };    // Q_n and its rows of D landed
  auto b_qempty = [&](int s) { return sBar + 8u * (3 + s); };
  const uint32_t b_s = sBar + 8u * 5;       // S^T_n done
  const uint32_t b_dp = sBar + 8u * 6;      // dP^T_n done
  const uint32_t b_p = sBar + 8u * 7;       // P^T_n written (256 arrivals)
  const uint32_t b_ds = sBar + 8u * 8;      // dS^T_n written to TMEM and shared memory (256 arrivals)
  const uint32_t b_dq = sBar + 8u * 9;      // dQ_n done
  const uint32_t b_dqfree = sBar + 8u * 10; // dQ_n read out of TMEM (128 arrivals)
  const uint32_t b_drain = sBar + 8u * 11;
  const uint32_t b_ofull = sBar + 8u * 12;  // dO_n and its rows of m, inv landed
  const uint32_t b_oempty = sBar + 8u * 13; // dO_n read by dP^T_n and dV_n
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sgen + (sBar - sbase) + 8 * 14);
  volatile int *abort = reinterpret_cast<volatile int *>(sgen + (sBar - sbase) + 8 * 14 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  ZoneTile zt;
  if (!zt.init(args.blocks, args.zone_blk_base, blockIdx.x >> 3, blockIdx.x & 7)) return;
  const int e0 = args.col_ptr[(int64_t)h * args.cap + zt.blk];
  const int e1 = args.col_ptr[(int64_t)h * args.cap + zt.blk + 1];
  const int row_base = (int)((int64_t)h * args.N);

  if (threadIdx.x == 0) {
    tc::mbar_init(b_kv, 1);
    for (int s = 0; s < kFbQStages; ++s) {
      tc::mbar_init(b_qfull(s), 1);
      tc::mbar_init(b_qempty(s), 1);
    }
    tc::mbar_init(b_s, 1);
    tc::mbar_init(b_dp, 1);
    tc::mbar_init(b_p, 256);
    tc::mbar_init(b_ds, 256);
    tc::mbar_init(b_dq, 1);
    tc::mbar_init(b_dqfree, 128);
    tc::mbar_init(b_drain, 1);
    tc::mbar_init(b_ofull, 1);
    tc::mbar_init(b_oempty, 1);
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 12) {
    tc::tmem_alloc(smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tdK = tmem, tdV = tmem + 128, tS = tmem + 256, tDP = tmem + 384;
  const uint32_t limit = args.wait_limit;

  if (warp >= 12) {
    setmaxnreg_dec<kFbRegsIssue>();
    if (warp == 13) {
      // ---------------------------------------------------------------- producer
      if (lane == 0) {
        tc::prefetch_tmap(&tmQ);
        tc::prefetch_tmap(&tmK);
        tc::prefetch_tmap(&tmV);
        tc::prefetch_tmap(&tmO);
        tc::mbar_expect_tx(b_kv, 2 * kTcTileBytes);
        tc::tma_load_2d(sK, &tmK, 0, row_base + zt.r0, b_kv);
        tc::tma_load_2d(sK + kTcTileBytes / 2, &tmK, 64, row_base + zt.r0, b_kv);
        tc::tma_load_2d(sV, &tmV, 0, row_base + zt.r0, b_kv);
        tc::tma_load_2d(sV + kTcTileBytes / 2, &tmV, 64, row_base + zt.r0, b_kv);
        KeyTiles qt;   // query sub-tiles of the query blocks that selected this key block
        qt.init(args.row_idx, args.blocks, e0, e1);
        int nq = 0, no = 0;   // Q and dO fills issued
        for (; qt.valid(); qt.next()) {
          const int s = nq % kFbQStages;
          if (!tc::mbar_wait(b_qempty(s), ((uint32_t)(nq / kFbQStages) & 1u) ^ 1u, abort, limit)) break;
          tc::mbar_expect_tx(b_qfull(s), kTcTileBytes + 512);
          tc::bulk_load(sD(s), args.delta_pad + row_base + qt.row(), 512, b_qfull(s));
          tc::tma_load_2d(sQ(s), &tmQ, 0, row_base + qt.row(), b_qfull(s));
          tc::tma_load_2d(sQ(s) + kTcTileBytes / 2, &tmQ, 64, row_base + qt.row(), b_qfull(s));
          ++nq;
          // dV of the previous tile done: its P phase, the last reader of m and inv, is over
          if (!tc::mbar_wait(b_oempty, ((uint32_t)(nq - 1) & 1u) ^ 1u, abort, limit)) break;
          tc::mbar_expect_tx(b_ofull, kTcTileBytes + 1024);
          tc::bulk_load(sMI, args.stat_m + row_base + qt.row(), 512, b_ofull);
          tc::bulk_load(sMI + 512, args.stat_inv + row_base + qt.row(), 512, b_ofull);
          tc::tma_load_2d(sO, &tmO, 0, row_base + qt.row(), b_ofull);
          tc::tma_load_2d(sO + kTcTileBytes / 2, &tmO, 64, row_base + qt.row(), b_ofull);
          ++no;
        }
        // wait (bounded, ignoring abort) for the copies still in flight before the CTA may exit
        volatile int no_abort = 0;
        tc::mbar_wait(b_kv, 0, &no_abort, limit);
        for (int k = max(0, nq - kFbQStages); k < nq; ++k)
          tc::mbar_wait(b_qfull(k % kFbQStages), (uint32_t)(k / kFbQStages) & 1u, &no_abort, limit);
        if (no > 0) tc::mbar_wait(b_ofull, (uint32_t)(no - 1) & 1u, &no_abort, limit);
      }
    } else if (warp == 12) {
      // -------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        const int nsteps = count_key_tiles(args.row_idx, args.blocks, e0, e1);
        constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);   // S^T: bf16, both K-major
        constexpr uint32_t idDP = tc::idesc_f16(128, 128, false, false);   // dP^T: fp16, both K-major
        constexpr uint32_t idV = tc::idesc_f16(128, 128, false, true);     // dV: fp16, B MN-major
        constexpr uint32_t idK = tc::idesc_bf16(128, 128, false, true);    // dK: bf16, B MN-major
        constexpr uint32_t idQ = tc::idesc_bf16(128, 128, true, true);     // dQ: bf16, A and B MN-major
        bool ok = tc::mbar_wait(b_kv, 0, abort, limit);
        const uint64_t dK = tc::sw128_desc(sK, 16, 1024), dV = tc::sw128_desc(sV, 16, 1024);
        const uint64_t dKmn = tc::sw128_desc(sK, kTcTileBytes / 2, 1024);   // K as B of dQ: [keys][d]
        const uint64_t dSmn = tc::sw128_desc(sDS, kTcTileBytes / 2, 1024);  // dS_hi as A of dQ: [keys][queries]
        const uint64_t dSlo = tc::sw128_desc(sDSlo, kTcTileBytes / 2, 1024); // dS_lo, the same layout
        auto issue_s = [&](int n) {   // S^T_n = K Q_n^T
          const uint64_t dQ = tc::sw128_desc(sQ(n % kFbQStages), 16, 1024);
  #pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (uint32_t)(k >> 2) * (kTcTileBytes / 2) + (uint32_t)(k & 3) * 32u;
            tc::mma_ss(tS, tc::desc_adv(dK, off), tc::desc_adv(dQ, off), idS, k > 0);
          }
          tc::mma_commit(b_s);
        };
        auto issue_dp = [&]() {   // dP^T_n = V dO_n^T
          const uint64_t dO = tc::sw128_desc(sO, 16, 1024);
  #pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (uint32_t)(k >> 2) * (kTcTileBytes / 2) + (uint32_t)(k & 3) * 32u;
            tc::mma_ss(tDP, tc::desc_adv(dV, off), tc::desc_adv(dO, off), idDP, k > 0);
          }
          tc::mma_commit(b_dp);
        };
        auto wait_q = [&](int n) {
          return tc::mbar_wait(b_qfull(n % kFbQStages), (uint32_t)(n / kFbQStages) & 1u, abort, limit);
        };
        auto wait_o = [&](int n) { return tc::mbar_wait(b_ofull, (uint32_t)n & 1u, abort, limit); };
        if (ok && nsteps > 0) {
          ok = wait_q(0);
          if (ok) {
            tc::tc_fence_after();
            issue_s(0);
            ok = wait_o(0);
            if (ok) {
              tc::tc_fence_after();
              issue_dp();
            }
          }
        }
        for (int n = 0; ok && n < nsteps; ++n) {
          const int s = n % kFbQStages;
          const bool more = n + 1 < nsteps;
          if (!tc::mbar_wait(b_p, (uint32_t)n & 1u, abort, limit)) break;
          tc::tc_fence_after();
          const uint64_t dOmn = tc::sw128_desc(sO, kTcTileBytes / 2, 1024);
  #pragma unroll
          for (int k = 0; k < 8; ++k)   // dV += P^T_n dO_n, 16 queries per step
            tc::mma_ts(tdV, tS + half_col(k), tc::desc_adv(dOmn, 2048u * k), idV, (n > 0 || k > 0) ? 1u : 0u);
          tc::mma_commit(b_oempty);      // dO_n read by dP^T_n and dV_n
          if (more) {
            if (!wait_q(n + 1)) break;
            tc::tc_fence_after();
            issue_s(n + 1);
          }
          if (!tc::mbar_wait(b_ds, (uint32_t)n & 1u, abort, limit)) break;
          tc::tc_fence_after();
          const uint64_t dQmn = tc::sw128_desc(sQ(s), kTcTileBytes / 2, 1024);
  #pragma unroll
          for (int k = 0; k < 8; ++k)   // dK += dS_hi^T_n Q_n
            tc::mma_ts(tdK, tDP + half_col(k), tc::desc_adv(dQmn, 2048u * k), idK, (n > 0 || k > 0) ? 1u : 0u);
  #pragma unroll
          for (int k = 0; k < 8; ++k)   // dK += dS_lo^T_n Q_n, 32 columns further on
            tc::mma_ts(tdK, tDP + half_col(k) + 32u, tc::desc_adv(dQmn, 2048u * k), idK, 1u);
          tc::mma_commit(b_qempty(s));   // Q_n read by S^T_n and dK_n
  #pragma unroll
          for (int k = 0; k < 8; ++k)   // dQ_n = dS_hi K + dS_lo K, 16 keys per step, over the dS^T columns
            tc::mma_ss(tDP, tc::desc_adv(dSmn, 2048u * k), tc::desc_adv(dKmn, 2048u * k), idQ, k > 0);
  #pragma unroll
          for (int k = 0; k < 8; ++k)
            tc::mma_ss(tDP, tc::desc_adv(dSlo, 2048u * k), tc::desc_adv(dKmn, 2048u * k), idQ, 1u);
          tc::mma_commit(b_dq);
          if (more) {
            if (!tc::mbar_wait(b_dqfree, (uint32_t)n & 1u, abort, limit)) break;
            if (!wait_o(n + 1)) break;
            tc::tc_fence_after();
            issue_dp();
          }
        }
        tc::mma_commit(b_drain);
        volatile int no_abort = 0;
        tc::mbar_wait(b_drain, 0, &no_abort, limit);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------ elementwise warps
    if constexpr (kFbRegsMath > 128) setmaxnreg_inc<kFbRegsMath>();   // 128: the launch count stands
    if constexpr (kFbRegsMath < 128) setmaxnreg_dec<kFbRegsMath>();
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;        // query columns [64*half, 64*half + 64)
    const int row = 32 * q + lane;           // key row of the tile
    const bool krow = row < zt.rows;         // padding key rows of a 64-key tile give dS = 0 for dQ
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const uint32_t colS = tS + lane_off + 64u * (uint32_t)half, colDP = tDP + lane_off + 64u * (uint32_t)half;
    // this thread's 128-byte row of dS in the MN-major A operand of dQ: half `half` of the
    // query columns, key row `row`, 16-byte chunks swizzled by the row's low three bits
    uint8_t *ds_row = sgen + (sDS - sbase) + (uint32_t)half * (kTcTileBytes / 2) + (uint32_t)row * 128u;
    const BwdScales sc(args.amax, args.heads, h);
    const float cS = args.scale_log2;                  // S^T -> log2 units
    const float cdP = pow2f(-sc.ev - sc.edo);          // dP^T (scaled fp16 operands) -> dP
    KeyTiles qt;
    qt.init(args.row_idx, args.blocks, e0, e1);
    int n = 0;
    bool ok = true;
    for (; qt.valid(); qt.next(), ++n) {
      const int qv = qt.keys();   // valid queries in this tile
      const int s = n % kFbQStages;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_qfull(s), (uint32_t)(n / kFbQStages) & 1u, abort, limit))) {
        ok = false;
        break;
      }
      const float4 *st_m = reinterpret_cast<const float4 *>(sgen + (sMI - sbase)) + 16 * half;
      const float4 *st_i = st_m + 32;
      const float4 *st_d = reinterpret_cast<const float4 *>(sgen + (sD(s) - sbase)) + 16 * half;
      // ---- P^T over S^T (dV of the previous tile, which read P^T there, ran before S^T_n)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_s, (uint32_t)n & 1u, abort, limit) &&
                                       tc::mbar_wait(b_ofull, (uint32_t)n & 1u, abort, limit))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      uint32_t pv[2][32];   // S^T, then 2^15 P (the forward's truncated form) kept for dS^T
      tc::tmem_ld32(colS, pv[0]);
      tc::tmem_ld32(colS + 32u, pv[1]);
      tc::tmem_ld_wait();
      const bool full = qv >= 64 * half + 64;   // no padding columns in this half
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pa[16];
#pragma unroll
        for (int g = 0; g < 8; ++g) {   // four query columns at a time
          float4 M = st_m[8 * cc + g];  // -(ceil(LSE log2e) - 15)
          float4 I = st_i[8 * cc + g];  // 2^(ceil(LSE log2e) - LSE log2e)
          if (!full) {
            const int c0 = 64 * half + 32 * cc + 4 * g;
            if (c0 + 0 >= qv) M.x = -INFINITY, I.x = 0.f;
            if (c0 + 1 >= qv) M.y = -INFINITY, I.y = 0.f;
            if (c0 + 2 >= qv) M.z = -INFINITY, I.z = 0.f;
            if (c0 + 3 >= qv) M.w = -INFINITY, I.w = 0.f;
          }
          const float2 x01 = tc::fma2(tc::f2u(pv[cc][4 * g + 0], pv[cc][4 * g + 1]), tc::f2(cS, cS), tc::f2(M.x, M.y));
          const float2 x23 = tc::fma2(tc::f2u(pv[cc][4 * g + 2], pv[cc][4 * g + 3]), tc::f2(cS, cS), tc::f2(M.z, M.w));
          const float p0 = tc::ex2(x01.x), p1 = tc::ex2(x01.y), p2 = tc::ex2(x23.x), p3 = tc::ex2(x23.y);
          // 2^15 P, from the forward's truncated values; dV takes it rounded to fp16
          const float2 c01 = tc::mul2(tc::f2(trunc11(p0), trunc11(p1)), tc::f2(I.x, I.y));
          const float2 c23 = tc::mul2(tc::f2(trunc11(p2), trunc11(p3)), tc::f2(I.z, I.w));
          pv[cc][4 * g + 0] = __float_as_uint(c01.x);
          pv[cc][4 * g + 1] = __float_as_uint(c01.y);
          pv[cc][4 * g + 2] = __float_as_uint(c23.x);
          pv[cc][4 * g + 3] = __float_as_uint(c23.y);
          pa[2 * g] = pack_f16(c01.x, c01.y);
          pa[2 * g + 1] = pack_f16(c23.x, c23.y);
        }
        tc::tmem_st16(colS + 16u * cc, pa);
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      if (!(args.debug_stall && n == 0)) tc::mbar_arrive(b_p);
      // ---- dS^T = P^T (dP^T - D): over dP^T for dK, and into shared memory for dQ.
      // dP^T_n ran after the drain warps had read dQ_{n-1}, and dQ_{n-1} after it read dS.
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_dp, (uint32_t)n & 1u, abort, limit))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      // four chunks of 16 query columns; chunk c+1's load overlaps chunk c's arithmetic
      uint32_t dpa[16], dpb[16], lo01[8];
      tc::tmem_ld16(colDP, dpa);
      tc::tmem_ld_wait_regs(dpa);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t(&cur)[16] = (c & 1) ? dpb : dpa;
        uint32_t(&nxt)[16] = (c & 1) ? dpa : dpb;
        if (c < 3) tc::tmem_ld16(colDP + 16u * (c + 1), nxt);
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int g = 0; g < 4; ++g) {   // four query columns at a time: 16c + 4g ..
          const float4 Dv = st_d[4 * c + g];   // padding columns have P = 0, so dS = 0 there
          const int j = 16 * c + 4 * g;        // column within the half
          const uint32_t *pc = &pv[j >> 5][j & 31];
          // 2^15 dS = 2^15 P (dP - D)
          const float2 d01 = tc::mul2(tc::f2u(pc[0], pc[1]),
                                      tc::fma2(tc::f2u(cur[4 * g + 0], cur[4 * g + 1]), tc::f2(cdP, cdP), tc::f2(-Dv.x, -Dv.y)));
          const float2 d23 = tc::mul2(tc::f2u(pc[2], pc[3]),
                                      tc::fma2(tc::f2u(cur[4 * g + 2], cur[4 * g + 3]), tc::f2(cdP, cdP), tc::f2(-Dv.z, -Dv.w)));
          // dS_hi = dS truncated to bf16 (the top 16 bits), dS_lo = bf16(dS - dS_hi), the
          // difference exact in fp32: about 16 significant bits together
          const float h0 = __uint_as_float(__float_as_uint(d01.x) & 0xffff0000u);
          const float h1 = __uint_as_float(__float_as_uint(d01.y) & 0xffff0000u);
          const float h2 = __uint_as_float(__float_as_uint(d23.x) & 0xffff0000u);
          const float h3 = __uint_as_float(__float_as_uint(d23.y) & 0xffff0000u);
          hi[2 * g] = __byte_perm(__float_as_uint(d01.x), __float_as_uint(d01.y), 0x7632);
          hi[2 * g + 1] = __byte_perm(__float_as_uint(d23.x), __float_as_uint(d23.y), 0x7632);
          const float2 r01 = tc::sub2(d01, tc::f2(h0, h1));
          const float2 r23 = tc::sub2(d23, tc::f2(h2, h3));
          lo[2 * g] = pack_bf16(r01.x, r01.y);
          lo[2 * g + 1] = pack_bf16(r23.x, r23.y);
        }
        tc::tmem_st8(colDP + 8u * c, hi);   // columns already read
#pragma unroll
        for (int u = 0; u < 2; ++u) {   // 16-byte chunk 2c + u of the row: queries 8(2c + u) .. +7
          const int ch = 2 * c + u;
          const uint32_t off = (uint32_t)((ch ^ (row & 7)) << 4);
          const uint4 w = krow ? make_uint4(hi[4 * u], hi[4 * u + 1], hi[4 * u + 2], hi[4 * u + 3])
                               : make_uint4(0u, 0u, 0u, 0u);
          const uint4 wl = krow ? make_uint4(lo[4 * u], lo[4 * u + 1], lo[4 * u + 2], lo[4 * u + 3])
                                : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4 *>(ds_row + off) = w;
          *reinterpret_cast<uint4 *>(ds_row + kTcTileBytes + off) = wl;
        }
        // dS_lo^T goes to columns 32 + 8c, which chunks 2 and 3 occupy until they are read
        if (c < 3) tc::tmem_ld_wait_regs(nxt);
        if (c == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) lo01[e] = lo[e];
        } else if (c == 1) {   // chunk 2 has been read
          tc::tmem_st8(colDP + 32u, lo01);
          tc::tmem_st8(colDP + 40u, lo);
        } else if (c == 2) {   // chunk 3 has been read
          tc::tmem_st8(colDP + 48u, lo);
        } else {
          tc::tmem_st8(colDP + 56u, lo);
        }
      }
      tc::tmem_st_wait();
      fence_proxy_async_smem();   // the dQ product reads dS through the async proxy
      tc::tc_fence_before();
      tc::mbar_arrive(b_ds);
    }
    if (__all_sync(0xffffffffu, ok && !*abort) && row < zt.rows) {
      bool have = n > 0;
      if (have && !__all_sync(0xffffffffu, tc::mbar_wait(b_drain, 0, abort, limit))) have = false;
      if (!*abort) {
        if (have) tc::tc_fence_after();
        const int64_t grow = (int64_t)h * args.N + zt.r0 + row;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          __nv_bfloat16 *out = (which ? args.dv : args.dk) + grow * 128 + 64 * half;
          // dV carries 2^(e_dO + 15), dK 2^15 and lacks the softmax scale
          const float mul = which ? pow2f(-sc.edo - 15) : args.scale * (1.f / 32768.f);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t v[32];
            if (have) {
              tc::tmem_ld32((which ? tdV : tdK) + lane_off + 64u * half + 32u * cc, v);
              tc::tmem_ld_wait();
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = 0u;
            }
#pragma unroll
            for (int v8 = 0; v8 < 4; ++v8) {
              uint4 w;
              uint32_t *wp = &w.x;
#pragma unroll
              for (int e = 0; e < 4; ++e)
                wp[e] = pack_bf16(__uint_as_float(v[8 * v8 + 2 * e]) * mul, __uint_as_float(v[8 * v8 + 2 * e + 1]) * mul);
              *reinterpret_cast<uint4 *>(out + 32 * cc + 8 * v8) = w;
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ drain
    setmaxnreg_inc<kFbRegsDrain>();
    const int q = warp;
    const int r = 32 * q + lane;             // query row of the tile
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    KeyTiles qt;
    qt.init(args.row_idx, args.blocks, e0, e1);
    int n = 0;
    for (; qt.valid(); qt.next(), ++n) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_dq, (uint32_t)n & 1u, abort, limit))) break;
      tc::tc_fence_after();
      const bool vrow = r < qt.keys();
      const int64_t grow = (int64_t)qt.row() + r;
      float *dst = dqacc + dqacc_off(args.N, h, grow, 0);
      uint32_t v[4][32];   // the whole row first: the columns are free for dP^T_{n+1} at once
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(tDP + lane_off + 32u * c, v[c]);
      tc::tmem_ld_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(b_dqfree);
      if (vrow) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 8; ++j)        // column quad 8 c + j
            red_add_v4(dst + (int64_t)(8 * c + j) * 256, __uint_as_float(v[c][4 * j]),
                       __uint_as_float(v[c][4 * j + 1]), __uint_as_float(v[c][4 * j + 2]),
                       __uint_as_float(v[c][4 * j + 3]));
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// dQ = scale 2^-15 * accumulator, one CTA per (64-row group, head): the
// group's 32 KB of the accumulator is read contiguously, transposed through
// shared memory and written as 64 contiguous bf16 rows of 128.
__global__ void __launch_bounds__(256) dq_convert_kernel(const float *__restrict__ dqacc, int64_t N, float scale,
                                                         __nv_bfloat16 *__restrict__ dq) {
  __shared__ float4 t[64][33];   // [row][column quad], padded against bank conflicts
  const int64_t grp = blockIdx.x, h = blockIdx.y;
  const float mul = scale * (1.f / 32768.f);
  const float4 *src = reinterpret_cast<const float4 *>(dqacc + ((int64_t)h * (N >> 6) + grp) * 8192);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int f = it * 256 + threadIdx.x;   // f = quad * 64 + row
    t[f & 63][f >> 6] = src[f];
  }
  __syncthreads();
  __nv_bfloat16 *out = dq + ((int64_t)h * N + grp * 64) * 128;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int u = it * 256 + threadIdx.x;   // 8-column piece: row u / 16, columns 8 (u % 16) ..
    const int rr = u >> 4, p = u & 15;
    const float4 a = t[rr][2 * p], b = t[rr][2 * p + 1];
    uint4 w;
    w.x = pack_bf16(a.x * mul, a.y * mul);
    w.y = pack_bf16(a.z * mul, a.w * mul);
    w.z = pack_bf16(b.x * mul, b.y * mul);
    w.w = pack_bf16(b.z * mul, b.w * mul);
    *reinterpret_cast<uint4 *>(out + (int64_t)rr * 128 + 8 * p) = w;
  }
}

}  // namespace prism
