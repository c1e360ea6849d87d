// Block-sparse attention backward in one tcgen05 kernel (head_dim 128): dK, dV
// and dQ from one pass over the transposed selection.
//
// bsa_bwd_tc_kernel  one CTA per (128-key tile, head), walking the query tiles
//   of the query blocks that selected its key block.  Per query tile n:
//     S^T_n  = K Q_n^T          (both operands in shared memory)
//     dP^T_n = V dO_n^T
//     P^T_n  = exp2(S^T scale log2e - LSE log2e)  bf16 over S^T      (elementwise warps)
//     dV    += P^T_n dO_n       (A from tensor memory)
//     dS^T_n = P^T (dP^T - D)   bf16 over dP^T, and into shared memory
//     dK    += dS^T_n Q_n       (A from tensor memory, as the same bf16 pair:
//                                the sum runs over every selecting query row)
//     dQ_n   = dS_n K           (A = dS from shared memory, MN-major, as a bf16
//                                pair dS_hi + dS_lo, dS_lo = bf16(dS - dS_hi):
//                                two products, about 16 significant bits of dS;
//                                written over the dP^T columns once dK_n has
//                                read dS^T)
//   and four drain warps move dQ_n out of tensor memory into an fp32
//   accumulator in global memory with vector reductions (red.global.add.v4).
//   The query-side recomputation of S and dP (and of P's exponentials) that a
//   kernel owning dQ needs is gone: five products and one exponential per
//   score instead of seven and two.  The price is that dQ is summed in fp32
//   in the order the reductions reach L2 (not bit-reproducible run to run).
//
//   Tensor-pipe order per tile: dV_n, S^T_{n+1}, dK_n (hi, lo), dQ_n (hi,
//   lo), dP^T_{n+1}; the last waits until dQ_n has left the shared columns.
//   dS_hi^T sits in the first 32 columns of each elementwise half's 64 in the
//   dP^T range, dS_lo^T in the next 32.
//   The split dS matters for dQ: each row of dS sums to zero (D is the
//   P-weighted mean of dP), so dQ_r = scale sum_c dS_rc k_c cancels, and a
//   single bf16 rounding of every dS_rc (2^-9) leaves errors that do not.
//   Shared memory holds Q in two stages and dO in one (dO_{n+1} is loaded
//   while S^T_{n+1}, dK_n and dQ_n run).
//   TMEM: dK | dV | S^T (P^T) | dP^T (dS^T, then dQ).
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
// 128 per thread, the elementwise warpgroups take 144 each (their state, P of
// the row half kept for dS, stays unspilled), the drain warpgroup keeps 112
// (half a dQ row at a time) and the MMA/producer warpgroup 112
// (112 + 2 x 144 + 112 = 4 x 128).
// Every wait is bounded and follows the abort protocol of the other tcgen05
// kernels.
#pragma once

#include "attn_tc_bwd.cuh"

namespace prism {

constexpr int kFbThreads = 512;
constexpr int kFbQStages = 2;
// K, V, dS_hi, dS_lo, 2 x Q, dO tiles; 2 x (LSE*log2e, D) rows of 128 floats; barriers.
constexpr int kFbSmemBytes = kTcTileBytes * (5 + kFbQStages) + 2 * 1024 + 256;
static_assert(kFbSmemBytes <= 232448, "fused backward shared memory");

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
constexpr int kFbRegsDrain = 112, kFbRegsMath = 144, kFbRegsIssue = 112;
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
  const uint32_t sStat0 = sbase + (uint32_t)(5 + kFbQStages) * kTcTileBytes;   // [2][256] floats
  auto sStat = [&](int s) { return sStat0 + 1024u * (uint32_t)s; };
  const uint32_t sBar = sStat0 + 2048;
  const uint32_t b_kv = sBar;
  auto b_qfull = [&](int s) { return sBar + 8u * (1 + s); };    // Q_n and its rows of LSE, D landed
  auto b_qempty = [&](int s) { return sBar + 8u * (3 + s); };
  const uint32_t b_s = sBar + 8u * 5;       // S^T_n done
  const uint32_t b_dp = sBar + 8u * 6;      // dP^T_n done
  const uint32_t b_p = sBar + 8u * 7;       // P^T_n written (256 arrivals)
  const uint32_t b_ds = sBar + 8u * 8;      // dS^T_n written to TMEM and shared memory (256 arrivals)
  const uint32_t b_dq = sBar + 8u * 9;      // dQ_n done
  const uint32_t b_dqfree = sBar + 8u * 10; // dQ_n read out of TMEM (128 arrivals)
  const uint32_t b_drain = sBar + 8u * 11;
  const uint32_t b_ofull = sBar + 8u * 12;  // dO_n landed
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
          tc::mbar_expect_tx(b_qfull(s), kTcTileBytes + 1024);
          tc::bulk_load(sStat(s), args.lse2_pad + row_base + qt.row(), 512, b_qfull(s));
          tc::bulk_load(sStat(s) + 512, args.delta_pad + row_base + qt.row(), 512, b_qfull(s));
          tc::tma_load_2d(sQ(s), &tmQ, 0, row_base + qt.row(), b_qfull(s));
          tc::tma_load_2d(sQ(s) + kTcTileBytes / 2, &tmQ, 64, row_base + qt.row(), b_qfull(s));
          ++nq;
          if (!tc::mbar_wait(b_oempty, ((uint32_t)(nq - 1) & 1u) ^ 1u, abort, limit)) break;
          tc::mbar_expect_tx(b_ofull, kTcTileBytes);
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
        constexpr uint32_t idNT = tc::idesc_bf16(128, 128, false, false);   // S^T, dP^T: both K-major
        constexpr uint32_t idMN = tc::idesc_bf16(128, 128, false, true);    // dV, dK: B MN-major
        constexpr uint32_t idQ = tc::idesc_bf16(128, 128, true, true);      // dQ: A and B MN-major
        bool ok = tc::mbar_wait(b_kv, 0, abort, limit);
        const uint64_t dK = tc::sw128_desc(sK, 16, 1024), dV = tc::sw128_desc(sV, 16, 1024);
        const uint64_t dKmn = tc::sw128_desc(sK, kTcTileBytes / 2, 1024);   // K as B of dQ: [d][keys]
        const uint64_t dSmn = tc::sw128_desc(sDS, kTcTileBytes / 2, 1024);  // dS_hi as A of dQ: [queries][keys]
        const uint64_t dSlo = tc::sw128_desc(sDSlo, kTcTileBytes / 2, 1024); // dS_lo, the same layout
        auto issue_s = [&](int n) {   // S^T_n = K Q_n^T
          const uint64_t dQ = tc::sw128_desc(sQ(n % kFbQStages), 16, 1024);
  #pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (uint32_t)(k >> 2) * (kTcTileBytes / 2) + (uint32_t)(k & 3) * 32u;
            tc::mma_ss(tS, tc::desc_adv(dK, off), tc::desc_adv(dQ, off), idNT, k > 0);
          }
          tc::mma_commit(b_s);
        };
        auto issue_dp = [&]() {   // dP^T_n = V dO_n^T
          const uint64_t dO = tc::sw128_desc(sO, 16, 1024);
  #pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (uint32_t)(k >> 2) * (kTcTileBytes / 2) + (uint32_t)(k & 3) * 32u;
            tc::mma_ss(tDP, tc::desc_adv(dV, off), tc::desc_adv(dO, off), idNT, k > 0);
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
            tc::mma_ts(tdV, tS + half_col(k), tc::desc_adv(dOmn, 2048u * k), idMN, (n > 0 || k > 0) ? 1u : 0u);
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
          for (int k = 0; k < 8; ++k)   // dK += dS^T_n Q_n
            tc::mma_ts(tdK, tDP + half_col(k), tc::desc_adv(dQmn, 2048u * k), idMN, (n > 0 || k > 0) ? 1u : 0u);
  #pragma unroll
          for (int k = 0; k < 8; ++k)   // dK += dS_lo^T_n Q_n
            tc::mma_ts(tdK, tDP + half_col(k) + 32u, tc::desc_adv(dQmn, 2048u * k), idMN, 1u);
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
    setmaxnreg_inc<kFbRegsMath>();
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;        // query columns [64*half, 64*half + 64)
    const int row = 32 * q + lane;           // key row of the tile
    const bool krow = row < zt.rows;         // padding key rows of a 64-key tile give dS = 0 for dQ
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const uint32_t colS = tS + lane_off + 64u * (uint32_t)half, colDP = tDP + lane_off + 64u * (uint32_t)half;
    // this thread's 128-byte row of dS in the MN-major A operand of dQ: half `half` of the
    // query columns, key row `row`, 16-byte chunks swizzled by the row's low three bits
    uint8_t *ds_row = sgen + (sDS - sbase) + (uint32_t)half * (kTcTileBytes / 2) + (uint32_t)row * 128u;
    const float sl2 = args.scale_log2;
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
      const float4 *st_l = reinterpret_cast<const float4 *>(sgen + (sStat(s) - sbase)) + 16 * half;
      const float4 *st_d = st_l + 32;
      // ---- P^T over S^T (dV of the previous tile, which read P^T there, ran before S^T_n)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_s, (uint32_t)n & 1u, abort, limit))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      uint32_t pv[2][32];   // S^T, then P^T as float bits, kept for dS^T
      tc::tmem_ld32(colS, pv[0]);
      tc::tmem_ld32(colS + 32u, pv[1]);
      tc::tmem_ld_wait();
      const bool full = qv >= 64 * half + 64;   // no padding columns in this half
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int g = 0; g < 8; ++g) {   // four query columns at a time
          float4 L = st_l[8 * cc + g];  // -LSE*log2e
          if (!full) {
            const int c0 = 64 * half + 32 * cc + 4 * g;
            if (c0 + 0 >= qv) L.x = -INFINITY;
            if (c0 + 1 >= qv) L.y = -INFINITY;
            if (c0 + 2 >= qv) L.z = -INFINITY;
            if (c0 + 3 >= qv) L.w = -INFINITY;
          }
          const float2 x01 = tc::fma2(tc::f2u(pv[cc][4 * g + 0], pv[cc][4 * g + 1]), tc::f2(sl2, sl2), tc::f2(L.x, L.y));
          const float2 x23 = tc::fma2(tc::f2u(pv[cc][4 * g + 2], pv[cc][4 * g + 3]), tc::f2(sl2, sl2), tc::f2(L.z, L.w));
          const float p0 = tc::ex2(x01.x);
          const float p1 = tc::ex2(x01.y);
          const float p2 = tc::ex2(x23.x);
          const float p3 = tc::ex2(x23.y);
          pv[cc][4 * g + 0] = __float_as_uint(p0);
          pv[cc][4 * g + 1] = __float_as_uint(p1);
          pv[cc][4 * g + 2] = __float_as_uint(p2);
          pv[cc][4 * g + 3] = __float_as_uint(p3);
          pk[2 * g] = pack_bf16(p0, p1);
          pk[2 * g + 1] = pack_bf16(p2, p3);
        }
        tc::tmem_st16(colS + 16u * cc, pk);
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      if (!(args.debug_stall && n == 0)) tc::mbar_arrive(b_p);
      // ---- dS^T = P^T (dP^T - D): over dP^T for dK, and into shared memory for dQ.
      // dP^T_n ran after dQ_{n-1} had read the previous dS from shared memory.
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_dp, (uint32_t)n & 1u, abort, limit))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      uint32_t lo0[16];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dp[32], dk[16], lo[16];
        tc::tmem_ld32(colDP + 32u * cc, dp);   // chunk 0's stores below land on columns already read
        tc::tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 Dv = st_d[8 * cc + g];   // padding columns have P = 0, so dS = 0 there
          const float2 d01 = tc::mul2(tc::f2u(pv[cc][4 * g + 0], pv[cc][4 * g + 1]),
                                      tc::sub2(tc::f2u(dp[4 * g + 0], dp[4 * g + 1]), tc::f2(Dv.x, Dv.y)));
          const float2 d23 = tc::mul2(tc::f2u(pv[cc][4 * g + 2], pv[cc][4 * g + 3]),
                                      tc::sub2(tc::f2u(dp[4 * g + 2], dp[4 * g + 3]), tc::f2(Dv.z, Dv.w)));
          dk[2 * g] = pack_bf16(d01.x, d01.y);
          dk[2 * g + 1] = pack_bf16(d23.x, d23.y);
          // the residuals d - bf16(d), exact in fp32, as the low bf16 halves
          const float2 r01 = tc::sub2(d01, tc::f2(bf16_lo(dk[2 * g]), bf16_hi(dk[2 * g])));
          const float2 r23 = tc::sub2(d23, tc::f2(bf16_lo(dk[2 * g + 1]), bf16_hi(dk[2 * g + 1])));
          lo[2 * g] = pack_bf16(r01.x, r01.y);
          lo[2 * g + 1] = pack_bf16(r23.x, r23.y);
        }
        tc::tmem_st16(colDP + 16u * cc, dk);
        // the low halves go to columns 32..63 of the range, which chunk 1's load must
        // have read first: chunk 0's are kept until then
        if (cc == 0) {
#pragma unroll
          for (int e = 0; e < 16; ++e) lo0[e] = lo[e];
        } else {
          tc::tmem_st16(colDP + 32u, lo0);
          tc::tmem_st16(colDP + 48u, lo);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {   // 16-byte chunk 4cc + c of the row: queries 8(4cc + c) .. +7
          const int ch = 4 * cc + c;
          const uint32_t off = (uint32_t)((ch ^ (row & 7)) << 4);
          const uint4 w = krow ? make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3])
                               : make_uint4(0u, 0u, 0u, 0u);
          const uint4 wl = krow ? make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3])
                                : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4 *>(ds_row + off) = w;
          *reinterpret_cast<uint4 *>(ds_row + kTcTileBytes + off) = wl;
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
          const float mul = which ? 1.f : args.scale;
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
    setmaxnreg_dec<kFbRegsDrain>();
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
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {         // columns [64 hf, 64 hf + 64)
        uint32_t v[2][32];
        tc::tmem_ld32(tDP + lane_off + 64u * hf, v[0]);
        tc::tmem_ld32(tDP + lane_off + 64u * hf + 32u, v[1]);
        tc::tmem_ld_wait();
        if (hf == 1) {                         // every column has been read: they are free
          tc::tc_fence_before();
          tc::mbar_arrive(b_dqfree);
        }
        if (vrow) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int j = 0; j < 8; ++j)        // column quad 16 hf + 8 c + j
              red_add_v4(dst + (int64_t)(16 * hf + 8 * c + j) * 256, __uint_as_float(v[c][4 * j]),
                         __uint_as_float(v[c][4 * j + 1]), __uint_as_float(v[c][4 * j + 2]),
                         __uint_as_float(v[c][4 * j + 3]));
        }
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

// dQ = scale * accumulator, one CTA per (64-row group, head): the group's
// 32 KB of the accumulator is read contiguously, transposed through shared
// memory and written as 64 contiguous bf16 rows of 128.
__global__ void __launch_bounds__(256) dq_convert_kernel(const float *__restrict__ dqacc, int64_t N, float scale,
                                                         __nv_bfloat16 *__restrict__ dq) {
  __shared__ float4 t[64][33];   // [row][column quad], padded against bank conflicts
  const int64_t grp = blockIdx.x, h = blockIdx.y;
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
    w.x = pack_bf16(a.x * scale, a.y * scale);
    w.y = pack_bf16(a.z * scale, a.w * scale);
    w.z = pack_bf16(b.x * scale, b.y * scale);
    w.w = pack_bf16(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4 *>(out + (int64_t)rr * 128 + 8 * p) = w;
  }
}

}  // namespace prism
