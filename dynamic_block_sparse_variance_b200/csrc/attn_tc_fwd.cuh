// Block-sparse attention forward on the 5th-generation tensor cores (tcgen05).
//
// One CTA per (128-row query tile, head); head_dim 128.  Six warps:
//   warp 0      TMA producer: the Q tile once, then 128-key K and V tiles of the
//               selected key blocks into a 3-stage ring (128-byte swizzle).
//   warp 1      allocates 512 TMEM columns; one thread issues the MMAs:
//               S_n = Q K_n^T (A, B from shared memory) into one of two S
//               buffers, and O += P_n V_n with P_n read from tensor memory.
//   warps 2..5  softmax, one thread per query row (its TMEM lane): S row ->
//               running max (log2 domain, an integer, moved lazily only when
//               the max grows by more than 2^8) -> P = exp2(.) truncated to
//               11 significant bits, written back over S as fp16 -> row sum
//               of those values; final normalisation, O (bf16 + residual), LSE.
// The PV product is fp16 x fp16: V comes as fp16 scaled per head by 2^e_h
// (see v16.cuh) and the epilogue folds 2^-e_h into 1/l.
// Why the integer max and the sum of truncated P: O is then exactly
// sum_c t(2^(x_c - m)) v_c / l for any integer m (truncation to 11 bits
// commutes with scaling by a power of two), so the backward, given only the
// LSE, truncates its own exp2(x_c - m') to the same values and its P matches
// the P that formed O.  The row sums D = rowsum(dO o O) of the backward are then
// consistent with its dS = P (dP - D), whose rows must sum to zero.
// MMA order S_0, S_1, PV_0, S_2, PV_1, ... lets QK^T of step n+1 run while the
// softmax of step n is computed.  Every wait is bounded; a stalled wait raises
// a CTA-wide abort, latches PRISM_ETIMEOUT and the CTA drains and frees TMEM.
#pragma once

#include "tc_common.cuh"
#include "v16.cuh"

namespace prism {

constexpr int kTcStages = 3;
constexpr int kTcTileBytes = 128 * 128 * 2;                // one 128 x 128 bf16 tile
constexpr int kTcSmemBytes = kTcTileBytes * (1 + 2 * kTcStages) + 1024 /*barriers*/ + 1024 /*align*/;

struct TcFwdArgs {
  const prism_block *blocks;
  const int32_t *zone_blk_base;
  const int32_t *row_ptr;
  const int32_t *col;
  int64_t N, cap;
  float scale_log2;
  const uint32_t *vmax;   // per head: bf16 bits of max |v|; V arrives as fp16 scaled by 2^e_h
  __nv_bfloat16 *o;
  __nv_bfloat16 *o_res;
  float *lse;
  uint32_t wait_limit;
  int debug_stall;   // test knob: the softmax never signals P_0, so the MMA wait times out
  int skip256;       // zones of 256-token blocks are left to the paired kernel
};

// Iterates the 128-key sub-tiles of the key blocks col[e0..e1).
struct KeyTiles {
  const int32_t *col;
  const prism_block *blocks;
  int e, e1, sub, nsub, size;
  int start;
  __device__ __forceinline__ void init(const int32_t *c, const prism_block *b, int e0, int e1_) {
    col = c; blocks = b; e = e0; e1 = e1_; sub = 0;
    load();
  }
  __device__ __forceinline__ void load() {
    if (e < e1) {
      const prism_block blk = blocks[col[e]];
      start = blk.start;
      size = blk.size;
      nsub = (size + 127) >> 7;
    }
  }
  __device__ __forceinline__ bool valid() const { return e < e1; }
  __device__ __forceinline__ int row() const { return start + (sub << 7); }
  __device__ __forceinline__ int keys() const { return min(128, size - (sub << 7)); }
  __device__ __forceinline__ void next() {
    if (++sub >= nsub) {
      sub = 0;
      ++e;
      load();
    }
  }
};

__device__ __forceinline__ int count_key_tiles(const int32_t *col, const prism_block *blocks, int e0, int e1) {
  int n = 0;
  for (int e = e0; e < e1; ++e) n += (blocks[col[e]].size + 127) >> 7;
  return n;
}

__global__ void __launch_bounds__(192, 1) bsa_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                            const __grid_constant__ CUtensorMap tmK,
                                                            const __grid_constant__ CUtensorMap tmV,
                                                            const TcFwdArgs args) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t *sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t sQ = sbase;
  const uint32_t sK0 = sQ + kTcTileBytes;
  auto sK = [&](int s) { return sK0 + (uint32_t)s * 2 * kTcTileBytes; };
  auto sV = [&](int s) { return sK0 + (uint32_t)s * 2 * kTcTileBytes + kTcTileBytes; };
  const uint32_t sBar = sQ + kTcTileBytes * (1 + 2 * kTcStages);
  const uint32_t b_q = sBar;
  auto b_kfull = [&](int s) { return sBar + 8u * (1 + s); };
  auto b_vfull = [&](int s) { return sBar + 8u * (4 + s); };
  auto b_kempty = [&](int s) { return sBar + 8u * (7 + s); };
  auto b_vempty = [&](int s) { return sBar + 8u * (10 + s); };
  auto b_sfull = [&](int b) { return sBar + 8u * (13 + b); };
  auto b_pfull = [&](int b) { return sBar + 8u * (15 + b); };
  const uint32_t b_ofull = sBar + 8u * 17;
  const uint32_t b_drain = sBar + 8u * 18;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sgen + (sBar - sbase) + 8 * 20);
  volatile int *abort = reinterpret_cast<volatile int *>(sgen + (sBar - sbase) + 8 * 20 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int m = blockIdx.x >> 3, t = blockIdx.x & 7;
  const int b0 = args.zone_blk_base[m];
  const int B = args.blocks[b0].size;
  if (B >= 128 && t >= 4) return;  // zones of 128/256 blocks hold four 128-row tiles
  if (B == 256 && args.skip256) return;
  int qb, r0, qrows;
  if (B == 64) {
    qb = b0 + t;
    r0 = m * kZoneTokens + 64 * t;
    qrows = 64;
  } else {
    r0 = m * kZoneTokens + 128 * t;
    qb = b0 + (128 * t) / B;
    qrows = 128;
  }
  const int e0 = args.row_ptr[(int64_t)h * args.cap + qb];
  const int e1 = args.row_ptr[(int64_t)h * args.cap + qb + 1];
  const int row_base = (int)((int64_t)h * args.N);

  if (threadIdx.x == 0) {
    tc::mbar_init(b_q, 1);
    for (int s = 0; s < kTcStages; ++s) {
      tc::mbar_init(b_kfull(s), 1);
      tc::mbar_init(b_vfull(s), 1);
      tc::mbar_init(b_kempty(s), 1);
      tc::mbar_init(b_vempty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(b_sfull(b), 1);
      tc::mbar_init(b_pfull(b), 128);
    }
    tc::mbar_init(b_ofull, 1);
    tc::mbar_init(b_drain, 1);
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto tS = [&](int b) { return tmem + 128u * (uint32_t)b; };   // two S / P buffers
  const uint32_t tO = tmem + 256;                                  // O accumulator
  const uint32_t limit = args.wait_limit;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_tmap(&tmQ);
      tc::prefetch_tmap(&tmK);
      tc::prefetch_tmap(&tmV);
      tc::mbar_expect_tx(b_q, kTcTileBytes);
      tc::tma_load_2d(sQ, &tmQ, 0, row_base + r0, b_q);
      tc::tma_load_2d(sQ + kTcTileBytes / 2, &tmQ, 64, row_base + r0, b_q);
      KeyTiles kt;
      kt.init(args.col, args.blocks, e0, e1);
      int nk = 0, nv = 0;   // K and V fills issued
      for (; kt.valid(); kt.next()) {
        const int s = nk % kTcStages;
        const uint32_t ph = (uint32_t)(nk / kTcStages) & 1u;
        if (!tc::mbar_wait(b_kempty(s), ph ^ 1u, abort, limit)) break;
        tc::mbar_expect_tx(b_kfull(s), kTcTileBytes);
        tc::tma_load_2d(sK(s), &tmK, 0, row_base + kt.row(), b_kfull(s));
        tc::tma_load_2d(sK(s) + kTcTileBytes / 2, &tmK, 64, row_base + kt.row(), b_kfull(s));
        ++nk;
        if (!tc::mbar_wait(b_vempty(s), ph ^ 1u, abort, limit)) break;
        tc::mbar_expect_tx(b_vfull(s), kTcTileBytes);
        tc::tma_load_2d(sV(s), &tmV, 0, row_base + kt.row(), b_vfull(s));
        tc::tma_load_2d(sV(s) + kTcTileBytes / 2, &tmV, 64, row_base + kt.row(), b_vfull(s));
        ++nv;
      }
      // drain: every fill issued lands before the CTA exits (at most one
      // outstanding fill per stage, so each parity wait is unambiguous)
      volatile int no_abort = 0;
      tc::mbar_wait(b_q, 0, &no_abort, limit);
      for (int k = max(0, nk - kTcStages); k < nk; ++k)
        tc::mbar_wait(b_kfull(k % kTcStages), (uint32_t)(k / kTcStages) & 1u, &no_abort, limit);
      for (int k = max(0, nv - kTcStages); k < nv; ++k)
        tc::mbar_wait(b_vfull(k % kTcStages), (uint32_t)(k / kTcStages) & 1u, &no_abort, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int nsteps = count_key_tiles(args.col, args.blocks, e0, e1);
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = tc::idesc_f16(128, 128, false, true);   // P (TMEM) x V, fp16
      bool ok = tc::mbar_wait(b_q, 0, abort, limit);
      const uint64_t dQ = tc::sw128_desc(sQ, 16, 1024);
      auto issue_s = [&](int n) -> bool {
        const int s = n % kTcStages;
        if (!tc::mbar_wait(b_kfull(s), (uint32_t)(n / kTcStages) & 1u, abort, limit)) return false;
        tc::tc_fence_after();
        const uint64_t dK = tc::sw128_desc(sK(s), 16, 1024);
        const uint32_t tSn = tS(n & 1);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * (kTcTileBytes / 2) + (uint32_t)(k & 3) * 32u;
          tc::mma_ss(tSn, tc::desc_adv(dQ, off), tc::desc_adv(dK, off), idS, k > 0);
        }
        tc::mma_commit(b_sfull(n & 1));
        tc::mma_commit(b_kempty(s));
        return true;
      };
      if (ok && nsteps > 0) ok = issue_s(0);
      for (int n = 0; ok && n < nsteps; ++n) {
        if (n + 1 < nsteps && !issue_s(n + 1)) break;
        const int s = n % kTcStages;
        if (!tc::mbar_wait(b_pfull(n & 1), (uint32_t)(n >> 1) & 1u, abort, limit)) break;
        if (!tc::mbar_wait(b_vfull(s), (uint32_t)(n / kTcStages) & 1u, abort, limit)) break;
        tc::tc_fence_after();
        const uint64_t dV = tc::sw128_desc(sV(s), kTcTileBytes / 2, 1024);
        const uint32_t tPn = tS(n & 1);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_ts(tO, tPn + 8u * k, tc::desc_adv(dV, 2048u * k), idO, (n > 0 || k > 0) ? 1u : 0u);
        tc::mma_commit(b_vempty(s));
        tc::mma_commit(b_ofull);
      }
      // drain: all issued MMAs complete before TMEM is released
      tc::mma_commit(b_drain);
      volatile int no_abort = 0;
      tc::mbar_wait(b_drain, 0, &no_abort, limit);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = 32 * q + lane;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const float sl2 = args.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    KeyTiles kt;
    kt.init(args.col, args.blocks, e0, e1);
    int n = 0;
    bool ok = true;
    for (; kt.valid(); kt.next(), ++n) {
      const int b = n & 1;
      // waits and tensor-memory accesses stay warp-uniform (tcgen05.ld/st are
      // warp-collective): a lane that gives up makes the whole warp give up
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_sfull(b), (uint32_t)(n >> 1) & 1u, abort, limit))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      uint32_t raw[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(tS(b) + lane_off + 32u * c, raw[c]);
      tc::tmem_ld_wait();
      const int kv = kt.keys();
      if (kv < 128) {   // a 64-key block: the upper half of the tile is padding
#pragma unroll
        for (int c = 2; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[c][e] = __float_as_uint(-INFINITY);
      }
      // row max with eight independent chains
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(raw[c][e]));
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      mx *= sl2;
      // lazy rescaling: only rows whose max grew by more than 2^8 move m_run,
      // which stays an integer, so every rescale is an exact power of two
      const bool grow = mx > m_run + 8.f;
      float alpha = 1.f;
      if (grow) {
        const float m_new = ceilf(mx);
        alpha = pow2_or_zero(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      if (n > 0 && __any_sync(0xffffffffu, grow)) {
        // O is rescaled once every earlier P V has landed (rows that did not
        // grow are multiplied by 1)
        if (!__all_sync(0xffffffffu, tc::mbar_wait(b_ofull, (uint32_t)(n - 1) & 1u, abort, limit))) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tc::tmem_ld32(tO + lane_off + 32u * c, ov);
          tc::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tc::tmem_st32(tO + lane_off + 32u * c, ov);
        }
      }
      float r8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) r8[e] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // P truncated to 11 significant bits: exactly the fp16 operand of the
          // product, and l sums the same values
          const float p0 = trunc11(tc::ex2(fmaf(__uint_as_float(raw[c][2 * e]), sl2, -m_run)));
          const float p1 = trunc11(tc::ex2(fmaf(__uint_as_float(raw[c][2 * e + 1]), sl2, -m_run)));
          pk[e] = pack_f16(p0, p1);
          r8[e & 7] += p0 + p1;
        }
        tc::tmem_st16(tS(b) + lane_off + 16u * c, pk);
      }
      l_run += ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
      tc::tmem_st_wait();
      tc::tc_fence_before();
      if (!(args.debug_stall && n == 0)) tc::mbar_arrive(b_pfull(b));
    }
    // epilogue
    const int nsteps = n;
    const int64_t orow_idx = (int64_t)h * args.N + r0 + row;
    if (__all_sync(0xffffffffu, ok && !*abort) && row < qrows) {   // row < qrows is warp-uniform
      float inv = 0.f;
      if (nsteps > 0) {
        // the single-phase drain barrier completes after the last P V
        if (__all_sync(0xffffffffu, tc::mbar_wait(b_drain, 0, abort, limit))) {
          tc::tc_fence_after();
          inv = l_run > 0.f ? pow2f(-v16_exponent(args.vmax[h])) / l_run : 0.f;
        } else {
          ok = false;
        }
      }
      if (ok) {
        __nv_bfloat16 *orow = args.o + orow_idx * 128;
        __nv_bfloat16 *rrow = args.o_res ? args.o_res + orow_idx * 128 : nullptr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          if (nsteps > 0) {
            tc::tmem_ld32(tO + lane_off + 32u * c, ov);
            tc::tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = 0u;
          }
#pragma unroll
          for (int v8 = 0; v8 < 4; ++v8) {
            uint4 u, r;
            uint32_t *up = &u.x, *rp = &r.x;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(ov[8 * v8 + 2 * e]) * inv;
              const float x1 = __uint_as_float(ov[8 * v8 + 2 * e + 1]) * inv;
              up[e] = pack_bf16(x0, x1);
              rp[e] = pack_bf16(x0 - bf16_lo(up[e]), x1 - bf16_hi(up[e]));
            }
            *reinterpret_cast<uint4 *>(orow + 32 * c + 8 * v8) = u;
            if (rrow) *reinterpret_cast<uint4 *>(rrow + 32 * c + 8 * v8) = r;
          }
        }
        args.lse[orow_idx] = (nsteps > 0 && l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace prism

namespace prism {

// ---------------------------------------------------------------------------
// Paired forward: one CTA per (256-token query block, head).  The block's two
// 128-row tiles A and B share every K/V tile (one TMA load serves both), and
// their softmax warp groups ping-pong with the MMA issuer:
//   S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) S_A(2) ...
// so one tile's softmax runs while the other tile's MMAs execute.
// TMEM: S_A | O_A | S_B | O_B.  S_g(n+1) is issued after PV_g(n), hence its
// completion also proves PV_g(n) complete, which is what the lazy O rescale
// of step n+1 needs.
constexpr int kTc2Stages = 2;
constexpr int kTc2SmemBytes = kTcTileBytes * (2 + 2 * kTc2Stages) + 256 + 1024;
constexpr int kTc2Threads = 320;   // producer, MMA, 2 x 4 softmax warps

__global__ void __launch_bounds__(kTc2Threads, 1) bsa_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                     const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const TcFwdArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t *sgen = smem_raw + (sbase - smem_u32(smem_raw));
  auto sQ = [&](int g) { return sbase + (uint32_t)g * kTcTileBytes; };
  auto sK = [&](int s) { return sbase + (uint32_t)(2 + 2 * s) * kTcTileBytes; };
  auto sV = [&](int s) { return sbase + (uint32_t)(3 + 2 * s) * kTcTileBytes; };
  const uint32_t sBar = sbase + (uint32_t)(2 + 2 * kTc2Stages) * kTcTileBytes;
  const uint32_t b_q = sBar;
  auto b_kfull = [&](int s) { return sBar + 8u * (1 + s); };
  auto b_vfull = [&](int s) { return sBar + 8u * (3 + s); };
  auto b_kempty = [&](int s) { return sBar + 8u * (5 + s); };
  auto b_vempty = [&](int s) { return sBar + 8u * (7 + s); };
  auto b_sfull = [&](int g) { return sBar + 8u * (9 + g); };
  auto b_pfull = [&](int g) { return sBar + 8u * (11 + g); };
  const uint32_t b_drain = sBar + 8u * 13;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sgen + (sBar - sbase) + 8 * 16);
  volatile int *abort = reinterpret_cast<volatile int *>(sgen + (sBar - sbase) + 8 * 16 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int m = blockIdx.x >> 1, t = blockIdx.x & 1;
  const int b0 = args.zone_blk_base[m];
  if (args.blocks[b0].size != 256) return;   // zones of 64/128 blocks run in the single-tile kernel
  const int qb = b0 + t;
  const int r0 = m * kZoneTokens + 256 * t;
  const int e0 = args.row_ptr[(int64_t)h * args.cap + qb];
  const int e1 = args.row_ptr[(int64_t)h * args.cap + qb + 1];
  const int row_base = (int)((int64_t)h * args.N);

  if (threadIdx.x == 0) {
    tc::mbar_init(b_q, 1);
    for (int s = 0; s < kTc2Stages; ++s) {
      tc::mbar_init(b_kfull(s), 1);
      tc::mbar_init(b_vfull(s), 1);
      tc::mbar_init(b_kempty(s), 1);
      tc::mbar_init(b_vempty(s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      tc::mbar_init(b_sfull(g), 1);
      tc::mbar_init(b_pfull(g), 128);
    }
    tc::mbar_init(b_drain, 1);
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto tS = [&](int g) { return tmem + 256u * (uint32_t)g; };
  auto tO = [&](int g) { return tmem + 256u * (uint32_t)g + 128u; };
  const uint32_t limit = args.wait_limit;

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tmap(&tmQ);
      tc::prefetch_tmap(&tmK);
      tc::prefetch_tmap(&tmV);
      tc::mbar_expect_tx(b_q, 2 * kTcTileBytes);
      for (int g = 0; g < 2; ++g) {
        tc::tma_load_2d(sQ(g), &tmQ, 0, row_base + r0 + 128 * g, b_q);
        tc::tma_load_2d(sQ(g) + kTcTileBytes / 2, &tmQ, 64, row_base + r0 + 128 * g, b_q);
      }
      KeyTiles kt;
      kt.init(args.col, args.blocks, e0, e1);
      int nk = 0, nv = 0;
      for (; kt.valid(); kt.next()) {
        const int s = nk % kTc2Stages;
        const uint32_t ph = (uint32_t)(nk / kTc2Stages) & 1u;
        if (!tc::mbar_wait(b_kempty(s), ph ^ 1u, abort, limit)) break;
        tc::mbar_expect_tx(b_kfull(s), kTcTileBytes);
        tc::tma_load_2d(sK(s), &tmK, 0, row_base + kt.row(), b_kfull(s));
        tc::tma_load_2d(sK(s) + kTcTileBytes / 2, &tmK, 64, row_base + kt.row(), b_kfull(s));
        ++nk;
        if (!tc::mbar_wait(b_vempty(s), ph ^ 1u, abort, limit)) break;
        tc::mbar_expect_tx(b_vfull(s), kTcTileBytes);
        tc::tma_load_2d(sV(s), &tmV, 0, row_base + kt.row(), b_vfull(s));
        tc::tma_load_2d(sV(s) + kTcTileBytes / 2, &tmV, 64, row_base + kt.row(), b_vfull(s));
        ++nv;
      }
      volatile int no_abort = 0;
      tc::mbar_wait(b_q, 0, &no_abort, limit);
      for (int k = max(0, nk - kTc2Stages); k < nk; ++k)
        tc::mbar_wait(b_kfull(k % kTc2Stages), (uint32_t)(k / kTc2Stages) & 1u, &no_abort, limit);
      for (int k = max(0, nv - kTc2Stages); k < nv; ++k)
        tc::mbar_wait(b_vfull(k % kTc2Stages), (uint32_t)(k / kTc2Stages) & 1u, &no_abort, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const int nsteps = count_key_tiles(args.col, args.blocks, e0, e1);
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = tc::idesc_f16(128, 128, false, true);   // P (TMEM) x V, fp16
      bool ok = tc::mbar_wait(b_q, 0, abort, limit);
      const uint64_t dQ[2] = {tc::sw128_desc(sQ(0), 16, 1024), tc::sw128_desc(sQ(1), 16, 1024)};
      auto issue_s = [&](int n, int g) {
        const uint64_t dK = tc::sw128_desc(sK(n % kTc2Stages), 16, 1024), dQg = dQ[g];
        const uint32_t tSg = tS(g);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * (kTcTileBytes / 2) + (uint32_t)(k & 3) * 32u;
          tc::mma_ss(tSg, tc::desc_adv(dQg, off), tc::desc_adv(dK, off), idS, k > 0);
        }
        tc::mma_commit(b_sfull(g));
      };
      auto issue_pv = [&](int n, int g) {
        const uint64_t dV = tc::sw128_desc(sV(n % kTc2Stages), kTcTileBytes / 2, 1024);
        const uint32_t tOg = tO(g), tPg = tS(g);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_ts(tOg, tPg + 8u * k, tc::desc_adv(dV, 2048u * k), idO, (n > 0 || k > 0) ? 1u : 0u);
      };
      auto wait_k = [&](int n) {
        return tc::mbar_wait(b_kfull(n % kTc2Stages), (uint32_t)(n / kTc2Stages) & 1u, abort, limit);
      };
      if (ok && nsteps > 0) {
        ok = wait_k(0);
        if (ok) {
          tc::tc_fence_after();
          issue_s(0, 0);
          issue_s(0, 1);
          tc::mma_commit(b_kempty(0));
        }
      }
      for (int n = 0; ok && n < nsteps; ++n) {
        const int s = n % kTc2Stages;
        for (int g = 0; g < 2 && ok; ++g) {
          if (!tc::mbar_wait(b_pfull(g), (uint32_t)n & 1u, abort, limit)) { ok = false; break; }
          if (g == 0 && !tc::mbar_wait(b_vfull(s), (uint32_t)(n / kTc2Stages) & 1u, abort, limit)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          issue_pv(n, g);
          if (g == 1) tc::mma_commit(b_vempty(s));
          if (n + 1 < nsteps) {
            if (g == 0 && !wait_k(n + 1)) { ok = false; break; }
            // S_g(n+1) overwrites the P columns PV_g(n) reads; the tensor pipe
            // executes one thread's MMAs in issue order, as the other kernels rely on
            tc::tc_fence_after();
            issue_s(n + 1, g);
            if (g == 1) tc::mma_commit(b_kempty((n + 1) % kTc2Stages));
          }
        }
      }
      tc::mma_commit(b_drain);
      volatile int no_abort = 0;
      tc::mbar_wait(b_drain, 0, &no_abort, limit);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int g = (warp - 2) >> 2;           // tile A (rows 0..127) or B (128..255)
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const float sl2 = args.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    KeyTiles kt;
    kt.init(args.col, args.blocks, e0, e1);
    int n = 0;
    bool ok = true;
    for (; kt.valid(); kt.next(), ++n) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(b_sfull(g), (uint32_t)n & 1u, abort, limit))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const int kv = kt.keys();
      // the whole S row in registers, one batched TMEM load
      uint32_t raw[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(tS(g) + lane_off + 32u * c, raw[c]);
      tc::tmem_ld_wait();
      if (kv < 128) {   // a 64-key block: the upper half of the tile is padding
#pragma unroll
        for (int c = 2; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[c][e] = __float_as_uint(-INFINITY);
      }
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(raw[c][e]));
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      mx *= sl2;
      const bool grow = mx > m_run + 8.f;   // integer m_run, exact power-of-two rescales
      float alpha = 1.f;
      if (grow) {
        const float m_new = ceilf(mx);
        alpha = pow2_or_zero(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      float r8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) r8[e] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // P truncated to 11 significant bits: exactly the fp16 operand of the
          // product, and l sums the same values
          const float p0 = trunc11(tc::ex2(fmaf(__uint_as_float(raw[c][2 * e]), sl2, -m_run)));
          const float p1 = trunc11(tc::ex2(fmaf(__uint_as_float(raw[c][2 * e + 1]), sl2, -m_run)));
          pk[e] = pack_f16(p0, p1);
          r8[e & 7] += p0 + p1;
        }
        tc::tmem_st16(tS(g) + lane_off + 16u * c, pk);
      }
      if (n > 0 && __any_sync(0xffffffffu, grow)) {
        // rare: rescale O (S_g(n) was issued after PV_g(n-1), so O has settled;
        // PV_g(n) waits for this step's P signal, issued below)
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tc::tmem_ld32(tO(g) + lane_off + 32u * c, ov);
          tc::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tc::tmem_st32(tO(g) + lane_off + 32u * c, ov);
        }
      }
      l_run += ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(b_pfull(g));
    }
    const int nsteps = n;
    const int64_t orow_idx = (int64_t)h * args.N + r0 + 128 * g + row;
    if (__all_sync(0xffffffffu, ok && !*abort)) {
      float inv = 0.f;
      if (nsteps > 0) {
        if (__all_sync(0xffffffffu, tc::mbar_wait(b_drain, 0, abort, limit))) {
          tc::tc_fence_after();
          inv = l_run > 0.f ? pow2f(-v16_exponent(args.vmax[h])) / l_run : 0.f;
        } else {
          ok = false;
        }
      }
      if (ok) {
        __nv_bfloat16 *orow = args.o + orow_idx * 128;
        __nv_bfloat16 *rrow = args.o_res ? args.o_res + orow_idx * 128 : nullptr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          if (nsteps > 0) {
            tc::tmem_ld32(tO(g) + lane_off + 32u * c, ov);
            tc::tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = 0u;
          }
#pragma unroll
          for (int v8 = 0; v8 < 4; ++v8) {
            uint4 u, r;
            uint32_t *up = &u.x, *rp = &r.x;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(ov[8 * v8 + 2 * e]) * inv;
              const float x1 = __uint_as_float(ov[8 * v8 + 2 * e + 1]) * inv;
              up[e] = pack_bf16(x0, x1);
              rp[e] = pack_bf16(x0 - bf16_lo(up[e]), x1 - bf16_hi(up[e]));
            }
            *reinterpret_cast<uint4 *>(orow + 32 * c + 8 * v8) = u;
            if (rrow) *reinterpret_cast<uint4 *>(rrow + 32 * c + 8 * v8) = r;
          }
        }
        args.lse[orow_idx] = (nsteps > 0 && l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace prism
