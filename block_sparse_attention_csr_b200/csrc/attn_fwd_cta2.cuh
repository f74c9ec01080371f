// Block-sparse forward of Radial Attention on sm_100a: one query tile per
// CTA, two CTAs per MMA (tcgen05 cta_group::2).
//
// Same computation as the other forward kernels (O = softmax(Q K^T * scale +
// M) V and LSE, Eq.2 of the Radial Attention review on jaehun.me, §3, over the
// active 128x128 tiles of §4.2).  A 2-CTA cluster owns the neighbouring query
// tiles (2p, 2p+1) of one head -- CTA rank r holds tile 2p + r -- and walks
// the ascending union of their CSR rows.  Every MMA is M = 256: the even CTA
// issues S = Q K^T and O += P V for both tiles at once.  Each CTA loads its
// own query tile, HALF of every key tile (keys 64 r .. 64 r + 63: B of S is
// split by N) and HALF of every value tile (columns 64 r .. 64 r + 63: B of
// PV is split by N), so a K / V tile crosses L2 -> SM once for two query
// tiles, as in the two-tile kernel.
//
// What the pair buys over one CTA with two query tiles: TMEM holds, per
// query tile, two S buffers and a separate P double buffer, so S(u+2) is
// issued as soon as the softmax has read S(u) -- the tensor core never waits
// for a P to be consumed before it can compute the next S.
//
// Warp roles per CTA (384 threads):
//   warp 0      TMA producer (this CTA's Q tile, K / V halves; 4-slot rings,
//               K two union columns ahead of V).  Loads count their bytes on
//               the even CTA's barriers, which the even CTA's producer arms.
//   warp 1      TMEM allocation for the pair (both CTAs); in the even CTA,
//               lane 0 issues every MMA and commits to the barriers of both
//               CTAs at once (multicast commit).
//   warps 2-3   idle.
//   warps 4-11  softmax of this CTA's tile, as in the one-tile kernel: warpgroup
//               wg takes key columns [64 wg, 64 wg + 64), one thread per row;
//               the two warps of a TMEM lane quarter exchange row maxima and
//               sums.  Each warp's release of an S buffer, a P buffer or the
//               O accumulator arrives on the even CTA's barrier (16 warps in
//               all).  A union column that holds nothing of this CTA's tile
//               is answered with P = 0.
//
// TMEM (512 columns, same addresses in both CTAs): S0 [0,128), S1 [128,256),
// O [256,384), P0 [384,448), P1 [448,512) (P as packed bf16 pairs).
//
// Shared memory per CTA: Q [128 x 128] + 4 K halves [64 x 128] + 4 V halves
// [128 x 64], bf16, 128-byte swizzle in 64-column boxes (160 KB).
//
// Only head_dim 128 is implemented (a V half of 64 columns is exactly one
// 128-byte swizzle atom).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "attn_fwd.cuh"
#include "attn_fwd_pair.cuh"
#include "mask_build.cuh"
#include "sm100_primitives.cuh"

namespace radial {

// Exponential pairs of the softmax evaluated on the FMA pipe (exp2_fma_x2)
// instead of the MUFU: bit e selects pair e of every 16-pair (32-key) chunk.
#ifndef RADIAL_EXP2_FMA_PAIRS
#define RADIAL_EXP2_FMA_PAIRS 0u
#endif
__host__ __device__ constexpr bool exp2_on_fma(int e) { return ((RADIAL_EXP2_FMA_PAIRS >> e) & 1u) != 0u; }

template <int D>
struct FwdCta2Cfg {
  static_assert(D == 128, "the CTA-pair forward is implemented for head_dim 128");
  static constexpr int Q_BYTES = 128 * D * 2;         // this CTA's query tile
  static constexpr int KH_BYTES = 64 * D * 2;         // 64 keys x D
  static constexpr int VH_BYTES = 128 * (D / 2) * 2;  // 128 keys x D/2
  static constexpr int NBOX = D / 64;
  static constexpr int K_SLOTS = 4;
  static constexpr int V_SLOTS = 4;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + K_SLOTS * KH_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + V_SLOTS * VH_BYTES;
  static constexpr int SMEM_X = SMEM_BAR + 512;  // float[2][128] row exchange
  static constexpr int SMEM_BYTES = SMEM_X + 1024 + 1024;
  static constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_P0 = 384;
};

struct Cta2Bars {
  // waited on in the even CTA only (armed by its producer / arrived on by
  // the softmax warps of both CTAs)
  uint64_t q_full, o_empty;
  uint64_t k_full[4], v_full[4];
  uint64_t s_empty[2], p_full[2];
  // signalled in both CTAs by the multicast commits of the MMA thread
  uint64_t q_empty, mma_done;
  uint64_t k_empty[4], v_empty[4];
  uint64_t s_full[2], pv_done[2];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Cta2Bars) <= 512, "barriers overlap the row exchange buffer");

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    radial_fwd_cta2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const FwdPairParams p) {
  using C = FwdCta2Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::SMEM_Q;
  uint8_t* sK = smem + C::SMEM_K;
  uint8_t* sV = smem + C::SMEM_V;
  Cta2Bars* bars = reinterpret_cast<Cta2Bars*>(smem + C::SMEM_BAR);
  volatile int* abort_flag = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool even = rank == 0;
  const int cl = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  // the even CTA's copy of a barrier, as a shared::cluster address
  auto at_even = [](uint64_t* b) { return mapa_shared(smem_u32(b), 0u); };

  if (threadIdx.x == 0) {
    bars->abort = 0;
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->o_empty, 16);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->mma_done, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_empty[i], 16);
      mbar_init(&bars->p_full[i], 16);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->pv_done[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&bars->tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before anything arrives on them
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t kc = 0, vc = 0, item_i = 0;
      bool ok = true;  // false once a wait gave up: issue nothing more
      auto load_k = [&](int kb, int h, int b) {
        const uint32_t sl = kc % C::K_SLOTS, use = kc / C::K_SLOTS;
        if (!ok || (use > 0 && !mbar_wait(&bars->k_empty[sl], (use - 1) & 1, abort_flag))) {
          ok = false;
          return;
        }
        // a half that lies wholly past the sequence is not loaded: its keys
        // are masked in every row, whatever the slot holds
        const bool odd_half = kb * 128 + 64 < p.n;
        if (even) mbar_arrive_expect_tx(&bars->k_full[sl], (odd_half ? 2 : 1) * C::KH_BYTES);
        if (even || odd_half) {
          const uint32_t full = at_even(&bars->k_full[sl]);
#pragma unroll
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d_pair(sK + sl * C::KH_BYTES + x * 8192, &tmK, full, x * 64, kb * 128 + 64 * rank, h, b);
        }
        ++kc;
      };
      auto load_v = [&](int kb, int h, int b) {
        const uint32_t sl = vc % C::V_SLOTS, use = vc / C::V_SLOTS;
        if (!ok || (use > 0 && !mbar_wait(&bars->v_empty[sl], (use - 1) & 1, abort_flag))) {
          ok = false;
          return;
        }
        if (even) mbar_arrive_expect_tx(&bars->v_full[sl], 2 * C::VH_BYTES);
        tma_load_4d_pair(sV + sl * C::VH_BYTES, &tmV, at_even(&bars->v_full[sl]), 64 * rank, kb * 128, h, b);
        ++vc;
      };
      for (int item = cl; ok && item < p.items; item += ncl, ++item_i) {
        const int bh = item / p.np;
        const int pr = p.pair_order ? RADIAL_CHECK_INDEX(p.pair_order[item - bh * p.np], 0, p.np) : item - bh * p.np;
        const int b = bh / p.heads, h = bh - b * p.heads;
        if (item_i > 0 && !mbar_wait(&bars->q_empty, (item_i - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        // an odd last pair has no second tile: the odd CTA loads nothing and
        // its softmax answers every column with P = 0
        const bool two = 2 * pr + 1 < p.nt;
        if (even) mbar_arrive_expect_tx(&bars->q_full, (two ? 2 : 1) * C::Q_BYTES);
        if (even || two) {
          const uint32_t qfull = at_even(&bars->q_full);
#pragma unroll
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d_pair(sQ + x * 16384, &tmQ, qfull, x * 64, (2 * pr + static_cast<int>(rank)) * 128, h, b);
        }
        const int u0 = p.pair_ptr[pr], u1 = p.pair_ptr[pr + 1];
        for (int u = u0; u < u0 + 2 && u < u1; ++u) load_k(RADIAL_CHECK_INDEX(p.pair_col[u], 0, p.nt), h, b);
        for (int u = u0; u < u1; ++u) {
          if (u + 2 < u1) load_k(RADIAL_CHECK_INDEX(p.pair_col[u + 2], 0, p.nt), h, b);
          load_v(RADIAL_CHECK_INDEX(p.pair_col[u], 0, p.nt), h, b);
        }
      }
      // Drain: the even CTA's barriers count both CTAs' copies, so once their
      // last phases completed, nothing is in flight into either CTA.
      if (even) {
        if (item_i > 0) mbar_wait_drain_cl(&bars->q_full, (item_i - 1) & 1);
        for (uint32_t x = (kc > C::K_SLOTS ? kc - C::K_SLOTS : 0); x < kc; ++x)
          mbar_wait_drain_cl(&bars->k_full[x % C::K_SLOTS], (x / C::K_SLOTS) & 1);
        for (uint32_t x = (vc > C::V_SLOTS ? vc - C::V_SLOTS : 0); x < vc; ++x)
          mbar_wait_drain_cl(&bars->v_full[x % C::V_SLOTS], (x / C::V_SLOTS) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (even && lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(256, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(256, D, false, true);
      constexpr uint64_t kKSlot = C::KH_BYTES >> 4, kVSlot = C::VH_BYTES >> 4;
      const uint64_t dQ = smem_desc(smem_u32(sQ), 16, 1024, kSwizzle128B);
      const uint64_t dK0 = smem_desc(smem_u32(sK), 16, 1024, kSwizzle128B);
      const uint64_t dV0 = smem_desc(smem_u32(sV), 16384, 1024, kSwizzle128B);
      uint32_t it = 0, item_i = 0;
      bool ok = true;  // false once a wait gave up: issue nothing more
      // S_g = Q K_g^T for both tiles into S buffer g & 1 (K slot g % K_SLOTS)
      auto issue_s = [&](uint32_t g, bool last) {
        const uint32_t ks = g % C::K_SLOTS, sb = g & 1;
        if (!ok || !mbar_wait_cl(&bars->k_full[ks], (g / C::K_SLOTS) & 1, abort_flag) ||
            (g >= 2 && !mbar_wait_cl(&bars->s_empty[sb], ((g >> 1) - 1) & 1, abort_flag))) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint64_t dk = dK0 + ks * kKSlot;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off_q = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          const uint64_t off_k = static_cast<uint64_t>(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4);
          mma_ss_pair(tmem + C::TM_S0 + sb * 128, dQ + off_q, dk + off_k, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit_pair(&bars->s_full[sb]);
        mma_commit_pair(&bars->k_empty[ks]);
        if (last) mma_commit_pair(&bars->q_empty);
      };
      // O += P_g V_g for both tiles (P buffer g & 1, V slot g % V_SLOTS)
      auto issue_pv = [&](uint32_t g, bool first) {
        const uint32_t vs = g % C::V_SLOTS, pb = g & 1;
        if (!ok || !mbar_wait_cl(&bars->p_full[pb], (g >> 1) & 1, abort_flag) ||
            !mbar_wait_cl(&bars->v_full[vs], (g / C::V_SLOTS) & 1, abort_flag) ||
            (first && item_i > 0 && !mbar_wait_cl(&bars->o_empty, (item_i - 1) & 1, abort_flag))) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint64_t dv = dV0 + vs * kVSlot;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_pair(tmem + C::TM_O, tmem + C::TM_P0 + pb * 64 + kk * 8, dv + kk * (2048 >> 4), idesc_o,
                      (!first || kk > 0) ? 1u : 0u);
        mma_commit_pair(&bars->pv_done[pb]);
        mma_commit_pair(&bars->v_empty[vs]);
      };
      for (int item = cl; ok && item < p.items; item += ncl, ++item_i) {
        const int bh = item / p.np;
        const int pr = p.pair_order ? RADIAL_CHECK_INDEX(p.pair_order[item - bh * p.np], 0, p.np) : item - bh * p.np;
        const uint32_t n = static_cast<uint32_t>(p.pair_ptr[pr + 1] - p.pair_ptr[pr]);
        if (!mbar_wait_cl(&bars->q_full, item_i & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(it, n == 1);
        if (n > 1) issue_s(it + 1, n == 2);
        for (uint32_t j = 0; j < n; ++j) {
          // S_{j+2} needs only that both softmaxes have read S_j: issue it first
          if (j + 2 < n) issue_s(it + j + 2, j + 3 == n);
          issue_pv(it + j, j == 0);
        }
        it += n;
      }
      // Every MMA must have completed before the pair's TMEM is released.
      mma_commit_pair(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int col0 = wg * 64;
    float* xchg = reinterpret_cast<float*>(smem + C::SMEM_X);
    volatile float* x_mine = xchg + wg * 128 + row;
    volatile float* x_peer = xchg + (1 - wg) * 128 + row;
    const int bar_id = 1 + quarter;
    auto exchange = [&](float v) {
      named_bar_sync(bar_id, 64);
      *x_mine = v;
      named_bar_sync(bar_id, 64);
      return *x_peer;
    };
    // ok turns false (warp-uniform, for good) once a wait gave up.  The warps
    // then keep walking the plan -- the two warps of a lane quarter must meet
    // at every exchange, whose named barrier has no time limit -- but arrive
    // on nothing and store nothing; every later wait returns at once.
    bool ok = true;
    auto checked = [&](bool waited) {
      ok = __all_sync(0xffffffffu, ok && waited);
      return ok;
    };
    // one arrival per warp on the even CTA's barrier, after this warp's TMEM
    // accesses have completed
    auto warp_arrive = [&](uint64_t* b) {
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive_cluster(at_even(b));
    };
    const uint8_t in_bit = rank ? kPairIn1 : kPairIn0;
    const uint8_t part_bit = rank ? kPairPart1 : kPairPart0;
    constexpr float kRescaleThreshold = 8.0f;  // log2 units
    FwdParams mp{};
    mp.f = p.f;
    mp.s = p.s;
    mp.n = p.n;
    mp.sink = p.sink;
    mp.hd = p.hd;
    mp.cd = p.cd;
    uint32_t it = 0;
    for (int item = cl; item < p.items; item += ncl) {
      const int bh = item / p.np;
      const int pr = p.pair_order ? RADIAL_CHECK_INDEX(p.pair_order[item - bh * p.np], 0, p.np) : item - bh * p.np;
      const int b = bh / p.heads, h = bh - b * p.heads;
      const int t = 2 * pr + static_cast<int>(rank);
      const int a = t * 128 + row;
      const bool valid = t < p.nt && a < p.n;
      const int qi = valid ? a / p.s : 0;
      const int qk = valid ? a - qi * p.s : 0;
      const int u0 = p.pair_ptr[pr];
      const uint32_t n = static_cast<uint32_t>(p.pair_ptr[pr + 1] - u0);
      float m = -INFINITY;  // running max of scaled logits, log2 domain
      float l = 0.f;        // this warp's part of the running sum
      bool started = false;  // a column of this tile has been processed
      uint8_t fl_next = p.pair_flag[u0];
      int kb_next = RADIAL_CHECK_INDEX(p.pair_col[u0], 0, p.nt);
      // S of the column being processed.  While a column's P is computed, the
      // next column's S (already in the other S buffer) is loaded into the
      // halves of r that P no longer needs, so the TMEM round trip of one
      // column hides behind the exponentials of the previous one.
      uint32_t r[64];
      bool preloaded = false;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t g = it + j, sb = g & 1;
        const uint8_t fl = fl_next;
        const int kb = kb_next;
        if (j + 1 < n) {
          fl_next = p.pair_flag[u0 + j + 1];
          kb_next = RADIAL_CHECK_INDEX(p.pair_col[u0 + j + 1], 0, p.nt);
        }
        const uint32_t tm_p = tmem + lane_addr + C::TM_P0 + sb * 64 + wg * 32;
        if (!(fl & in_bit)) {
          // the column belongs to the other tile only: S is not needed, P = 0
          checked(mbar_wait(&bars->s_full[sb], (g >> 1) & 1, abort_flag));
          tc_fence_after();
          warp_arrive(&bars->s_empty[sb]);
          if (g >= 2) {
            checked(mbar_wait(&bars->pv_done[sb], ((g >> 1) - 1) & 1, abort_flag));
            tc_fence_after();
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = 0u;
          tmem_st16(tm_p, w);
          tmem_st16(tm_p + 16, w);
          tmem_wait_st();
          warp_arrive(&bars->p_full[sb]);
          continue;
        }
        if (!preloaded) {
          checked(mbar_wait(&bars->s_full[sb], (g >> 1) & 1, abort_flag));
          tc_fence_after();
          const uint32_t tm_s = tmem + lane_addr + C::TM_S0 + sb * 128;
          tmem_ld32(tm_s + col0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(tm_s + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        }
        // the mask bits of a PARTIAL tile are computed while the load is in flight
        const bool part = (fl & part_bit) != 0;
        uint32_t mw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        uint32_t live = 3u;   // 32-key chunks with an allowed key in some lane of the warp
        uint32_t mixed = 0u;  // chunks that need the per-element select
        if (part) {
          mw[0] = mw[1] = mw[2] = mw[3] = 0u;
          if (valid) row_mask_bits(mp, qi, qk, kb * 128 + col0, mw);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (!__any_sync(0xffffffffu, mw[c] != 0u)) live &= ~(1u << c);
            else if (!__all_sync(0xffffffffu, mw[c] == 0xffffffffu)) mixed |= 1u << c;
          }
        }
        tmem_wait_ld();
        regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        // S buffer sb may now take S_{g+2}
        warp_arrive(&bars->s_empty[sb]);
        float acc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (mixed & (1u << c)) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (!((mw[c] >> e) & 1u)) r[32 * c + e] = 0xff800000u;  // -inf
          }
          if (live & (1u << c)) {
#pragma unroll
            for (int e = 32 * c; e < 32 * c + 32; e += 8)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                acc[k] = max3f(acc[k], __uint_as_float(r[e + k]), __uint_as_float(r[e + 4 + k]));
          }
        }
        const float mloc = max3f(acc[0], acc[1], fmaxf(acc[2], acc[3]));
        const float m_tile = fmaxf(mloc, exchange(mloc)) * p.scale_log2;
        // lazy rescaling: m moves only when the tile's maximum exceeds it by
        // more than the threshold (P stays below 2^8)
        const bool grow = m_tile > m + kRescaleThreshold;
        const bool resc = started && __any_sync(0xffffffffu, grow);
        const float factor = (grow && started) ? ex2_approx(m - m_tile) : 1.0f;
        if (grow) {
          l *= factor;
          m = m_tile;
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t negm = f2_pack(-m_use, -m_use);
        // P buffer sb was last read by PV_{g-2}
        if (g >= 2) {
          checked(mbar_wait(&bars->pv_done[sb], ((g >> 1) - 1) & 1, abort_flag));
          tc_fence_after();
        }
        // the next column's S is loaded into r as this column's P frees it
        const bool next_in = j + 1 < n && (fl_next & in_bit);
        const uint32_t sbn = (g + 1) & 1;
        const uint32_t tm_sn = tmem + lane_addr + C::TM_S0 + sbn * 128;
        uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t w[16];
          if (!(live & (1u << c))) {
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = 0u;
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int k2 = 32 * c + 2 * e;
              const uint64_t xs = f2_fma(f2_pack(__uint_as_float(r[k2]), __uint_as_float(r[k2 + 1])), sl2, negm);
              uint64_t pe;
              if (exp2_on_fma(e)) {
                pe = exp2_fma_x2(xs);
              } else {
                float x0, x1;
                f2_unpack(xs, x0, x1);
                pe = f2_pack(ex2_approx(x0), ex2_approx(x1));
              }
              acc2[e & 1] = f2_add(acc2[e & 1], pe);
              float q0, q1;
              f2_unpack(pe, q0, q1);
              w[e] = pack_bf16x2(q0, q1);
            }
          }
          // P (bf16 pairs) of keys [col0 + 32 c, +32) -> P columns (col0 + 32 c) / 2
          tmem_st16(tm_p + c * 16, w);
          if (next_in) {
            if (c == 0) {
              checked(mbar_wait(&bars->s_full[sbn], ((g + 1) >> 1) & 1, abort_flag));
              tc_fence_after();
            }
            tmem_ld32(tm_sn + col0 + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
          }
        }
        preloaded = next_in;
        const uint64_t s01 = f2_add(acc2[0], acc2[1]);
        float s0, s1;
        f2_unpack(s01, s0, s1);
        l += s0 + s1;
        if (resc) {
          // O holds every PV up to PV_{g-1} once that one completes; this warp
          // rescales its half of the output columns
          checked(mbar_wait(&bars->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag));
          tc_fence_after();
          const uint32_t tm_o = tmem + lane_addr + C::TM_O + wg * (D / 2);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t ro[32];
            tmem_ld32(tm_o + c * 32, ro);
            tmem_wait_ld();
            regs_ready(ro);
#pragma unroll
            for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * factor);
            tmem_st32(tm_o + c * 32, ro);
          }
        }
        tmem_wait_st();
        warp_arrive(&bars->p_full[sb]);
        started = true;
      }
      // -------------------------------------------------------- epilogue
      const uint32_t g_last = it + n - 1;
      checked(mbar_wait(&bars->pv_done[g_last & 1], (g_last >> 1) & 1, abort_flag));
      tc_fence_after();
      const float lt = l + exchange(l);
      const float inv_l = lt > 0.f ? 1.0f / lt : 0.f;
      __nv_bfloat16* orow = p.o + static_cast<int64_t>(b) * p.o_sb + static_cast<int64_t>(h) * p.o_sh +
                            static_cast<int64_t>(valid ? a : 0) * p.o_sn + wg * (D / 2);
      const uint32_t tm_o = tmem + lane_addr + C::TM_O + wg * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ro[32];
        tmem_ld32(tm_o + c * 32, ro);
        tmem_wait_ld();
        if (valid && ok) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(ro[2 * e]) * inv_l, __uint_as_float(ro[2 * e + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      warp_arrive(&bars->o_empty);
      if (wg == 0 && valid && ok) {
        const float lse = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.n + a] = lse;
      }
      it += n;
    }
  }

  // ------------------------------------------------------------ teardown
  // Neither CTA releases TMEM or exits while the other may still be in its
  // loop: the even CTA's MMAs read the odd CTA's shared memory and write its
  // TMEM, and the odd CTA's copies and arrivals land in the even CTA.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace radial
