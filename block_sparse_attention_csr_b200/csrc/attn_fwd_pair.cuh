// Block-sparse forward of Radial Attention on sm_100a, two query tiles per CTA.
//
// Same computation as attn_fwd.cuh (O = softmax(Q K^T * scale + M) V and LSE,
// Eq.2 of the Radial Attention review, over the active 128x128 tiles of
// §4.2), but each CTA owns a pair of neighbouring 128-row query tiles
// (2p, 2p+1) of one head and walks the ascending union of their CSR rows, so
// every K / V tile brought into shared memory feeds two query tiles: half the
// L2 -> SM traffic per MMA of the one-tile kernel.  Neighbouring query tiles
// of the radial mask share most of their key tiles (same frames, windows
// shifted by 128 tokens); a key tile only one of them needs is computed for
// that tile alone.
//
// Warp roles (384 threads, 168 registers each):
//   warp 0      TMA producer: Q0, Q1 once per item; K and V through
//               separate 3-slot / 2-slot rings, K one union column ahead of V.
//   warps 2-3   idle (keep the softmax warps on warpgroup boundaries).
//   warp 1      TMEM allocator, single-thread tcgen05.mma issuer.  Per union
//               column u and tile i: first O_i += P_i(u') V(u') for the tile's
//               pending column u' < u, then S_i(u) = Q_i K(u)^T.  The order
//               PV0, S0, PV1, S1 gives each softmax warpgroup the other
//               tile's two MMAs (1024 tensor cycles) to turn S into P.
//   warps 4-7   softmax warpgroup of tile 0, warps 8-11 of tile 1: one thread
//               per query row; as in the one-tile kernel (lazy rescaling,
//               packed fp32x2 math).  To fit 168 registers only S columns
//               [0,64) stay in registers after the row max; columns [64,128)
//               are read from TMEM again when P is formed (P overwrites only
//               columns [0,64)).  Measured faster than re-reading all of S
//               with per-chunk mask modes.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D);
// P_i (bf16 pairs) is written over S_i columns [0,64) once S_i has been read.
// The commit that signals S_i(u) also covers every earlier MMA of the issuing
// thread, so when a softmax warpgroup sees S_i(u), PV_i(u') has completed:
// P_i(u') is consumed and O_i is up to date for a rescale.  S_i(u+1) is
// issued after PV_i(u) in the same MMA stream and executes after it.
//
// Shared memory: Q0, Q1 + 3 K slots + 2 V slots, 128 x D bf16 each, 128-byte
// swizzle in 64-column boxes (224 KB at D = 128).
//
// Work items are (batch*head, pair) in head-major order; within a head the
// pairs run longest-first when an order array is given (the default), else in
// ascending query position.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "attn_fwd.cuh"
#include "mask_build.cuh"
#include "sm100_primitives.cuh"

namespace radial {

struct FwdPairParams {
  const int32_t* pair_ptr;
  const int32_t* pair_col;
  const uint8_t* pair_flag;
  const int32_t* pair_order;
  int32_t np;  // pairs per head
  int32_t nt;  // query tiles per head
  int32_t f, s, n, sink;
  int32_t heads, items;  // items = batch * heads * np
  int64_t o_sb, o_sh, o_sn;
  __nv_bfloat16* o;
  float* lse;
  float scale_log2;
  const int32_t* hd;  // ablation-mask distance tables (nullptr: closed form)
  const int32_t* cd;
};

template <int D>
struct FwdPairCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NBOX = D / 64;
  static constexpr int K_SLOTS = 3;
  static constexpr int V_SLOTS = 2;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = 2 * TILE_BYTES;
  static constexpr int SMEM_V = SMEM_K + K_SLOTS * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + V_SLOTS * TILE_BYTES;
  static constexpr int SMEM_BYTES = SMEM_BAR + 512 + 1024;
  static constexpr uint32_t TM_S = 0, TM_O = 256;
};

struct PairBars {
  uint64_t q_full, q_empty, mma_done;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    radial_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const FwdPairParams p) {
  using C = FwdPairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::SMEM_Q;
  uint8_t* sK = smem + C::SMEM_K;
  uint8_t* sV = smem + C::SMEM_V;
  PairBars* bars = reinterpret_cast<PairBars*>(smem + C::SMEM_BAR);
  volatile int* abort_flag = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    bars->abort = 0;
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->mma_done, 1);
    for (int i = 0; i < C::K_SLOTS; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], 128);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t kc = 0, vc = 0, item_i = 0;
      auto load_k = [&](int kb, int h, int b) {
        const uint32_t sl = kc % C::K_SLOTS, use = kc / C::K_SLOTS;
        if (use > 0) mbar_wait(&bars->k_empty[sl], (use - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->k_full[sl], C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_4d(sK + sl * C::TILE_BYTES + x * 16384, &tmK, &bars->k_full[sl], x * 64, kb * 128, h, b);
        ++kc;
      };
      auto load_v = [&](int kb, int h, int b) {
        const uint32_t sl = vc & 1, use = vc >> 1;
        if (use > 0) mbar_wait(&bars->v_empty[sl], (use - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->v_full[sl], C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_4d(sV + sl * C::TILE_BYTES + x * 16384, &tmV, &bars->v_full[sl], x * 64, kb * 128, h, b);
        ++vc;
      };
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.np;
        const int pr = p.pair_order ? p.pair_order[item - bh * p.np] : item - bh * p.np;
        const int b = bh / p.heads, h = bh - b * p.heads;
        const bool two = 2 * pr + 1 < p.nt;
        if (item_i > 0) mbar_wait(&bars->q_empty, (item_i - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->q_full, (two ? 2 : 1) * C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x) {
          tma_load_4d(sQ + x * 16384, &tmQ, &bars->q_full, x * 64, (2 * pr) * 128, h, b);
          if (two) tma_load_4d(sQ + C::TILE_BYTES + x * 16384, &tmQ, &bars->q_full, x * 64, (2 * pr + 1) * 128, h, b);
        }
        const int u0 = p.pair_ptr[pr], u1 = p.pair_ptr[pr + 1];
        load_k(p.pair_col[u0], h, b);
        for (int u = u0; u < u1; ++u) {
          if (u + 1 < u1) load_k(p.pair_col[u + 1], h, b);
          load_v(p.pair_col[u], h, b);
        }
      }
      for (uint32_t x = (kc > C::K_SLOTS ? kc - C::K_SLOTS : 0); x < kc; ++x)
        mbar_wait_drain(&bars->k_full[x % C::K_SLOTS], (x / C::K_SLOTS) & 1);
      for (uint32_t x = (vc > 2 ? vc - 2 : 0); x < vc; ++x) mbar_wait_drain(&bars->v_full[x & 1], (x >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The issuing thread is the tensor pipe's only feeder: every instruction
    // between two tcgen05.mma delays the pipe.  All shared-memory descriptors
    // are therefore built once; a slot or K-step is a compile-time offset
    // added to the start-address field (addresses stay below 256 KB, so the
    // 14-bit field never carries).
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      constexpr uint64_t kSlot = C::TILE_BYTES >> 4;  // one tile, in descriptor units
      const uint64_t dq0 = smem_desc(smem_u32(sQ), 16, 1024, kSwizzle128B);
      const uint64_t dk0 = smem_desc(smem_u32(sK), 16, 1024, kSwizzle128B);
      const uint64_t dv0 = smem_desc(smem_u32(sV), 16384, 1024, kSwizzle128B);
      const uint32_t tS = tmem + C::TM_S, tO = tmem + C::TM_O;
      uint32_t kc = 0, vc = 0, item_i = 0;
      uint32_t g[2] = {0u, 0u};       // S tiles issued per query tile (all items)
      uint32_t icnt[2] = {0u, 0u};    // items completed per query tile
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.np;
        const int pr = p.pair_order ? p.pair_order[item - bh * p.np] : item - bh * p.np;
        const int u0 = p.pair_ptr[pr], u1 = p.pair_ptr[pr + 1];
        mbar_wait(&bars->q_full, item_i & 1, abort_flag);
        tc_fence_after();
        bool pending[2] = {false, false};   // a PV waits for the previous column's V
        uint32_t pend_g[2] = {0u, 0u};
        bool first_pv[2] = {true, true};
        bool used[2] = {false, false};
        auto issue_pv = [&](int i, uint32_t vslot_count) {
          const uint32_t gi = pend_g[i];
          mbar_wait(&bars->p_full[i], gi & 1, abort_flag);
          const uint32_t vs = vslot_count & 1;
          mbar_wait(&bars->v_full[vs], (vslot_count >> 1) & 1, abort_flag);
          if (first_pv[i] && icnt[i] > 0) mbar_wait(&bars->o_empty[i], (icnt[i] - 1) & 1, abort_flag);
          tc_fence_after();
          const uint64_t dv = dv0 + vs * kSlot;
          const uint32_t tPi = tS + i * 128, tOi = tO + i * 128;
          mma_ts(tOi, tPi, dv, idesc_o, first_pv[i] ? 0u : 1u);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk) mma_ts(tOi, tPi + kk * 8, dv + kk * (2048 >> 4), idesc_o, 1u);
          first_pv[i] = false;
          pending[i] = false;
        };
        uint8_t fl_next = p.pair_flag[u0];
        for (int u = u0; u < u1; ++u) {
          const uint8_t fl = fl_next;
          if (u + 1 < u1) fl_next = p.pair_flag[u + 1];
          const uint32_t ks = kc % C::K_SLOTS;
          mbar_wait(&bars->k_full[ks], (kc / C::K_SLOTS) & 1, abort_flag);
          tc_fence_after();
          const uint64_t dk = dk0 + ks * kSlot;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (pending[i]) issue_pv(i, vc - 1);  // V of the previous column
            if (fl & (i == 0 ? kPairIn0 : kPairIn1)) {
              const uint64_t dq = dq0 + i * kSlot;
              const uint32_t tSi = tS + i * 128;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                constexpr uint64_t z = 0;
                const uint64_t off = z + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                mma_ss(tSi, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
              }
              mma_commit(&bars->s_full[i]);
              pending[i] = true;
              pend_g[i] = g[i];
              used[i] = true;
              ++g[i];
            }
          }
          mma_commit(&bars->k_empty[ks]);  // K(u) read by the S MMAs above
          ++kc;
          if (u > u0) mma_commit(&bars->v_empty[(vc - 1) & 1]);  // V(u-1): its PVs are issued
          if (u + 1 == u1) mma_commit(&bars->q_empty);
          ++vc;  // V(u) is the producer's next V; PVs of column u refer to vc - 1
        }
        // flush the last column's PVs, release its V, publish O
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (pending[i]) issue_pv(i, vc - 1);
        mma_commit(&bars->v_empty[(vc - 1) & 1]);
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (used[i]) {
            mma_commit(&bars->o_full[i]);
            ++icnt[i];
          }
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax WGs
    const int ti = (warp - 4) >> 2;            // which query tile of the pair
    const int quarter = warp & 3;              // TMEM lane quarter
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tm_s = tmem + lane_addr + C::TM_S + ti * 128;
    const uint32_t tm_o = tmem + lane_addr + C::TM_O + ti * 128;
    const uint8_t in_bit = ti == 0 ? kPairIn0 : kPairIn1;
    const uint8_t part_bit = ti == 0 ? kPairPart0 : kPairPart1;
    constexpr float kRescaleThreshold = 8.0f;
    FwdParams mp{};
    mp.f = p.f;
    mp.s = p.s;
    mp.n = p.n;
    mp.sink = p.sink;
    mp.hd = p.hd;
    mp.cd = p.cd;
    uint32_t g = 0, icnt = 0;
    for (int item = blockIdx.x; item < p.items; item += gridDim.x) {
      const int bh = item / p.np;
      const int pr = p.pair_order ? p.pair_order[item - bh * p.np] : item - bh * p.np;
      const int t = 2 * pr + ti;
      if (t >= p.nt) continue;  // odd tail: this pair has one tile
      const int b = bh / p.heads, h = bh - b * p.heads;
      const int a = t * 128 + row;
      const bool valid = a < p.n;
      const int qi = valid ? a / p.s : 0;
      const int qk = valid ? a - qi * p.s : 0;
      const int u0 = p.pair_ptr[pr], u1 = p.pair_ptr[pr + 1];
      float m = -INFINITY, l = 0.f;
      bool first = true;
      uint8_t fl_next = p.pair_flag[u0];
      int kb_next = p.pair_col[u0];
      for (int u = u0; u < u1; ++u) {
        const uint8_t fl = fl_next;
        const int kb = kb_next;
        if (u + 1 < u1) {
          fl_next = p.pair_flag[u + 1];
          kb_next = p.pair_col[u + 1];
        }
        if (!(fl & in_bit)) continue;
        mbar_wait(&bars->s_full[ti], g & 1, abort_flag);
        __syncwarp();
        tc_fence_after();
        // pass 1: row max over all 128 columns; keep columns [0,64)
        uint32_t mw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        const bool part = (fl & part_bit) != 0;
        if (part) {
          mw[0] = mw[1] = mw[2] = mw[3] = 0u;
          if (valid) row_mask_bits(mp, qi, qk, kb * 128, mw);
        }
        float sv[64];
        float acc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        // two TMEM round trips: chunks {0,1} (kept) then {2,3} (max only)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[64];
          tmem_ld32(tm_s + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(tm_s + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_wait_ld();
          float x[64];
          if (part) {
#pragma unroll
            for (int e = 0; e < 64; ++e)
              x[e] = ((mw[2 * half + (e >> 5)] >> (e & 31)) & 1u) ? __uint_as_float(r[e]) : -INFINITY;
          } else {
#pragma unroll
            for (int e = 0; e < 64; ++e) x[e] = __uint_as_float(r[e]);
          }
#pragma unroll
          for (int e = 0; e < 64; e += 8)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = max3f(acc[k], x[e + k], x[e + 4 + k]);
          if (half == 0) {
#pragma unroll
            for (int e = 0; e < 64; ++e) sv[e] = x[e];
          }
        }
        const float m_tile = max3f(acc[0], acc[1], fmaxf(acc[2], acc[3])) * p.scale_log2;
        const bool grow = m_tile > m + kRescaleThreshold;
        if (!first) {
          if (__any_sync(0xffffffffu, grow)) {
            // O_i already holds every earlier PV (covered by the S commit).
            const float factor = grow ? ex2_approx(m - m_tile) : 1.0f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tmem_ld32(tm_o + c * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * factor);
              tmem_st32(tm_o + c * 32, r);
            }
            if (grow) {
              l *= factor;
              m = m_tile;
            }
          }
        } else if (grow) {
          m = m_tile;
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t negm = f2_pack(-m_use, -m_use);
        uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
        // P from 32 logits x -> 16 packed bf16 pairs into TMEM columns [16 c, 16 c + 16)
        auto make_p = [&](const float (&x)[32], int c) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t xs = f2_fma(f2_pack(x[2 * e], x[2 * e + 1]), sl2, negm);
            uint64_t pe;
            if (use_poly_exp(e)) {
              pe = exp2_poly_x2(xs);
            } else {
              float x0, x1;
              f2_unpack(xs, x0, x1);
              pe = f2_pack(ex2_approx(x0), ex2_approx(x1));
            }
            acc2[e & 3] = f2_add(acc2[e & 3], pe);
            float p0, p1;
            f2_unpack(pe, p0, p1);
            w[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tm_s + c * 16, w);
        };
        {
          float x0[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x0[e] = sv[e];
          make_p(x0, 0);
        }
        // re-read chunk 2 while chunk 1 is turned into P (P only overwrites columns [0,64))
        uint32_t r2[32], r3[32];
        tmem_ld32(tm_s + 64, r2);
        {
          float x1[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x1[e] = sv[32 + e];
          make_p(x1, 1);
        }
        tmem_ld32(tm_s + 96, r3);
        tmem_wait_ld();
#pragma unroll
        for (int c = 2; c < 4; ++c) {
          const uint32_t (&r)[32] = c == 2 ? r2 : r3;
          float x[32];
          if (part) {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = ((mw[c] >> e) & 1u) ? __uint_as_float(r[e]) : -INFINITY;
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(r[e]);
          }
          make_p(x, c);
        }
        const uint64_t s01 = f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3]));
        float s0, s1;
        f2_unpack(s01, s0, s1);
        l += s0 + s1;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[ti]);
        first = false;
        ++g;
      }
      // -------------------------------------------------------- epilogue
      mbar_wait(&bars->o_full[ti], icnt & 1, abort_flag);
      __syncwarp();
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* orow = p.o + static_cast<int64_t>(b) * p.o_sb + static_cast<int64_t>(h) * p.o_sh +
                            static_cast<int64_t>(valid ? a : 0) * p.o_sn;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tm_o + c * 32, r);
        tmem_wait_ld();
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_empty[ti]);
      if (valid) {
        const float lse = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.n + a] = lse;
      }
      ++icnt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace radial
