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
// Warp roles (384 threads; at most 168 registers each, 127 used):
//   warp 0      TMA producer: Q0, Q1 once per item; K and V through
//               separate 3-slot / 2-slot rings, K one union column ahead of V.
//   warps 2-3   idle (keep the softmax warps on warpgroup boundaries).
//   warp 1      TMEM allocator, single-thread tcgen05.mma issuer.  Per union
//               column u and tile i: first O_i += P_i(u') V(u') for the tile's
//               pending column u' < u, then S_i(u) = Q_i K(u)^T.  The order
//               PV0, S0, PV1, S1 gives the softmax the other tile's two MMAs
//               (1024 tensor cycles) to turn S_i into P_i.
//   warps 4-11  softmax, both warpgroups on every S tile in turn (S0(u),
//               S1(u), S0(u+1), ...): warpgroup wg takes key columns
//               [64 wg, 64 wg + 64), one thread per query row; the two warps
//               on the same TMEM lane quarter exchange row maxima through
//               double-buffered shared memory, one named barrier per
//               exchange.  Lazy rescaling, packed fp32x2 math.  The MUFU
//               (16 exponentials per clock and SM) needs all of the 1024
//               cycles to exponentiate one 128x128 tile, so one warp per SMSP
//               and tile left it idle during every TMEM round trip; two warps
//               per SMSP on the same tile overlap those waits.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D);
// P_i (bf16 pairs) is written over S_i columns [0,64) once S_i has been read.
// The commit that signals S_i(u) also covers every earlier MMA of the issuing
// thread, so when a softmax warpgroup sees S_i(u), PV_i(u') has completed:
// P_i(u') is consumed and O_i is up to date for a rescale.  S_i(u+1) is
// issued after PV_i(u) in the same MMA stream and executes after it.
//
// Shared memory: Q0, Q1 + 3 K slots + 2 V slots, 128 x D bf16 each, 128-byte
// swizzle in 64-column boxes (224 KB at D = 128), then the barriers and the
// 2 KB row-exchange buffer: 227 KB, the per-block maximum.  The tiles need a
// 1024-byte aligned base; a launch whose shared memory base is off by more
// than the 768 bytes of slack does nothing and records kErrLayout.
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
  static constexpr int SMEM_X = SMEM_BAR + 256;  // float[2 slots][2 warpgroups][128 rows] row exchange
  // the tiles need a 1024-byte aligned base; the dynamic shared memory base
  // is aligned that way in practice, and the kernel checks that its
  // alignment pad fits this slack before it touches anything
  static constexpr int ALIGN_SLACK = 768;
  static constexpr int SMEM_BYTES = SMEM_X + 2048 + ALIGN_SLACK;
  static constexpr uint32_t TM_S = 0, TM_O = 256;
};

struct PairBars {
  uint64_t q_full, q_empty, mma_done;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PairBars) <= 256, "barriers overlap the row exchange buffer");
static_assert(FwdPairCfg<128>::K_SLOTS <= 3 && FwdPairCfg<128>::V_SLOTS <= 3, "ring barriers hold 3 slots");

template <int D>
__global__ void __launch_bounds__(384, 1)
    radial_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const FwdPairParams p) {
  using C = FwdPairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t align_pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (align_pad > static_cast<uint32_t>(C::ALIGN_SLACK)) {  // uniform over the grid: every thread returns
    if (threadIdx.x == 0) atomicExch(&g_device_error, kErrLayout);
    return;
  }
  uint8_t* smem = smem_raw + align_pad;
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
    for (int i = 0; i < C::V_SLOTS; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 256);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], 256);
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
        const uint32_t sl = vc % C::V_SLOTS, use = vc / C::V_SLOTS;
        if (use > 0) mbar_wait(&bars->v_empty[sl], (use - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->v_full[sl], C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_4d(sV + sl * C::TILE_BYTES + x * 16384, &tmV, &bars->v_full[sl], x * 64, kb * 128, h, b);
        ++vc;
      };
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.np;
        const int pr = p.pair_order ? RADIAL_CHECK_INDEX(p.pair_order[item - bh * p.np], 0, p.np) : item - bh * p.np;
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
        load_k(RADIAL_CHECK_INDEX(p.pair_col[u0], 0, p.nt), h, b);
        for (int u = u0; u < u1; ++u) {
          if (u + 1 < u1) load_k(RADIAL_CHECK_INDEX(p.pair_col[u + 1], 0, p.nt), h, b);
          load_v(RADIAL_CHECK_INDEX(p.pair_col[u], 0, p.nt), h, b);
        }
      }
      for (uint32_t x = (kc > C::K_SLOTS ? kc - C::K_SLOTS : 0); x < kc; ++x)
        mbar_wait_drain(&bars->k_full[x % C::K_SLOTS], (x / C::K_SLOTS) & 1);
      for (uint32_t x = (vc > C::V_SLOTS ? vc - C::V_SLOTS : 0); x < vc; ++x)
        mbar_wait_drain(&bars->v_full[x % C::V_SLOTS], (x / C::V_SLOTS) & 1);
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
        const int pr = p.pair_order ? RADIAL_CHECK_INDEX(p.pair_order[item - bh * p.np], 0, p.np) : item - bh * p.np;
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
          const uint32_t vs = vslot_count % C::V_SLOTS;
          mbar_wait(&bars->v_full[vs], (vslot_count / C::V_SLOTS) & 1, abort_flag);
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
          if (u > u0) mma_commit(&bars->v_empty[(vc - 1) % C::V_SLOTS]);  // V(u-1): its PVs are issued
          if (u + 1 == u1) mma_commit(&bars->q_empty);
          ++vc;  // V(u) is the producer's next V; PVs of column u refer to vc - 1
        }
        // flush the last column's PVs, release its V, publish O
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (pending[i]) issue_pv(i, vc - 1);
        mma_commit(&bars->v_empty[(vc - 1) % C::V_SLOTS]);
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
    // ------------------------------------------------------------ softmax
    // Both warpgroups work on every S tile: warpgroup wg owns its key
    // columns [64 wg, 64 wg + 64), warp (wg, quarter) the 32 rows of TMEM
    // lane quarter `quarter`.  The two warps sharing a quarter (same rows,
    // same SMSP) exchange partial row maxima -- and at the end row sums --
    // through shared memory, so both apply the same running maximum m.  Two
    // warps per SMSP keep the MUFU busy while one of them waits on TMEM.
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int col0 = wg * 64;
    // Exchange k (both warps of a quarter run the same sequence) uses slot
    // k & 1: xput writes this warp's value; xtake meets the peer at the
    // quarter's named barrier and reads the peer's value.  One barrier per
    // exchange: slot k & 1 is written again by exchange k + 2, after the
    // barrier of exchange k + 1, which the peer reaches only after its read
    // of exchange k.  (A single slot needs a second barrier before the write;
    // that version was 5-7 % slower.)
    volatile float* xchg = reinterpret_cast<volatile float*>(smem + C::SMEM_X);
    const int bar_id = 1 + quarter;
    uint32_t xk = 0;
    auto xput = [&](float v) { xchg[(xk & 1u) * 256 + wg * 128 + row] = v; };
    auto xtake = [&]() {
      named_bar_sync(bar_id, 64);
      const float v = xchg[(xk & 1u) * 256 + (1 - wg) * 128 + row];
      ++xk;
      return v;
    };
    constexpr float kRescaleThreshold = 8.0f;
    RowMaskGeom mp{};
    mp.f = p.f;
    mp.s = p.s;
    mp.n = p.n;
    mp.sink = p.sink;
    mp.hd = p.hd;
    mp.cd = p.cd;
    set_divisor(mp);
    uint32_t g[2] = {0u, 0u}, icnt[2] = {0u, 0u};
    for (int item = blockIdx.x; item < p.items; item += gridDim.x) {
      const int bh = item / p.np;
      const int pr = p.pair_order ? RADIAL_CHECK_INDEX(p.pair_order[item - bh * p.np], 0, p.np) : item - bh * p.np;
      const int b = bh / p.heads, h = bh - b * p.heads;
      const bool two = 2 * pr + 1 < p.nt;
      const int u0 = p.pair_ptr[pr], u1 = p.pair_ptr[pr + 1];
      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
      bool first[2] = {true, true};
      int qi[2], qk[2];
      bool valid[2];
#pragma unroll
      for (int ti = 0; ti < 2; ++ti) {
        const int a = (2 * pr + ti) * 128 + row;
        valid[ti] = a < p.n;
        qi[ti] = valid[ti] ? a / p.s : 0;
        qk[ti] = valid[ti] ? a - qi[ti] * p.s : 0;
      }
      uint8_t fl_next = p.pair_flag[u0];
      int kb_next = RADIAL_CHECK_INDEX(p.pair_col[u0], 0, p.nt);
      for (int u = u0; u < u1; ++u) {
        const uint8_t fl = fl_next;
        const int kb = kb_next;
        if (u + 1 < u1) {
          fl_next = p.pair_flag[u + 1];
          kb_next = RADIAL_CHECK_INDEX(p.pair_col[u + 1], 0, p.nt);
        }
#pragma unroll
        for (int ti = 0; ti < 2; ++ti) {
          if (!(fl & (ti == 0 ? kPairIn0 : kPairIn1))) continue;
          // The mask bits of a PARTIAL tile depend only on the key tile and the
          // row: they are formed before the wait for S, which they mostly fill
          // (PARTIAL tiles tend to wait longest on the MMA chain).
          const bool part = (fl & (ti == 0 ? kPairPart0 : kPairPart1)) != 0;
          uint32_t mw[2] = {0xffffffffu, 0xffffffffu};
          if (part) {
            const uint64_t m64 = valid[ti] ? row_mask64(mp, qi[ti], qk[ti], kb * 128 + col0) : 0ull;
            mw[0] = static_cast<uint32_t>(m64);
            mw[1] = static_cast<uint32_t>(m64 >> 32);
          }
          uint32_t live = 3u;  // 32-key chunks with an allowed key in some lane of the warp
          uint32_t mixed = 0u;  // chunks that need the per-element select
          if (part) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (!__any_sync(0xffffffffu, mw[c] != 0u)) live &= ~(1u << c);
              else if (!__all_sync(0xffffffffu, mw[c] == 0xffffffffu)) mixed |= 1u << c;
            }
          }
          mbar_wait(&bars->s_full[ti], g[ti] & 1, abort_flag);
          __syncwarp();
          tc_fence_after();
          const uint32_t tm_s = tmem + lane_addr + C::TM_S + ti * 128;
          uint32_t r[64];
          tmem_ld32(tm_s + col0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(tm_s + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_wait_ld();
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
                for (int k = 0; k < 4; ++k) acc[k] = max3f(acc[k], __uint_as_float(r[e + k]), __uint_as_float(r[e + 4 + k]));
            }
          }
          const float mloc = max3f(acc[0], acc[1], fmaxf(acc[2], acc[3]));
          // O_i holds every earlier PV (the S commit covers them); this warp
          // rescales its half of the output columns
          auto rescale_o = [&](float factor) {
            const uint32_t tm_o = tmem + lane_addr + C::TM_O + ti * 128 + wg * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              uint32_t ro[32];
              tmem_ld32(tm_o + c * 32, ro);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * factor);
              tmem_st32(tm_o + c * 32, ro);
            }
          };
          const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
          // P = exp2(S * scale * log2(e) - m) of this warp's 64 keys (bf16
          // pairs) -> TMEM columns (col0 + 32 c) / 2, over the consumed S;
          // returns the row's sum of them
          auto make_p = [&](float m_run) {
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
            const uint64_t negm = f2_pack(-m_use, -m_use);
            uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              uint32_t w[16];
              if (!(live & (1u << c))) {
#pragma unroll
                for (int e = 0; e < 16; ++e) w[e] = 0u;
                tmem_st16(tm_s + wg * 32 + c * 16, w);
                continue;
              }
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int k2 = 32 * c + 2 * e;
                const uint64_t xs = f2_fma(f2_pack(__uint_as_float(r[k2]), __uint_as_float(r[k2 + 1])), sl2, negm);
                float x0, x1;
                f2_unpack(xs, x0, x1);
                const uint64_t pe = f2_pack(ex2_approx(x0), ex2_approx(x1));
                acc2[e & 1] = f2_add(acc2[e & 1], pe);
                float p0, p1;
                f2_unpack(pe, p0, p1);
                w[e] = pack_bf16x2(p0, p1);
              }
              tmem_st16(tm_s + wg * 32 + c * 16, w);
            }
            const uint64_t s01 = f2_add(acc2[0], acc2[1]);
            float s0, s1;
            f2_unpack(s01, s0, s1);
            return s0 + s1;
          };
          // lazy rescaling: m moves only when the tile's row maximum exceeds it
          // by more than the threshold (P stays below 2^8)
          xput(mloc);
          const float m_tile = fmaxf(mloc, xtake()) * p.scale_log2;
          const bool grow = m_tile > m[ti] + kRescaleThreshold;
          const bool resc = !first[ti] && __any_sync(0xffffffffu, grow);
          const float factor = (grow && !first[ti]) ? ex2_approx(m[ti] - m_tile) : 1.0f;
          if (grow) {
            l[ti] *= factor;
            m[ti] = m_tile;
          }
          const float psum = make_p(m[ti]);
          if (resc) rescale_o(factor);
          l[ti] += psum;
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars->p_full[ti]);
          first[ti] = false;
          ++g[ti];
        }
      }
      // -------------------------------------------------------- epilogue
#pragma unroll
      for (int ti = 0; ti < 2; ++ti) {
        if (ti == 1 && !two) break;  // odd tail: this pair has one tile
        mbar_wait(&bars->o_full[ti], icnt[ti] & 1, abort_flag);
        __syncwarp();
        tc_fence_after();
        xput(l[ti]);
        const float lt = l[ti] + xtake();
        const float inv_l = lt > 0.f ? 1.0f / lt : 0.f;
        const int a = (2 * pr + ti) * 128 + row;
        __nv_bfloat16* orow = p.o + static_cast<int64_t>(b) * p.o_sb + static_cast<int64_t>(h) * p.o_sh +
                              static_cast<int64_t>(valid[ti] ? a : 0) * p.o_sn + wg * (D / 2);
        const uint32_t tm_o = tmem + lane_addr + C::TM_O + ti * 128 + wg * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t ro[32];
          tmem_ld32(tm_o + c * 32, ro);
          tmem_wait_ld();
          if (valid[ti]) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(ro[2 * e]) * inv_l, __uint_as_float(ro[2 * e + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->o_empty[ti]);
        if (wg == 0 && valid[ti]) {
          const float lse = lt > 0.f ? (m[ti] + log2f(lt)) * 0.69314718055994531f : -INFINITY;
          p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.n + a] = lse;
        }
        ++icnt[ti];
      }
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
