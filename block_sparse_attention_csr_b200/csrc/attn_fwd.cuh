// Block-sparse forward of Radial Attention on sm_100a.
//
// Computes O = softmax(Q K^T * scale + M) V and LSE per query row (the
// sparse-attention equation Eq.2 of the Radial Attention review, jaehun.me
// §3) over the active 128x128 tiles of the mask's CSR only (§4.2: the method
// runs block-wise on 128x128 token blocks).  Online softmax over the tiles of
// a row in the FlashAttention manner; the mask's element-level pattern is
// applied only on PARTIAL tiles.
//
// One persistent CTA per SM walks work items (batch*head, 128-row query tile)
// in a head-major order, longest rows first inside each head (row work varies
// with the temporal band).
//
// Warp roles (384 threads):
//   warp 0      TMA producer: the Q tile once per item, K and V tiles through
//               separate three-slot rings (K runs ahead: S needs it first).
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer.  S_j =
//               Q K_j^T goes into one of two TMEM S buffers; S_{j+2} is issued
//               as soon as the softmax has read S_j out of TMEM -- before P_j
//               exists -- so the tensor core never waits for the softmax to
//               hand back an S buffer.  O += P_j V_j follows when P_j is ready
//               (P in its own double buffer, read from TMEM as the A operand).
//   warps 2-3   idle (keep the softmax warps on warpgroup boundaries).
//   warps 4-11  softmax: warpgroup wg takes key columns [64 wg, 64 wg + 64)
//               of every S tile, one thread per query row (TMEM lane).  The
//               two warps on the same lane quarter exchange row maxima (and at
//               the end row sums) through shared memory.  PARTIAL tiles are
//               masked per element, with warp-uniform skipping of fully masked
//               or fully allowed 32-key chunks.  Running max in the log2
//               domain with lazy rescaling (O is rescaled in TMEM only when
//               the max grows by more than 2^8); at the end of the row O is
//               normalised and written (bf16) with LSE (fp32, natural log).
//
// TMEM (512 columns x 128 lanes): S0 [0,128), S1 [128,256), O [256,256+D),
// P0 [384,448), P1 [448,512) (P as packed bf16 pairs).
//
// Shared memory: Q [128 x D] + 3 K slots + 3 V slots [128 x D], bf16, written
// by TMA with the 128-byte swizzle in boxes of 64 columns.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mask_build.cuh"
#include "sm100_primitives.cuh"

namespace radial {

struct FwdParams {
  // 128-token tile plan of the mask (CSR over query tiles)
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const uint8_t* kind;
  const int32_t* order;  // query tiles, longest row first (nullptr: ascending)
  int32_t nt;            // query tiles per head
  // mask geometry for PARTIAL tiles
  int32_t f, s, n, sink;
  // tensors
  int32_t heads;
  int32_t items;  // batch * heads * nt
  int64_t o_sb, o_sh, o_sn;
  __nv_bfloat16* o;
  float* lse;
  float scale_log2;  // softmax scale * log2(e)
  // ablation-mask distance tables (nullptr: the method's closed form)
  const int32_t* hd;
  const int32_t* cd;
};

template <int D>
struct FwdCfg {
  static constexpr int K_SLOTS = 3;
  static constexpr int V_SLOTS = 3;
  static constexpr int TILE_BYTES = 128 * D * 2;  // one 128 x D bf16 tile
  static constexpr int NBOX = D / 64;             // 64-column swizzle boxes per tile
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = TILE_BYTES;
  static constexpr int SMEM_V = SMEM_K + K_SLOTS * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + V_SLOTS * TILE_BYTES;
  static constexpr int SMEM_X = SMEM_BAR + 256;  // float[2][128] row exchange
  static constexpr int SMEM_BYTES = SMEM_X + 1024 + 1024;  // + alignment slack
  static constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_P0 = 384;
  static constexpr uint32_t TM_COLS = 512;
};

// Barrier slots (uint64 each) inside the barrier area.
struct FwdBars {
  uint64_t q_full, q_empty, o_empty, mma_done;
  uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2];
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FwdBars) <= 256, "barriers overlap the row exchange buffer");

__device__ __forceinline__ void set_bits(uint32_t (&mw)[4], int lo, int hi) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int wlo = max(lo, 32 * w), whi = min(hi, 32 * w + 31);
    if (wlo <= whi) {
      const uint32_t nbits = static_cast<uint32_t>(whi - wlo + 1);
      const uint32_t bits = (nbits == 32u) ? 0xffffffffu : (((1u << nbits) - 1u) << (wlo - 32 * w));
      mw[w] |= bits;
    }
  }
}

// floor(x / s) for 0 <= x < 2^30 without an integer division: a float
// estimate from the reciprocal, then an exact correction of at most one step.
__device__ __forceinline__ int div_by(int x, int s) {
  int q = __float2int_rz(static_cast<float>(x) * __frcp_rn(static_cast<float>(s)));
  q += (q + 1) * s <= x;
  q -= q * s > x;
  return q;
}

// Allowed key columns (relative to b0, 128 wide) of query token a = i*s + k.
__device__ __forceinline__ void row_mask_bits(const FwdParams& p, int i, int k, int b0,
                                              uint32_t (&mw)[4]) {
  mw[0] = mw[1] = mw[2] = mw[3] = 0u;
  const int bend = min(b0 + 128, p.n);  // exclusive
  for (int j = div_by(b0, p.s); j * p.s < bend; ++j) {
    const int seg_lo = max(b0, j * p.s) - b0;
    const int seg_hi = min(bend, (j + 1) * p.s) - 1 - b0;
    int lo, hi;
    if (p.sink && j == 0) {
      lo = seg_lo;
      hi = seg_hi;
    } else {
      const int d = i > j ? i - j : j - i;
      const int h = half_width_of(p.hd, p.s, d);
      const int center = j * p.s + k - b0;
      if (h >= 0) {
        lo = max(seg_lo, center - h);
        hi = min(seg_hi, center + h);
      } else {
        const long long period = period_of(p.cd, p.s, d);
        if (d % period != 0) continue;
        lo = max(seg_lo, center);
        hi = min(seg_hi, center);
      }
    }
    if (lo <= hi) set_bits(mw, lo, hi);
  }
}

// Warp-uniform handling of one 32-column chunk of a PARTIAL tile: 0 = every
// lane of the warp allows all 32 columns (use S as is), 2 = every lane masks
// all of them (no TMEM read, no select, no exponential: P = 0), 1 = mixed
// (per-element select).  Two bits per chunk.
__device__ __forceinline__ uint32_t chunk_modes(const uint32_t (&mw)[4]) {
  uint32_t modes = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const bool all_ok = __all_sync(0xffffffffu, mw[c] == 0xffffffffu);
    const bool none = __all_sync(0xffffffffu, mw[c] == 0u);
    modes |= (all_ok ? 0u : (none ? 2u : 1u)) << (2 * c);
  }
  return modes;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    radial_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::SMEM_Q;
  uint8_t* sK = smem + C::SMEM_K;
  uint8_t* sV = smem + C::SMEM_V;
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::SMEM_BAR);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    bars->abort = 0;
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->o_empty, 256);
    mbar_init(&bars->mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_empty[b], 256);
      mbar_init(&bars->p_full[b], 256);
      mbar_init(&bars->pv_done[b], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TM_COLS);
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
        const int bh = item / p.nt;
        const int t = p.order ? RADIAL_CHECK_INDEX(p.order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
        const int b = bh / p.heads, h = bh - b * p.heads;
        if (item_i > 0) mbar_wait(&bars->q_empty, (item_i - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->q_full, C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_4d(sQ + x * 16384, &tmQ, &bars->q_full, x * 64, t * 128, h, b);
        const int p0 = p.row_ptr[t], p1 = p.row_ptr[t + 1];
        // K runs two columns ahead of V (S_{j+2} is issued before PV_j)
        for (int q = p0; q < p0 + 2 && q < p1; ++q) load_k(RADIAL_CHECK_INDEX(p.col_idx[q], 0, p.nt), h, b);
        for (int q = p0; q < p1; ++q) {
          if (q + 2 < p1) load_k(RADIAL_CHECK_INDEX(p.col_idx[q + 2], 0, p.nt), h, b);
          load_v(RADIAL_CHECK_INDEX(p.col_idx[q], 0, p.nt), h, b);
        }
      }
      // Drain: every slot's last fill must have landed before the CTA exits.
      for (uint32_t x = (kc > C::K_SLOTS ? kc - C::K_SLOTS : 0); x < kc; ++x)
        mbar_wait_drain(&bars->k_full[x % C::K_SLOTS], (x / C::K_SLOTS) & 1);
      for (uint32_t x = (vc > C::V_SLOTS ? vc - C::V_SLOTS : 0); x < vc; ++x)
        mbar_wait_drain(&bars->v_full[x % C::V_SLOTS], (x / C::V_SLOTS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Descriptors are built once; slots and K-steps are start-address offsets
    // (the issuing thread must spend almost nothing between two MMAs).
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      constexpr uint64_t kTile = C::TILE_BYTES >> 4;
      const uint64_t dQ = smem_desc(smem_u32(sQ), 16, 1024, kSwizzle128B);
      const uint64_t dK0 = smem_desc(smem_u32(sK), 16, 1024, kSwizzle128B);
      const uint64_t dV0 = smem_desc(smem_u32(sV), 16384, 1024, kSwizzle128B);
      uint32_t it = 0, item_i = 0;
      // S_g = Q K_g^T into S buffer g & 1 (K slot g % 3)
      auto issue_s = [&](uint32_t g, bool last) {
        const uint32_t ks = g % C::K_SLOTS, sb = g & 1;
        mbar_wait(&bars->k_full[ks], (g / C::K_SLOTS) & 1, abort_flag);
        if (g >= 2) mbar_wait(&bars->s_empty[sb], ((g >> 1) - 1) & 1, abort_flag);
        tc_fence_after();
        const uint64_t dk = dK0 + ks * kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          mma_ss(tmem + C::TM_S0 + sb * 128, dQ + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[sb]);
        mma_commit(&bars->k_empty[ks]);
        if (last) mma_commit(&bars->q_empty);
      };
      // O += P_g V_g (P buffer g & 1, V slot g % 3); first = first column of the item
      auto issue_pv = [&](uint32_t g, bool first) {
        const uint32_t vs = g % C::V_SLOTS, pb = g & 1;
        mbar_wait(&bars->p_full[pb], (g >> 1) & 1, abort_flag);
        mbar_wait(&bars->v_full[vs], (g / C::V_SLOTS) & 1, abort_flag);
        if (first && item_i > 0) mbar_wait(&bars->o_empty, (item_i - 1) & 1, abort_flag);
        tc_fence_after();
        const uint64_t dv = dV0 + vs * kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + C::TM_O, tmem + C::TM_P0 + pb * 64 + kk * 8, dv + kk * (2048 >> 4), idesc_o,
                 (!first || kk > 0) ? 1u : 0u);
        mma_commit(&bars->pv_done[pb]);
        mma_commit(&bars->v_empty[vs]);
      };
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.nt;
        const int t = p.order ? RADIAL_CHECK_INDEX(p.order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
        const uint32_t n = static_cast<uint32_t>(p.row_ptr[t + 1] - p.row_ptr[t]);
        mbar_wait(&bars->q_full, item_i & 1, abort_flag);
        tc_fence_after();
        issue_s(it, n == 1);
        if (n > 1) issue_s(it + 1, n == 2);
        for (uint32_t j = 0; j < n; ++j) {
          // S_{j+2} needs only that the softmax has read S_j: issue it first
          if (j + 2 < n) issue_s(it + j + 2, j + 3 == n);
          issue_pv(it + j, j == 0);
        }
        it += n;
      }
      // Every MMA must have completed before TMEM is released.
      mma_commit(&bars->mma_done);
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
    // write v, read the peer's: the first barrier guarantees the peer has read
    // the previous value, the second that it has written this one
    auto exchange = [&](float v) {
      named_bar_sync(bar_id, 64);
      *x_mine = v;
      named_bar_sync(bar_id, 64);
      return *x_peer;
    };
    constexpr float kRescaleThreshold = 8.0f;  // log2 units
    uint32_t it = 0, item_i = 0;
    for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
      const int bh = item / p.nt;
      const int t = p.order ? RADIAL_CHECK_INDEX(p.order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
      const int b = bh / p.heads, h = bh - b * p.heads;
      const int a = t * 128 + row;
      const bool valid = a < p.n;
      const int qi = valid ? a / p.s : 0;
      const int qk = valid ? a - qi * p.s : 0;
      const int p0 = p.row_ptr[t];
      const uint32_t n = static_cast<uint32_t>(p.row_ptr[t + 1] - p0);
      float m = -INFINITY;  // running max of scaled logits, log2 domain
      float l = 0.f;        // this warp's part of the running sum of exp2(logit - m)
      int kb_next = RADIAL_CHECK_INDEX(p.col_idx[p0], 0, p.nt);
      uint8_t kind_next = p.kind[p0];
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t g = it + j, sb = g & 1;
        const int kb = kb_next;
        const bool part = kind_next != kTileFull;
        if (j + 1 < n) {
          kb_next = RADIAL_CHECK_INDEX(p.col_idx[p0 + j + 1], 0, p.nt);
          kind_next = p.kind[p0 + j + 1];
        }
        mbar_wait(&bars->s_full[sb], (g >> 1) & 1, abort_flag);
        __syncwarp();
        tc_fence_after();
        const uint32_t tm_s = tmem + lane_addr + C::TM_S0 + sb * 128;
        uint32_t r[64];
        tmem_ld32(tm_s + col0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(tm_s + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        // the mask bits of a PARTIAL tile are computed while the load is in flight
        uint32_t mw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        uint32_t live = 3u;   // 32-key chunks with an allowed key in some lane of the warp
        uint32_t mixed = 0u;  // chunks that need the per-element select
        if (part) {
          mw[0] = mw[1] = mw[2] = mw[3] = 0u;
          if (valid) row_mask_bits(p, qi, qk, kb * 128 + col0, mw);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (!__any_sync(0xffffffffu, mw[c] != 0u)) live &= ~(1u << c);
            else if (!__all_sync(0xffffffffu, mw[c] == 0xffffffffu)) mixed |= 1u << c;
          }
        }
        tmem_wait_ld();
        // S buffer sb may now take S_{g+2}
        tc_fence_before();
        mbar_arrive(&bars->s_empty[sb]);
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
        const float m_tile = fmaxf(mloc, exchange(mloc)) * p.scale_log2;
        // lazy rescaling: m moves only when the tile's maximum exceeds it by
        // more than the threshold (P stays below 2^8)
        const bool grow = m_tile > m + kRescaleThreshold;
        const bool resc = j > 0 && __any_sync(0xffffffffu, grow);
        const float factor = (grow && j > 0) ? ex2_approx(m - m_tile) : 1.0f;
        if (grow) {
          l *= factor;
          m = m_tile;
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t negm = f2_pack(-m_use, -m_use);
        // P buffer sb was last read by PV_{g-2}
        if (g >= 2) {
          mbar_wait(&bars->pv_done[sb], ((g >> 1) - 1) & 1, abort_flag);
          __syncwarp();
          tc_fence_after();
        }
        const uint32_t tm_p = tmem + lane_addr + C::TM_P0 + sb * 64 + wg * 32;
        uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t w[16];
          if (!(live & (1u << c))) {
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = 0u;
            tmem_st16(tm_p + c * 16, w);
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
            float q0, q1;
            f2_unpack(pe, q0, q1);
            w[e] = pack_bf16x2(q0, q1);
          }
          // P (bf16 pairs) of keys [col0 + 32 c, +32) -> P columns (col0 + 32 c) / 2
          tmem_st16(tm_p + c * 16, w);
        }
        const uint64_t s01 = f2_add(acc2[0], acc2[1]);
        float s0, s1;
        f2_unpack(s01, s0, s1);
        l += s0 + s1;
        if (resc) {
          // O holds every PV up to PV_{g-1} once that one completes; this warp
          // rescales its half of the output columns
          mbar_wait(&bars->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag);
          __syncwarp();
          tc_fence_after();
          const uint32_t tm_o = tmem + lane_addr + C::TM_O + wg * (D / 2);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t ro[32];
            tmem_ld32(tm_o + c * 32, ro);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * factor);
            tmem_st32(tm_o + c * 32, ro);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[sb]);
      }
      // -------------------------------------------------------- epilogue
      const uint32_t g_last = it + n - 1;
      mbar_wait(&bars->pv_done[g_last & 1], (g_last >> 1) & 1, abort_flag);
      __syncwarp();
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
        if (valid) {
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
      mbar_arrive(&bars->o_empty);
      if (wg == 0 && valid) {
        const float lse = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.n + a] = lse;
      }
      it += n;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

}  // namespace radial
