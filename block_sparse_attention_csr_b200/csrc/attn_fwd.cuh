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
// with the temporal band; head-major keeps one head's K/V hot in L2).
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Q tile once per item, K/V tiles through a
//               STAGES-deep ring of shared-memory buffers.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               S_j = Q K_j^T into one of two TMEM S buffers, then
//               O += P_{j-1} V_{j-1} with P read from TMEM (A operand).
//   warps 2-5   softmax warpgroup: one thread per query row (TMEM lane).
//               Reads S_j from TMEM, masks PARTIAL tiles, keeps the running
//               max (log2 domain) and sum, writes P_j = exp2(..) as bf16 to
//               TMEM, rescales O in TMEM when the max grows by more than
//               2^8 (lazy rescaling), and at the end of the row normalises O
//               and writes O (bf16) and LSE (fp32, natural log).
//
// TMEM (512 columns x 128 lanes): S0 [0,128), S1 [128,256), O [256,256+D),
// P0 [384,448), P1 [448,512) (P as packed bf16 pairs).
//
// Shared memory: Q [128 x D] + STAGES x (K [128 x D] + V [128 x D]), bf16,
// TMA-written with the 128-byte swizzle in boxes of 64 columns.
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
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int STAGES = (D == 128) ? 3 : 4;
  static constexpr int TILE_BYTES = 128 * D * 2;  // one 128 x D bf16 tile
  static constexpr int NBOX = D / 64;             // 64-column swizzle boxes per tile
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = TILE_BYTES;
  static constexpr int SMEM_V = TILE_BYTES * (1 + STAGES);
  static constexpr int SMEM_BAR = TILE_BYTES * (1 + 2 * STAGES);
  static constexpr int SMEM_BYTES = SMEM_BAR + 256 + 1024;  // + barriers + alignment slack
  static constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_P0 = 384;
  static constexpr uint32_t TM_COLS = 512;
};

// Barrier slots (uint64 each) inside the barrier area.
struct FwdBars {
  uint64_t q_full, q_empty, o_empty;
  uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2];
  uint64_t k_full[4], v_full[4], kv_empty[4];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

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

// kFastSoftmax: tree reductions and packed fp32x2 FMA / add; otherwise the
// plain serial loop.  kPolyEvery > 0 computes every kPolyEvery-th pair of
// exponentials on the FMA pipe (exp2_poly_x2) instead of the MUFU.  Measured
// on B200 the softmax is issue-bound, not MUFU-bound (moving a quarter of the
// exponentials to the polynomial made the forward 4-5 % slower, half of them
// 13 %), so it is off.
constexpr int kPolyEvery = 0;
__host__ __device__ constexpr bool use_poly_exp(int e) {
  return kPolyEvery > 0 && (e % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1;
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

// Applies a chunk's mask in place to the raw fp32 bits of S (a fully masked
// chunk has word 0, so the select gives -inf there too).
__device__ __forceinline__ void mask_chunk_inplace(uint32_t (&r)[32], uint32_t word, uint32_t mode) {
  constexpr uint32_t kNegInf = 0xff800000u;
  if (mode != 0u) {
#pragma unroll
    for (int e = 0; e < 32; ++e) r[e] = ((word >> e) & 1u) ? r[e] : kNegInf;
  }
}

template <int D, bool kFastSoftmax>
__global__ void __launch_bounds__(192, 1)
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
    mbar_init(&bars->o_empty, 128);
    mbar_init(&bars->mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_empty[b], 128);
      mbar_init(&bars->p_full[b], 128);
      mbar_init(&bars->pv_done[b], 1);
    }
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
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
      uint32_t it = 0, item_i = 0;
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.nt;
        const int t = p.order ? p.order[item - bh * p.nt] : item - bh * p.nt;
        const int b = bh / p.heads, h = bh - b * p.heads;
        if (item_i > 0) mbar_wait(&bars->q_empty, (item_i - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->q_full, C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_4d(sQ + x * 16384, &tmQ, &bars->q_full, x * 64, t * 128, h, b);
        const int p0 = p.row_ptr[t], p1 = p.row_ptr[t + 1];
        for (int q = p0; q < p1; ++q, ++it) {
          const int kb = p.col_idx[q];
          const uint32_t st = it % C::STAGES;
          const uint32_t use = it / C::STAGES;
          if (use > 0) mbar_wait(&bars->kv_empty[st], (use - 1) & 1, abort_flag);
          mbar_arrive_expect_tx(&bars->k_full[st], C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d(sK + st * C::TILE_BYTES + x * 16384, &tmK, &bars->k_full[st], x * 64,
                        kb * 128, h, b);
          mbar_arrive_expect_tx(&bars->v_full[st], C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d(sV + st * C::TILE_BYTES + x * 16384, &tmV, &bars->v_full[st], x * 64,
                        kb * 128, h, b);
        }
      }
      // Drain: every stage's last fill must have landed before the CTA exits.
      for (uint32_t k = (it > C::STAGES ? it - C::STAGES : 0); k < it; ++k) {
        const uint32_t st = k % C::STAGES, use = k / C::STAGES;
        mbar_wait_drain(&bars->k_full[st], use & 1);
        mbar_wait_drain(&bars->v_full[st], use & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      // descriptors built once; stages and K-steps are start-address offsets
      constexpr uint64_t kTile = C::TILE_BYTES >> 4;
      const uint64_t dQ = smem_desc(smem_u32(sQ), 16, 1024, kSwizzle128B);
      const uint64_t dK0 = smem_desc(smem_u32(sK), 16, 1024, kSwizzle128B);
      const uint64_t dV0 = smem_desc(smem_u32(sV), 16384, 1024, kSwizzle128B);
      uint32_t it = 0, item_i = 0;
      auto issue_pv = [&](uint32_t g, uint32_t j) {
        const uint32_t st = g % C::STAGES, pb = g & 1;
        mbar_wait(&bars->p_full[pb], (g >> 1) & 1, abort_flag);
        mbar_wait(&bars->v_full[st], (g / C::STAGES) & 1, abort_flag);
        if (j == 0 && item_i > 0) mbar_wait(&bars->o_empty, (item_i - 1) & 1, abort_flag);
        tc_fence_after();
        const uint64_t dv = dV0 + st * kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + C::TM_O, tmem + C::TM_P0 + pb * 64 + kk * 8, dv + kk * (2048 >> 4), idesc_o,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->pv_done[pb]);
        mma_commit(&bars->kv_empty[st]);
      };
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.nt;
        const int t = p.order ? p.order[item - bh * p.nt] : item - bh * p.nt;
        const uint32_t n_tiles = static_cast<uint32_t>(p.row_ptr[t + 1] - p.row_ptr[t]);
        mbar_wait(&bars->q_full, item_i & 1, abort_flag);
        tc_fence_after();
        for (uint32_t j = 0; j < n_tiles; ++j) {
          const uint32_t g = it + j;
          const uint32_t st = g % C::STAGES, sb = g & 1;
          mbar_wait(&bars->k_full[st], (g / C::STAGES) & 1, abort_flag);
          if (g >= 2) mbar_wait(&bars->s_empty[sb], ((g >> 1) - 1) & 1, abort_flag);
          tc_fence_after();
          const uint64_t dk = dK0 + st * kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss(tmem + C::TM_S0 + sb * 128, dQ + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full[sb]);
          if (j + 1 == n_tiles) mma_commit(&bars->q_empty);
          if (j > 0) issue_pv(g - 1, j - 1);
        }
        issue_pv(it + n_tiles - 1, n_tiles - 1);
        it += n_tiles;
      }
      // Every MMA must have completed before TMEM is released.
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax WG
    const int quarter = warp & 3;               // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;        // row of the query tile
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr float kRescaleThreshold = 8.0f;  // log2 units
    uint32_t it = 0, item_i = 0;
    for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
      const int bh = item / p.nt;
      const int t = p.order ? p.order[item - bh * p.nt] : item - bh * p.nt;
      const int b = bh / p.heads, h = bh - b * p.heads;
      const int a = t * 128 + row;
      const bool valid = a < p.n;
      const int qi = valid ? a / p.s : 0;
      const int qk = valid ? a - qi * p.s : 0;
      const int p0 = p.row_ptr[t];
      const uint32_t n_tiles = static_cast<uint32_t>(p.row_ptr[t + 1] - p0);
      float m = -INFINITY;  // running max of scaled logits, log2 domain
      float l = 0.f;        // running sum of exp2(logit - m)
      for (uint32_t j = 0; j < n_tiles; ++j) {
        const uint32_t g = it + j, sb = g & 1;
        const int kb = p.col_idx[p0 + j];
        const bool partial = p.kind[p0 + j] != kTileFull;
        mbar_wait(&bars->s_full[sb], (g >> 1) & 1, abort_flag);
        __syncwarp();
        tc_fence_after();
        float sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + C::TM_S0 + sb * 128 + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(r[e]);
        }
        tc_fence_before();
        mbar_arrive(&bars->s_empty[sb]);
        if (partial) {
          uint32_t mw[4] = {0u, 0u, 0u, 0u};
          if (valid) row_mask_bits(p, qi, qk, kb * 128, mw);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!((mw[c >> 5] >> (c & 31)) & 1u)) sv[c] = -INFINITY;
        }
        float tmax;
        if constexpr (kFastSoftmax) {
          float acc[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
          for (int c = 4; c + 8 <= 128; c += 8)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = max3f(acc[k], sv[c + k], sv[c + 4 + k]);
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[k] = fmaxf(acc[k], sv[124 + k]);
          tmax = max3f(acc[0], acc[1], fmaxf(acc[2], acc[3]));
        } else {
          tmax = sv[0];
#pragma unroll
          for (int c = 1; c < 128; ++c) tmax = fmaxf(tmax, sv[c]);
        }
        const float m_tile = tmax * p.scale_log2;  // -inf stays -inf (scale > 0)
        const bool grow = m_tile > m + kRescaleThreshold;
        if (j > 0) {
          if (__any_sync(0xffffffffu, grow)) {
            // O is being accumulated by PV_{j-1}: wait for it, then rescale rows.
            mbar_wait(&bars->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag);
            __syncwarp();
            tc_fence_after();
            const float factor = grow ? ex2_approx(m - m_tile) : 1.0f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tmem_ld32(tmem + lane_addr + C::TM_O + c * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * factor);
              tmem_st32(tmem + lane_addr + C::TM_O + c * 32, r);
            }
            tmem_wait_st();
            if (grow) {
              l *= factor;
              m = m_tile;
            }
          }
        } else if (grow) {
          m = m_tile;
        }
        // P buffer sb was last read by PV_{g-2}.
        if (g >= 2) {
          mbar_wait(&bars->pv_done[sb], ((g >> 1) - 1) & 1, abort_flag);
          __syncwarp();
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        float lsum = 0.f;
        if constexpr (kFastSoftmax) {
          const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t negm = f2_pack(-m_use, -m_use);
          uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int i0 = c * 64 + 2 * e;
              const uint64_t x = f2_fma(f2_pack(sv[i0], sv[i0 + 1]), sl2, negm);
              uint64_t pe;
              if (use_poly_exp(e)) {
                pe = exp2_poly_x2(x);
              } else {
                float x0, x1;
                f2_unpack(x, x0, x1);
                pe = f2_pack(ex2_approx(x0), ex2_approx(x1));
              }
              acc2[e & 3] = f2_add(acc2[e & 3], pe);
              float p0, p1;
              f2_unpack(pe, p0, p1);
              w[e] = pack_bf16x2(p0, p1);
            }
            tmem_st32(tmem + lane_addr + C::TM_P0 + sb * 64 + c * 32, w);
          }
          const uint64_t s01 = f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3]));
          float s0, s1;
          f2_unpack(s01, s0, s1);
          lsum = s0 + s1;
        } else {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x0 = ex2_approx(fmaf(sv[c * 64 + 2 * e], p.scale_log2, -m_use));
              const float x1 = ex2_approx(fmaf(sv[c * 64 + 2 * e + 1], p.scale_log2, -m_use));
              lsum += x0 + x1;
              w[e] = pack_bf16x2(x0, x1);
            }
            tmem_st32(tmem + lane_addr + C::TM_P0 + sb * 64 + c * 32, w);
          }
        }
        l += lsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[sb]);
      }
      // -------------------------------------------------------- epilogue
      const uint32_t g_last = it + n_tiles - 1;
      mbar_wait(&bars->pv_done[g_last & 1], (g_last >> 1) & 1, abort_flag);
      __syncwarp();
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* orow = p.o + static_cast<int64_t>(b) * p.o_sb + static_cast<int64_t>(h) * p.o_sh +
                            static_cast<int64_t>(valid ? a : 0) * p.o_sn;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + C::TM_O + c * 32, r);
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
      mbar_arrive(&bars->o_empty);
      if (valid) {
        const float lse = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.n + a] = lse;
      }
      it += n_tiles;
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
