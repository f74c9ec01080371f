// Block-sparse backward of Radial Attention on sm_100a.
//
// Gradients of O = softmax(Q K^T * scale + M) V (the sparse-attention
// equation, Eq.2, of the Radial Attention review on jaehun.me, §3) with
// respect to Q, K and V, as the LoRA length-extension fine-tuning of §4.3
// back-propagates through every radial attention layer.  With
// P = exp(S*scale - LSE) (S = Q K^T, masked), Dr = rowsum(dO o O):
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - Dr),
//   dK = scale * dS^T Q,          dQ = scale * dS K.
// Only the mask's active 128x128 tiles are visited (§4.2, block-wise).
//
// Three kernels, no atomics, deterministic:
//  1. bwd_rowdot:  Dr[row] = sum_d dO*O (fp32, into the caller's workspace).
//  2. bwd_dkdv:    one work item per (batch*head, 128-key tile); walks the
//                  query tiles of the mask's CSC column: S^T = K Q^T and
//                  dP^T = V dO^T into TMEM; one thread per key row forms P^T
//                  and dS^T (bf16, written back over the consumed S^T / dP^T
//                  columns); dV += P^T dO and dK += dS^T Q accumulate in TMEM
//                  with P^T / dS^T as the TMEM A operand.
//  3. bwd_dq:      one work item per (batch*head, 128-query tile); walks the
//                  CSR row: S = Q K^T, dP = dO V^T into TMEM; one thread per
//                  query row forms dS (bf16, TMEM); dQ += dS K in TMEM.
// Recomputing S and dP in (3) costs 2 extra GEMMs per tile (7 instead of 5)
// and removes the fp32 dQ atomics a single fused pass would need.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "attn_fwd.cuh"
#include "mask_build.cuh"
#include "sm100_primitives.cuh"

namespace radial {

// ---------------------------------------------------------------------------
// 1. Dr = rowsum(dO o O)
// ---------------------------------------------------------------------------
template <int D>
__global__ void bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ dO, const __nv_bfloat16* __restrict__ O,
                                  int heads, int n, int64_t sb, int64_t sh, int64_t sn,
                                  int64_t rows, float* __restrict__ dr) {
  // 16 threads per row, 8 bf16 (16 bytes) per thread per step
  constexpr int TPR = 16;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / TPR;
  const int sub = threadIdx.x % TPR;
  float acc = 0.f;
  if (row < rows) {
    const int64_t bh = row / n;
    const int a = static_cast<int>(row - bh * n);
    const int b = static_cast<int>(bh / heads), h = static_cast<int>(bh - static_cast<int64_t>(b) * heads);
    const int64_t off = b * sb + h * sh + a * sn;
#pragma unroll
    for (int c = sub * 8; c < D; c += TPR * 8) {
      const uint4 x = *reinterpret_cast<const uint4*>(dO + off + c);
      const uint4 y = *reinterpret_cast<const uint4*>(O + off + c);
      const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&x);
      const __nv_bfloat162* yp = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 xf = __bfloat1622float2(xp[e]);
        const float2 yf = __bfloat1622float2(yp[e]);
        acc = fmaf(xf.x, yf.x, acc);
        acc = fmaf(xf.y, yf.y, acc);
      }
    }
  }
#pragma unroll
  for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (row < rows && sub == 0) dr[row] = acc;
}

struct BwdParams {
  // 128-token tile plan: CSR (query-major) and CSC (key-major)
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const uint8_t* kind;
  const int32_t* row_order;
  const int32_t* col_ptr;
  const int32_t* row_idx;
  const uint8_t* kind_t;
  const int32_t* col_order;
  int32_t nt;
  int32_t f, s, n, sink;
  int32_t heads, items;
  int64_t sb, sh, sn;  // element strides shared by all bf16 tensors
  const float* lse;    // [B, H, N]
  const float* dr;     // [B, H, N]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float scale;
  float scale_log2;
  const int32_t* hd;  // ablation-mask distance tables (nullptr: closed form)
  const int32_t* cd;
};

template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NBOX = D / 64;
  static constexpr int STAGES = 2;
  // smem: fixed pair (2 tiles) + STAGES x streamed pair (2 tiles each)
  static constexpr int SMEM_FIX = 0;
  static constexpr int SMEM_STREAM = 2 * TILE_BYTES;
  static constexpr int SMEM_VEC = SMEM_STREAM + STAGES * 2 * TILE_BYTES;  // 2 x 2 x 128 floats
  static constexpr int SMEM_BAR = SMEM_VEC + 2 * 2 * 128 * 4;
  static constexpr int SMEM_BYTES = SMEM_BAR + 256 + 1024;
  // dQ kernel: Q, dO fixed, then a K ring (read by S and, a tile later, by
  // dQ) and a V ring (read by dP only, so its slots free a step earlier)
  static constexpr int DQ_K_SLOTS = 3;
  static constexpr int DQ_V_SLOTS = 2;
  static constexpr int DQ_SMEM_K = SMEM_STREAM;
  static constexpr int DQ_SMEM_V = DQ_SMEM_K + DQ_K_SLOTS * TILE_BYTES;
  static constexpr int DQ_SMEM_BAR = DQ_SMEM_V + DQ_V_SLOTS * TILE_BYTES;
  static constexpr int DQ_SMEM_BYTES = DQ_SMEM_BAR + 256 + 1024;
};

struct BwdBars {
  uint64_t fix_full, fix_empty, acc_empty, mma_done;
  uint64_t s_full, s_free, ew_full[2], mma2_done[2];
  uint64_t st_full[2], st_empty[2];
  uint64_t dp_full, p_ready[2], ds_ready[2];  // dK/dV kernel: S^T and dP^T halves of the handoff
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];  // dQ kernel: the K and V rings
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(BwdBars) <= 256, "barrier area");

// ---------------------------------------------------------------------------
// 2. dK, dV: key-major walk of the CSC
// ---------------------------------------------------------------------------
// TMEM: dK [0,D) dV [128,128+D) S^T [256,384) dP^T [384,512).  Warps: 0
// producer, 1 MMA, 2-3 idle, 4-7 and 8-11 the two elementwise warpgroups
// (query columns [0,64) and [64,128) of each tile).  Warpgroup wg writes its
// bf16 P^T over S^T columns [64 wg, 64 wg + 32) and its dS^T over dP^T columns
// [64 wg, 64 wg + 32), i.e. over values it has already read.
// The elementwise work of a query tile runs in two passes, each released to
// the MMA thread on its own barrier: P^T (needs only S^T) and then dS^T (needs
// dP^T and the P^T values kept in registers).  The MMA stream per tile g is
// dV(g), S^T(g+1), dK(g), dP^T(g+1): dV(g) and the next S^T run while the
// elementwise warps form dS^T(g), and dK(g) and the next dP^T while they form
// P^T(g+1).  Each new S^T / dP^T follows, in the same in-order MMA stream,
// the MMA that reads the P^T / dS^T it overwrites.
template <int D>
__global__ void __launch_bounds__(384, 1)
    radial_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                           const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem + C::SMEM_FIX;
  uint8_t* sV = sK + C::TILE_BYTES;
  uint8_t* sQ = smem + C::SMEM_STREAM;                 // stage st: sQ + st*2*TILE
  float* sVec = reinterpret_cast<float*>(smem + C::SMEM_VEC);  // [2 buf][lse2 | dr][128]
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::SMEM_BAR);
  volatile int* abort_flag = &bars->abort;
  constexpr uint32_t TM_DK = 0, TM_DV = 128, TM_S = 256, TM_DP = 384;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    bars->abort = 0;
    mbar_init(&bars->fix_full, 1);
    mbar_init(&bars->fix_empty, 1);
    mbar_init(&bars->acc_empty, 256);
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 128);
    mbar_init(&bars->dp_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->p_ready[b], 256);
      mbar_init(&bars->ds_ready[b], 256);
      mbar_init(&bars->ew_full[b], 256);
      mbar_init(&bars->mma2_done[b], 1);
      mbar_init(&bars->st_full[b], 1);
      mbar_init(&bars->st_empty[b], 1);
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
    if (lane == 0) {
      uint32_t it = 0, item_i = 0;
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.nt;
        const int u = p.col_order ? RADIAL_CHECK_INDEX(p.col_order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
        const int b = bh / p.heads, h = bh - b * p.heads;
        if (item_i > 0) mbar_wait(&bars->fix_empty, (item_i - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->fix_full, 2 * C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x) {
          tma_load_4d(sK + x * 16384, &tmK, &bars->fix_full, x * 64, u * 128, h, b);
          tma_load_4d(sV + x * 16384, &tmV, &bars->fix_full, x * 64, u * 128, h, b);
        }
        for (int q = p.col_ptr[u]; q < p.col_ptr[u + 1]; ++q, ++it) {
          const int t = RADIAL_CHECK_INDEX(p.row_idx[q], 0, p.nt);
          const uint32_t st = it % C::STAGES, use = it / C::STAGES;
          if (use > 0) mbar_wait(&bars->st_empty[st], (use - 1) & 1, abort_flag);
          uint8_t* dstQ = sQ + st * 2 * C::TILE_BYTES;
          uint8_t* dstO = dstQ + C::TILE_BYTES;
          mbar_arrive_expect_tx(&bars->st_full[st], 2 * C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < C::NBOX; ++x) {
            tma_load_4d(dstQ + x * 16384, &tmQ, &bars->st_full[st], x * 64, t * 128, h, b);
            tma_load_4d(dstO + x * 16384, &tmdO, &bars->st_full[st], x * 64, t * 128, h, b);
          }
        }
      }
      for (uint32_t k = (it > C::STAGES ? it - C::STAGES : 0); k < it; ++k)
        mbar_wait_drain(&bars->st_full[k % C::STAGES], (k / C::STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, false, true);
      // descriptors built once; stages and K-steps are offsets (see the forward)
      constexpr uint64_t kTile = C::TILE_BYTES >> 4;
      const uint64_t dK = smem_desc(smem_u32(sK), 16, 1024, kSwizzle128B);
      const uint64_t dV = smem_desc(smem_u32(sV), 16, 1024, kSwizzle128B);
      const uint64_t dQk = smem_desc(smem_u32(sQ), 16, 1024, kSwizzle128B);       // Q, dO as K-major B
      const uint64_t dQmn = smem_desc(smem_u32(sQ), 16384, 1024, kSwizzle128B);   // Q, dO as MN-major B
      uint32_t it = 0, item_i = 0;
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.nt;
        const int u = p.col_order ? RADIAL_CHECK_INDEX(p.col_order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
        const uint32_t n_tiles = static_cast<uint32_t>(p.col_ptr[u + 1] - p.col_ptr[u]);
        mbar_wait(&bars->fix_full, item_i & 1, abort_flag);
        tc_fence_after();
        // S^T(g) = K Q_g^T and dP^T(g) = V dO_g^T (Q, dO of stage g as K-major B)
        auto issue_s = [&](uint32_t g) {
          const uint32_t st = g % C::STAGES;
          mbar_wait(&bars->st_full[st], (g / C::STAGES) & 1, abort_flag);
          tc_fence_after();
          const uint64_t qk = dQk + st * 2 * kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss(tmem + TM_S, dK + off, qk + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full);
        };
        auto issue_dp = [&](uint32_t g) {
          const uint32_t st = g % C::STAGES;
          const uint64_t ok = dQk + st * 2 * kTile + kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss(tmem + TM_DP, dV + off, ok + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->dp_full);
        };
        issue_s(it);
        issue_dp(it);
        for (uint32_t j = 0; j < n_tiles; ++j) {
          const uint32_t g = it + j, st = g % C::STAGES;
          const uint64_t qmn = dQmn + st * 2 * kTile, omn = qmn + kTile;
          // dV(g) += P^T(g) dO_g, once the elementwise warps have written P^T(g)
          mbar_wait(&bars->p_ready[g & 1], (g >> 1) & 1, abort_flag);
          if (j == 0 && item_i > 0) mbar_wait(&bars->acc_empty, (item_i - 1) & 1, abort_flag);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // K = 128 query rows, 16 per MMA
            mma_ts(tmem + TM_DV, tmem + TM_S + 64 * (kk >> 2) + 8 * (kk & 3), omn + kk * (2048 >> 4), idesc_g,
                   (j > 0 || kk > 0) ? 1u : 0u);
          // S^T(g+1) overwrites P^T(g) after dV(g) has read it (same MMA stream)
          if (j + 1 < n_tiles) issue_s(g + 1);
          // dK(g) += dS^T(g) Q_g
          mbar_wait(&bars->ds_ready[g & 1], (g >> 1) & 1, abort_flag);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + TM_DK, tmem + TM_DP + 64 * (kk >> 2) + 8 * (kk & 3), qmn + kk * (2048 >> 4), idesc_g,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars->mma2_done[g & 1]);
          mma_commit(&bars->st_empty[st]);
          if (j + 1 == n_tiles) mma_commit(&bars->fix_empty);
          // dP^T(g+1) overwrites dS^T(g) after dK(g) has read it
          if (j + 1 < n_tiles) issue_dp(g + 1);
        }
        it += n_tiles;
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0);
    }
  } else if (warp >= 4) {
    // Two warpgroups split each tile by query columns: warpgroup wg owns
    // queries [64 wg, 64 wg + 64) of the tile, for all 128 key rows (lanes).
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr float kLog2e = 1.4426950408889634f;
    float* my_vec = sVec + wg * 256;  // [2 buffers][64 lse2 | 64 dr]
    uint32_t it = 0, item_i = 0;
    for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
      const int bh = item / p.nt;
      const int u = p.col_order ? RADIAL_CHECK_INDEX(p.col_order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
      const int b = bh / p.heads, h = bh - b * p.heads;
      const int key = u * 128 + row;
      const bool valid = key < p.n;
      const int kj = valid ? key / p.s : 0;
      const int kl = valid ? key - kj * p.s : 0;
      RowMaskGeom mg{};
      mg.f = p.f;
      mg.s = p.s;
      mg.n = p.n;
      mg.sink = p.sink;
      mg.hd = p.hd;
      mg.cd = p.cd;
      set_divisor(mg);
      const int c0 = p.col_ptr[u];
      const uint32_t n_tiles = static_cast<uint32_t>(p.col_ptr[u + 1] - c0);
      const float* lse_bh = p.lse + static_cast<int64_t>(bh) * p.n;
      const float* dr_bh = p.dr + static_cast<int64_t>(bh) * p.n;
      for (uint32_t j = 0; j < n_tiles; ++j) {
        const uint32_t g = it + j;
        const int t = RADIAL_CHECK_INDEX(p.row_idx[c0 + j], 0, p.nt);
        const bool partial = p.kind_t[c0 + j] != kTileFull;
        // this warpgroup's 64 queries: lse2 and dr -> shared memory
        float* vbuf = my_vec + (g & 1) * 128;
        {
          const int a = t * 128 + 64 * wg + (row & 63);
          if (row < 64)
            vbuf[row] = a < p.n ? lse_bh[a] * kLog2e : INFINITY;
          else
            vbuf[row] = a < p.n ? dr_bh[a] : 0.f;
        }
        named_bar_sync(1 + wg, 128);
        // this warpgroup's 64 queries of the tile, one bit each
        uint32_t mw[2] = {0xffffffffu, 0xffffffffu};
        if (partial) {
          const uint64_t m64 = valid ? col_mask64(mg, kj, kl, t * 128 + 64 * wg) : 0ull;
          mw[0] = static_cast<uint32_t>(m64);
          mw[1] = static_cast<uint32_t>(m64 >> 32);
        }
        const uint32_t modes = partial ? chunk_modes(mw) : 0u;
        // pass 1: P^T = exp2(S^T * scale*log2e - lse2), kept in fp32 for pass 2
        mbar_wait(&bars->s_full, g & 1, abort_flag);
        __syncwarp();
        tc_fence_after();
        float pv[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int gc = 2 * wg + c;  // 32-column chunk of the tile
          const uint32_t mode = (modes >> (2 * c)) & 3u;
          uint32_t pw[16];
          if (mode == 2u) {  // every lane of the warp masks this chunk: P^T = 0
#pragma unroll
            for (int e = 0; e < 32; ++e) pv[32 * c + e] = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) pw[e] = 0u;
          } else {
            uint32_t rs[32];
            tmem_ld32(tmem + lane_addr + TM_S + gc * 32, rs);
            tmem_wait_ld();
            const uint32_t bits = mode == 0u ? 0xffffffffu : mw[c];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x = fmaf(__uint_as_float(rs[e]), p.scale_log2, -vbuf[c * 32 + e]);
              const float pe = ex2_approx(x);
              pv[32 * c + e] = (mode == 0u || ((bits >> e) & 1u)) ? pe : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) pw[e] = pack_bf16x2(pv[32 * c + 2 * e], pv[32 * c + 2 * e + 1]);
          }
          // bf16 P^T goes to this warpgroup's own columns, over S^T it has already read
          tmem_st16(tmem + lane_addr + TM_S + 64 * wg + c * 16, pw);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_ready[g & 1]);
        // pass 2: dS^T = P^T * (dP^T - Dr)
        mbar_wait(&bars->dp_full, g & 1, abort_flag);
        __syncwarp();
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int gc = 2 * wg + c;
          const uint32_t mode = (modes >> (2 * c)) & 3u;
          uint32_t dw[16];
          if (mode == 2u) {
#pragma unroll
            for (int e = 0; e < 16; ++e) dw[e] = 0u;
          } else {
            uint32_t rp[32];
            tmem_ld32(tmem + lane_addr + TM_DP + gc * 32, rp);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int q0 = c * 32 + 2 * e;  // query index inside this warpgroup's 64
              const float d0 = pv[q0] * (__uint_as_float(rp[2 * e]) - vbuf[64 + q0]);
              const float d1 = pv[q0 + 1] * (__uint_as_float(rp[2 * e + 1]) - vbuf[64 + q0 + 1]);
              dw[e] = pack_bf16x2(d0, d1);
            }
          }
          tmem_st16(tmem + lane_addr + TM_DP + 64 * wg + c * 16, dw);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready[g & 1]);
      }
      // epilogue: warpgroup 0 writes dK (scaled), warpgroup 1 writes dV
      const uint32_t g_last = it + n_tiles - 1;
      mbar_wait(&bars->mma2_done[g_last & 1], (g_last >> 1) & 1, abort_flag);
      __syncwarp();
      tc_fence_after();
      const int64_t off = static_cast<int64_t>(b) * p.sb + static_cast<int64_t>(h) * p.sh +
                          static_cast<int64_t>(valid ? key : 0) * p.sn;
      {
        const uint32_t col = wg == 0 ? TM_DK : TM_DV;
        const float mul = wg == 0 ? p.scale : 1.0f;
        __nv_bfloat16* dst = (wg == 0 ? p.dk : p.dv) + off;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + col + c * 32, r);
          tmem_wait_ld();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
            uint4* o4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) o4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
      it += n_tiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// 3. dQ: query-major walk of the CSR
// ---------------------------------------------------------------------------
// TMEM: S [0,128) dP [128,256) dQ [256,256+D) dS0 [384,448) dS1 [448,512).
// Warps: 0 producer, 1 MMA, 2-3 idle, 4-7 and 8-11 the elementwise
// warpgroups (key columns [0,64) and [64,128) of each tile).
// Shared memory: Q and dO of the query tile, a 3-slot K ring and a 2-slot V
// ring (224 KB at D = 128).  K(g) is read by S(g) and by dQ(g), which is
// issued a tile later; V(g) only by dP(g), so its slot is released by the
// commit after dP(g).  With one shared 2-stage ring the load of K/V(g + 1)
// could start only when dQ(g - 1) completed, just before S(g + 1) needs it:
// the MMA issuer waited about 1,200 of its 4,300 cycles per tile on it.
template <int D>
__global__ void __launch_bounds__(384, 1)
    radial_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                         const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::SMEM_FIX;
  uint8_t* sdO = sQ + C::TILE_BYTES;
  uint8_t* sK = smem + C::DQ_SMEM_K;  // slot g % DQ_K_SLOTS
  uint8_t* sV = smem + C::DQ_SMEM_V;  // slot g % DQ_V_SLOTS
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::DQ_SMEM_BAR);
  volatile int* abort_flag = &bars->abort;
  constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256, TM_DS = 384;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    bars->abort = 0;
    mbar_init(&bars->fix_full, 1);
    mbar_init(&bars->fix_empty, 1);
    mbar_init(&bars->acc_empty, 256);
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 256);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->ew_full[b], 256);
      mbar_init(&bars->mma2_done[b], 1);
    }
    for (int b = 0; b < C::DQ_K_SLOTS; ++b) {
      mbar_init(&bars->k_full[b], 1);
      mbar_init(&bars->k_empty[b], 1);
    }
    for (int b = 0; b < C::DQ_V_SLOTS; ++b) {
      mbar_init(&bars->v_full[b], 1);
      mbar_init(&bars->v_empty[b], 1);
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
    if (lane == 0) {
      uint32_t it = 0, item_i = 0;
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.nt;
        const int t = p.row_order ? RADIAL_CHECK_INDEX(p.row_order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
        const int b = bh / p.heads, h = bh - b * p.heads;
        if (item_i > 0) mbar_wait(&bars->fix_empty, (item_i - 1) & 1, abort_flag);
        mbar_arrive_expect_tx(&bars->fix_full, 2 * C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::NBOX; ++x) {
          tma_load_4d(sQ + x * 16384, &tmQ, &bars->fix_full, x * 64, t * 128, h, b);
          tma_load_4d(sdO + x * 16384, &tmdO, &bars->fix_full, x * 64, t * 128, h, b);
        }
        for (int q = p.row_ptr[t]; q < p.row_ptr[t + 1]; ++q, ++it) {
          const int kb = RADIAL_CHECK_INDEX(p.col_idx[q], 0, p.nt);
          const uint32_t ks = it % C::DQ_K_SLOTS, ku = it / C::DQ_K_SLOTS;
          if (ku > 0) mbar_wait(&bars->k_empty[ks], (ku - 1) & 1, abort_flag);
          mbar_arrive_expect_tx(&bars->k_full[ks], C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d(sK + ks * C::TILE_BYTES + x * 16384, &tmK, &bars->k_full[ks], x * 64, kb * 128, h, b);
          const uint32_t vs = it % C::DQ_V_SLOTS, vu = it / C::DQ_V_SLOTS;
          if (vu > 0) mbar_wait(&bars->v_empty[vs], (vu - 1) & 1, abort_flag);
          mbar_arrive_expect_tx(&bars->v_full[vs], C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d(sV + vs * C::TILE_BYTES + x * 16384, &tmV, &bars->v_full[vs], x * 64, kb * 128, h, b);
        }
      }
      for (uint32_t k = (it > C::DQ_K_SLOTS ? it - C::DQ_K_SLOTS : 0); k < it; ++k)
        mbar_wait_drain(&bars->k_full[k % C::DQ_K_SLOTS], (k / C::DQ_K_SLOTS) & 1);
      for (uint32_t k = (it > C::DQ_V_SLOTS ? it - C::DQ_V_SLOTS : 0); k < it; ++k)
        mbar_wait_drain(&bars->v_full[k % C::DQ_V_SLOTS], (k / C::DQ_V_SLOTS) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, false, true);
      constexpr uint64_t kTile = C::TILE_BYTES >> 4;
      const uint64_t dQ = smem_desc(smem_u32(sQ), 16, 1024, kSwizzle128B);
      const uint64_t dO = smem_desc(smem_u32(sdO), 16, 1024, kSwizzle128B);
      const uint64_t dKk = smem_desc(smem_u32(sK), 16, 1024, kSwizzle128B);       // K as K-major B
      const uint64_t dVk = smem_desc(smem_u32(sV), 16, 1024, kSwizzle128B);       // V as K-major B
      const uint64_t dKmn = smem_desc(smem_u32(sK), 16384, 1024, kSwizzle128B);   // K as MN-major B
      uint32_t it = 0, item_i = 0;
      auto issue_dq = [&](uint32_t g, uint32_t j) {
        const uint32_t ks = g % C::DQ_K_SLOTS, db = g & 1;
        mbar_wait(&bars->ew_full[db], (g >> 1) & 1, abort_flag);
        if (j == 0 && item_i > 0) mbar_wait(&bars->acc_empty, (item_i - 1) & 1, abort_flag);
        tc_fence_after();
        const uint64_t kmn = dKmn + ks * kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + TM_DQ, tmem + TM_DS + db * 64 + kk * 8, kmn + kk * (2048 >> 4), idesc_g,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->mma2_done[db]);
        mma_commit(&bars->k_empty[ks]);
      };
      for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
        const int bh = item / p.nt;
        const int t = p.row_order ? RADIAL_CHECK_INDEX(p.row_order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
        const uint32_t n_tiles = static_cast<uint32_t>(p.row_ptr[t + 1] - p.row_ptr[t]);
        mbar_wait(&bars->fix_full, item_i & 1, abort_flag);
        tc_fence_after();
        for (uint32_t j = 0; j < n_tiles; ++j) {
          const uint32_t g = it + j, ks = g % C::DQ_K_SLOTS, vs = g % C::DQ_V_SLOTS;
          mbar_wait(&bars->k_full[ks], (g / C::DQ_K_SLOTS) & 1, abort_flag);
          mbar_wait(&bars->v_full[vs], (g / C::DQ_V_SLOTS) & 1, abort_flag);
          if (g >= 1) mbar_wait(&bars->s_free, (g - 1) & 1, abort_flag);
          tc_fence_after();
          const uint64_t kk_ = dKk + ks * kTile, vk = dVk + vs * kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss(tmem + TM_S, dQ + off, kk_ + off, idesc_s, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss(tmem + TM_DP, dO + off, vk + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full);
          mma_commit(&bars->v_empty[vs]);  // dP(g) has read V(g)
          if (j + 1 == n_tiles) mma_commit(&bars->fix_empty);
          if (j > 0) issue_dq(g - 1, j - 1);
        }
        issue_dq(it + n_tiles - 1, n_tiles - 1);
        it += n_tiles;
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0);
    }
  } else if (warp >= 4) {
    const int wg = (warp - 4) >> 2;  // key columns [64 wg, 64 wg + 64) of each tile
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr float kLog2e = 1.4426950408889634f;
    uint32_t it = 0, item_i = 0;
    for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
      const int bh = item / p.nt;
      const int t = p.row_order ? RADIAL_CHECK_INDEX(p.row_order[item - bh * p.nt], 0, p.nt) : item - bh * p.nt;
      const int b = bh / p.heads, h = bh - b * p.heads;
      const int a = t * 128 + row;
      const bool valid = a < p.n;
      const int qi = valid ? a / p.s : 0;
      const int qk = valid ? a - qi * p.s : 0;
      RowMaskGeom mg{};
      mg.f = p.f;
      mg.s = p.s;
      mg.n = p.n;
      mg.sink = p.sink;
      mg.hd = p.hd;
      mg.cd = p.cd;
      set_divisor(mg);
      const float lse2 = valid ? p.lse[static_cast<int64_t>(bh) * p.n + a] * kLog2e : INFINITY;
      const float drow = valid ? p.dr[static_cast<int64_t>(bh) * p.n + a] : 0.f;
      const int p0 = p.row_ptr[t];
      const uint32_t n_tiles = static_cast<uint32_t>(p.row_ptr[t + 1] - p0);
      for (uint32_t j = 0; j < n_tiles; ++j) {
        const uint32_t g = it + j, db = g & 1;
        const int kb = RADIAL_CHECK_INDEX(p.col_idx[p0 + j], 0, p.nt);
        const bool partial = p.kind[p0 + j] != kTileFull;
        // this warpgroup's 64 keys of the tile, one bit each
        uint32_t mw[2] = {0xffffffffu, 0xffffffffu};
        if (partial) {
          const uint64_t m64 = valid ? row_mask64(mg, qi, qk, kb * 128 + 64 * wg) : 0ull;
          mw[0] = static_cast<uint32_t>(m64);
          mw[1] = static_cast<uint32_t>(m64 >> 32);
        }
        // dS buffer db was read by the dQ MMA of tile g-2
        if (g >= 2) {
          mbar_wait(&bars->mma2_done[db], ((g >> 1) - 1) & 1, abort_flag);
          __syncwarp();
        }
        const uint32_t modes = partial ? chunk_modes(mw) : 0u;
        mbar_wait(&bars->s_full, g & 1, abort_flag);
        __syncwarp();
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int gc = 2 * wg + c;
          const uint32_t mode = (modes >> (2 * c)) & 3u;
          uint32_t dw[16];
          if (mode == 2u) {  // every lane of the warp masks this chunk: dS = 0
#pragma unroll
            for (int e = 0; e < 16; ++e) dw[e] = 0u;
            if (c == 1) {  // S and dP fully read: the next tile's S / dP may overwrite them
              tc_fence_before();
              mbar_arrive(&bars->s_free);
            }
          } else {
            uint32_t rs[32], rp[32];
            tmem_ld32(tmem + lane_addr + TM_S + gc * 32, rs);
            tmem_ld32(tmem + lane_addr + TM_DP + gc * 32, rp);
            tmem_wait_ld();
            if (c == 1) {  // S and dP fully read: the next tile's S / dP may overwrite them
              tc_fence_before();
              mbar_arrive(&bars->s_free);
            }
            const uint32_t bits = mw[c];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float dv[2];
#pragma unroll
              for (int z = 0; z < 2; ++z) {
                float pv = ex2_approx(fmaf(__uint_as_float(rs[2 * e + z]), p.scale_log2, -lse2));
                if (mode != 0u) pv = ((bits >> (2 * e + z)) & 1u) ? pv : 0.f;
                dv[z] = pv * (__uint_as_float(rp[2 * e + z]) - drow);
              }
              dw[e] = pack_bf16x2(dv[0], dv[1]);
            }
          }
          tmem_st16(tmem + lane_addr + TM_DS + db * 64 + gc * 16, dw);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->ew_full[db]);
      }
      const uint32_t g_last = it + n_tiles - 1;
      mbar_wait(&bars->mma2_done[g_last & 1], (g_last >> 1) & 1, abort_flag);
      __syncwarp();
      tc_fence_after();
      __nv_bfloat16* dst = p.dq + static_cast<int64_t>(b) * p.sb + static_cast<int64_t>(h) * p.sh +
                           static_cast<int64_t>(valid ? a : 0) * p.sn;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col = (D / 2) * wg + 32 * c;  // this warpgroup's half of the dQ row
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + TM_DQ + col, r);
        tmem_wait_ld();
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * p.scale, __uint_as_float(r[2 * e + 1]) * p.scale);
          uint4* o4 = reinterpret_cast<uint4*>(dst + col);
#pragma unroll
          for (int v = 0; v < 4; ++v) o4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
      it += n_tiles;
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
