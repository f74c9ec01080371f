// Dense bf16 GEMM on tcgen05 for the LoRA-adapted projections around the
// attention (the Radial Attention review on jaehun.me, §4.3: LoRA adapters on
// the Q/K/V/O projections are what the length-extension fine-tuning trains).
//
//   C[M, N] = alpha * sum_seg A_seg[M, K_seg] B_seg[N, K_seg]^T  (+ beta * C)
//
// Both operands of every segment are K-major (row-major with K contiguous).
// Two K segments let one pass compute y = x W^T + u B^T, i.e. the frozen
// projection and the low-rank update into the same accumulator.  Output is
// bf16 (optionally beta * the old value added, for dx summed over the q, k,
// v projections), or an fp32 accumulate-add used by split-K (the adapter
// gradients contract over all tokens).
//
// Tiles of 128 x BN outputs (BN = 256 for wide outputs, 128 otherwise), K in
// blocks of 64 (one 128-byte swizzle box); a persistent grid walks (M tile,
// N tile, K split) items.
// Warp roles (256 threads): warp 0 TMA producer (4-stage ring of A and B
// boxes); warp 1 TMEM allocation and single-thread MMA issue (M = 128,
// N = BN) into one of two accumulators (so the epilogue of one item overlaps
// the next item's MMAs);
// warps 4-7 the epilogue, one thread per output row (TMEM lane).
// Rows or columns past M, N read as zeros (TMA) and are not stored; K past a
// segment's end reads as zeros.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100_primitives.cuh"

namespace radial {

struct GemmParams {
  int32_t M, N;
  int32_t kb0;       // 64-wide K blocks of segment 0
  int32_t kb_total;  // of both segments
  int32_t tiles_m, tiles_n, splits, kb_per_split;
  int32_t items;     // tiles_m * tiles_n * splits
  float alpha, beta;
  __nv_bfloat16* c;  // bf16 output (acc == nullptr)
  float* acc;        // fp32 accumulate-add output (split-K)
  int64_t ldc;       // elements
};

template <int BN>
struct GemmCfg {
  static_assert(BN == 128 || BN == 256, "output tile width");
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = 128 * 64 * 2;  // 128 rows x 64 K, bf16
  static constexpr int B_BYTES = BN * 64 * 2;   // BN rows x 64 K
  static constexpr int SMEM_A = 0;
  static constexpr int SMEM_B = STAGES * A_BYTES;
  static constexpr int SMEM_BAR = SMEM_B + STAGES * B_BYTES;
  static constexpr int SMEM_BYTES = SMEM_BAR + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulators
};

struct GemmBars {
  uint64_t full[4], empty[4];
  uint64_t acc_full[2], acc_empty[2], mma_done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(GemmBars) <= 256, "gemm barrier area");

template <int BN>
__global__ void __launch_bounds__(256, 1)
    radial_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                       const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem + C::SMEM_A;
  uint8_t* sB = smem + C::SMEM_B;
  GemmBars* bars = reinterpret_cast<GemmBars*>(smem + C::SMEM_BAR);
  volatile int* abort_flag = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    bars->abort = 0;
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->acc_full[i], 1);
      mbar_init(&bars->acc_empty[i], 128);
    }
    mbar_init(&bars->mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // K blocks [kb_begin, kb_end) of an item
  auto item_range = [&](int item, int& tm, int& tn, int& kb_begin, int& kb_end) {
    const int split = item % p.splits;
    const int tile = item / p.splits;
    tm = tile / p.tiles_n;
    tn = tile - tm * p.tiles_n;
    kb_begin = split * p.kb_per_split;
    kb_end = min(p.kb_total, kb_begin + p.kb_per_split);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA0);
      tma_prefetch_desc(&tmB0);
      if (p.kb_total > p.kb0) {
        tma_prefetch_desc(&tmA1);
        tma_prefetch_desc(&tmB1);
      }
      uint32_t kc = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.items; item += gridDim.x) {
        int tm, tn, kb0, kb1;
        item_range(item, tm, tn, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++kc) {
          const uint32_t st = kc % C::STAGES, use = kc / C::STAGES;
          if (use > 0 && !mbar_wait(&bars->empty[st], (use - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->full[st], C::A_BYTES + C::B_BYTES);
          const bool seg0 = kb < p.kb0;
          const int kx = (seg0 ? kb : kb - p.kb0) * 64;
          tma_load_2d(sA + st * C::A_BYTES, seg0 ? &tmA0 : &tmA1, &bars->full[st], kx, tm * 128);
          tma_load_2d(sB + st * C::B_BYTES, seg0 ? &tmB0 : &tmB1, &bars->full[st], kx, tn * BN);
        }
      }
      for (uint32_t x = (kc > C::STAGES ? kc - C::STAGES : 0); x < kc; ++x)
        mbar_wait_drain(&bars->full[x % C::STAGES], (x / C::STAGES) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, false);
      constexpr uint64_t kBoxA = C::A_BYTES >> 4, kBoxB = C::B_BYTES >> 4;
      const uint64_t dA0 = smem_desc(smem_u32(sA), 16, 1024, kSwizzle128B);
      const uint64_t dB0 = smem_desc(smem_u32(sB), 16, 1024, kSwizzle128B);
      uint32_t kc = 0, item_i = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.items; item += gridDim.x, ++item_i) {
        int tm, tn, kb0, kb1;
        item_range(item, tm, tn, kb0, kb1);
        const uint32_t ab = item_i & 1;
        if (item_i >= 2 && !mbar_wait(&bars->acc_empty[ab], ((item_i >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        for (int kb = kb0; kb < kb1; ++kb, ++kc) {
          const uint32_t st = kc % C::STAGES;
          if (!mbar_wait(&bars->full[st], (kc / C::STAGES) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + ab * BN, dA0 + st * kBoxA + ((kk * 32) >> 4), dB0 + st * kBoxB + ((kk * 32) >> 4), idesc,
                   (kb > kb0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars->empty[st]);
        }
        mma_commit(&bars->acc_full[ab]);
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t item_i = 0;
    for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++item_i) {
      int tm, tn, kb0, kb1;
      item_range(item, tm, tn, kb0, kb1);
      const uint32_t ab = item_i & 1;
      const bool waited = mbar_wait(&bars->acc_full[ab], (item_i >> 1) & 1, abort_flag);
      __syncwarp();
      tc_fence_after();
      const int row = tm * 128 + quarter * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + ab * BN + c * 32, r);
        tmem_wait_ld();
        const int col0 = tn * BN + c * 32;
        if (!waited || row >= p.M || col0 >= p.N) continue;
        if (p.acc) {
          float* dst = p.acc + static_cast<int64_t>(row) * p.ldc + col0;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (col0 + e < p.N) atomicAdd(dst + e, p.alpha * __uint_as_float(r[e]));
        } else {
          __nv_bfloat16* dst = p.c + static_cast<int64_t>(row) * p.ldc + col0;
#pragma unroll
          for (int g = 0; g < 4; ++g) {  // groups of 8 columns (N is a multiple of 8)
            if (col0 + 8 * g >= p.N) break;
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = p.alpha * __uint_as_float(r[8 * g + e]);
            if (p.beta != 0.f) {
              const uint4 old = *reinterpret_cast<const uint4*>(dst + 8 * g);
              const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&old);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 of = __bfloat1622float2(o2[e]);
                v[2 * e] += p.beta * of.x;
                v[2 * e + 1] += p.beta * of.y;
              }
            }
            *reinterpret_cast<uint4*>(dst + 8 * g) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                                pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// out[c, r] = in[r, c] for a bf16 [R, Cc] matrix (row strides in elements).
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* __restrict__ in, int64_t ld_in,
                                                            int R, int Cc, __nv_bfloat16* __restrict__ out,
                                                            int64_t ld_out) {
  // 64 x 64 tiles moved as bf16 pairs: every warp access is a whole 128-byte
  // line.  Rows of 66 bf16 (33 words) keep the column reads at two-way bank
  // conflicts.  Pairs need even column offsets, which the callers' leading
  // dimensions and column counts (multiples of 8) give; ragged edges fall
  // back to single elements.
  __shared__ __align__(16) __nv_bfloat16 tile[64][66];
  const int c0 = blockIdx.x * 64, r0 = blockIdx.y * 64;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int y = ty + 8 * k, r = r0 + y, c = c0 + 2 * tx;
    if (r < R) {
      const __nv_bfloat16* src = in + static_cast<int64_t>(r) * ld_in + c;
      if (c + 1 < Cc) {
        *reinterpret_cast<__nv_bfloat162*>(&tile[y][2 * tx]) = *reinterpret_cast<const __nv_bfloat162*>(src);
      } else if (c < Cc) {
        tile[y][2 * tx] = src[0];
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int y = ty + 8 * k, c = c0 + y, r = r0 + 2 * tx;  // output row c, output columns r, r + 1
    if (c < Cc) {
      __nv_bfloat16* dst = out + static_cast<int64_t>(c) * ld_out + r;
      if (r + 1 < R) {
        __nv_bfloat162 v;
        v.x = tile[2 * tx][y];
        v.y = tile[2 * tx + 1][y];
        *reinterpret_cast<__nv_bfloat162*>(dst) = v;
      } else if (r < R) {
        dst[0] = tile[2 * tx][y];
      }
    }
  }
}

// out (bf16) = in (fp32), n elements.
__global__ void f32_to_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = __float2bfloat16_rn(in[i]);
}

}  // namespace radial
