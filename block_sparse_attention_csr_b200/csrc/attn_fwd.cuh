// Forward-pass definitions shared by the attention kernels: the parameter
// block of the forward, and the element mask of PARTIAL tiles.
//
// The forward computes O = softmax(Q K^T * scale + M) V and LSE per query row
// (the sparse-attention equation Eq.2 of the Radial Attention review,
// jaehun.me §3) over the active 128x128 tiles of the mask's CSR only (§4.2:
// the method runs block-wise on 128x128 token blocks).  The mask's
// element-level pattern is applied on PARTIAL tiles only: each softmax
// thread derives the allowed key columns of its query row from the frame
// segments the key tile spans (row_mask64 below), and warps skip or keep
// whole 32-key chunks when every lane agrees (chunk_modes).  The kernel
// itself is in attn_fwd_pair.cuh.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mask_build.cuh"
#include "sm100_primitives.cuh"

namespace radial {

// Geometry the element mask of a query row needs: f frames of s tokens
// (n = f * s), the sink flag, and an ablation mask's per-distance tables
// (nullptr: the method's closed form).
struct RowMaskGeom {
  int32_t f, s, n, sink;
  const int32_t* hd;
  const int32_t* cd;
  uint32_t s_mul;  // floor(x / s) = (x * s_mul) >> s_shift, set by set_divisor
  int32_t s_shift;
};

// Exact division by the frame size with one multiply and one shift
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994, Thm 4.2 with N = 31): with l = ceil(log2 s) and
// m = ceil(2^(31+l) / s) < 2^32, floor(x / s) = floor(x m / 2^(31+l)) for every
// 0 <= x < 2^31.  Computed once per thread; the per-tile divisions then stay
// off the exponential unit (an integer divide or a float reciprocal would
// issue there).
__device__ __forceinline__ void set_divisor(RowMaskGeom& p) {
  int l = 0;
  while (l < 31 && (1u << l) < static_cast<uint32_t>(p.s)) ++l;
  const uint64_t num = (uint64_t(1) << (31 + l)) + static_cast<uint64_t>(p.s) - 1;
  p.s_mul = static_cast<uint32_t>(num / static_cast<uint64_t>(p.s));
  p.s_shift = 31 + l;
}
__device__ __forceinline__ int div_s(const RowMaskGeom& p, int x) {
  return static_cast<int>((static_cast<uint64_t>(static_cast<uint32_t>(x)) * p.s_mul) >> p.s_shift);
}

// Bits [lo, hi] of a 64-bit word, 0 <= lo <= hi <= 63.
__device__ __forceinline__ uint64_t bit_range64(int lo, int hi) {
  return (~0ull >> (63 - hi)) & (~0ull << lo);
}

// Token t = own*s + pos (a query for the row mask, a key for the column mask)
// against the tokens of frame j held by window columns [lo_s, hi_s] (relative
// to b0): the band |pos - pos'| <= h(d), or the sampled diagonal, as bits.
__device__ __forceinline__ uint64_t interval_bits64(const RowMaskGeom& p, int own, int pos, int b0, int j, int lo_s,
                                                    int hi_s) {
  const int d = own > j ? own - j : j - own;
  const int h = half_width_of(p.hd, p.s, d);
  const int center = j * p.s + pos - b0;
  int lo, hi;
  if (h >= 0) {
    lo = max(lo_s, center - h);
    hi = min(hi_s, center + h);
  } else {
    if (d % period_of(p.cd, p.s, d) != 0) return 0ull;
    lo = max(lo_s, center);
    hi = min(hi_s, center);
  }
  return lo <= hi ? bit_range64(lo, hi) : 0ull;
}

// Allowed partners in window [b0, b0 + 64) of token own*s + pos, one word
// (bit c = token b0 + c; tokens at or past n are not allowed).  kKeys = false:
// the token is a query and the window holds keys (the sink is key frame 0);
// kKeys = true: the token is a key and the window holds queries (a key of
// frame 0 is seen by every query).  With s >= 64 the window holds at most two
// frame segments, each one interval.
template <bool kKeys>
__device__ __forceinline__ uint64_t window_mask64(const RowMaskGeom& p, int own, int pos, int b0) {
  const int bend = min(b0 + 64, p.n) - b0;  // columns inside the sequence
  if (bend <= 0) return 0ull;
  if (kKeys && p.sink && own == 0) return bit_range64(0, bend - 1);
  auto seg = [&](int j, int lo_s, int hi_s) -> uint64_t {
    if (!kKeys && p.sink && j == 0) return bit_range64(lo_s, hi_s);
    return interval_bits64(p, own, pos, b0, j, lo_s, hi_s);
  };
  int j = div_s(p, b0);
  if (p.s >= 64) {
    const int e = (j + 1) * p.s - b0;  // first column of frame j + 1
    if (e >= bend) return seg(j, 0, bend - 1);
    return seg(j, 0, e - 1) | seg(j + 1, e, bend - 1);
  }
  uint64_t m = 0ull;
  for (; j * p.s < b0 + bend; ++j) m |= seg(j, max(0, j * p.s - b0), min(bend, (j + 1) * p.s - b0) - 1);
  return m;
}

// Allowed keys [b0, b0 + 64) of query token i*s + k.
__device__ __forceinline__ uint64_t row_mask64(const RowMaskGeom& p, int i, int k, int b0) {
  return window_mask64<false>(p, i, k, b0);
}

// Allowed queries [a0, a0 + 64) of key token j*s + l (the transpose).
__device__ __forceinline__ uint64_t col_mask64(const RowMaskGeom& p, int j, int l, int a0) {
  return window_mask64<true>(p, j, l, a0);
}

// Warp-uniform handling of a thread's two 32-column chunks of a PARTIAL tile:
// 0 = every lane of the warp allows all 32 columns (use S as is), 2 = every
// lane masks all of them (no TMEM read, no select, no exponential: P = 0),
// 1 = mixed (per-element select).  Two bits per chunk.
__device__ __forceinline__ uint32_t chunk_modes(const uint32_t (&mw)[2]) {
  uint32_t modes = 0;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const bool all_ok = __all_sync(0xffffffffu, mw[c] == 0xffffffffu);
    const bool none = __all_sync(0xffffffffu, mw[c] == 0u);
    modes |= (all_ok ? 0u : (none ? 2u : 1u)) << (2 * c);
  }
  return modes;
}

}  // namespace radial
