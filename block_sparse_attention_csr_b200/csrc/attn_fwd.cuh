// Forward-pass definitions shared by the attention kernels: the parameter
// block of the forward, and the element mask of PARTIAL tiles.
//
// The forward computes O = softmax(Q K^T * scale + M) V and LSE per query row
// (the sparse-attention equation Eq.2 of the Radial Attention review,
// jaehun.me §3) over the active 128x128 tiles of the mask's CSR only (§4.2:
// the method runs block-wise on 128x128 token blocks).  The mask's
// element-level pattern is applied on PARTIAL tiles only: each softmax
// thread derives the allowed key columns of its query row from the frame
// segments the key tile spans (row_mask_bits below), and warps skip or keep
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
__device__ __forceinline__ void row_mask_bits(const RowMaskGeom& p, int i, int k, int b0,
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

}  // namespace radial
