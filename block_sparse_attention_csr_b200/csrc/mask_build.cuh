// Device builder of the radial mask's block CSR / CSC.
//
// Mask (the Radial Attention review on jaehun.me, §4.2: temporal bands of
// Fig.5a, shrinking spatial diagonal of Fig.5b, 4D mask Eq.4 flattened to 2D,
// attention sink of App. A.1 Eq.8; the toy example fixes the width reading):
// query token a = i*s + k, key token b = j*s + l, d = |i - j|,
// r = floor(log2(max(d, 1))), h = floor(s / 2^r) - 1, c = ceil(2^r / s);
// allowed iff (sink and j == 0) or (h >= 0 and |k - l| <= h)
//          or (h < 0 and d mod c == 0 and k == l).
//
// Blocks (§4.2, block-wise execution): tile (qb, kb) of B x B tokens is
// ACTIVE iff it holds an allowed pair of in-range tokens, FULL iff both
// blocks are inside [0, n) and every pair is allowed, else PARTIAL.
//
// Pipeline: one thread per tile classifies it by splitting both blocks into
// per-frame segments and testing each segment pair as an interval problem
// (closest / farthest |k - l| against h); per-row and per-column counts;
// exclusive scans; order-preserving compaction into CSR and CSC; ranking of
// rows and columns by count for longest-first scheduling.
#pragma once

#include <cstdint>

namespace radial {

constexpr uint8_t kTileFull = 1;
constexpr uint8_t kTilePartial = 2;

struct MaskGeom {
  int32_t f, s, n, B, nb, sink;
  // per-frame-distance half width h(d) and sampled-diagonal period c(d) of an
  // ablation mask; nullptr selects the method's own closed form
  const int32_t* hd;
  const int32_t* cd;
};

// h(d) and c(d): the closed form r = floor(log2 max(d,1)), h = floor(s/2^r)-1,
// c = ceil(2^r/s), or the table of an ablation mask.
// floor(log2 d) for d >= 1 by shifts and compares.  The attention kernels
// evaluate it per PARTIAL tile next to a stream of exponentials; a count of
// leading zeros (like a conversion or a reciprocal) issues at the exponential
// unit's rate of 16 per clock and SM and would queue behind them.
__device__ __forceinline__ int floor_log2(int d) {
  int r = 0;
  if (d >> 16) { d >>= 16; r += 16; }
  if (d >> 8) { d >>= 8; r += 8; }
  if (d >> 4) { d >>= 4; r += 4; }
  if (d >> 2) { d >>= 2; r += 2; }
  return r + (d >> 1);
}
__device__ __forceinline__ int half_width_of(const int32_t* hd, int s, int d) {
  if (hd) return hd[d];
  const int r = floor_log2(d > 1 ? d : 1);
  return (s >> r) - 1;
}
__device__ __forceinline__ long long period_of(const int32_t* cd, int s, int d) {
  if (cd) return cd[d];
  const int r = floor_log2(d > 1 ? d : 1);
  return ((1LL << r) + s - 1) / s;
}

// Segment pair test.  Query positions [k0,k1] of frame i against key positions
// [l0,l1] of frame j.  Sets any / all for "some pair allowed" / "every pair".
__device__ __forceinline__ void segment_pair(const MaskGeom& g, int i, int k0, int k1, int j, int l0,
                                             int l1, bool& any, bool& all) {
  if (g.sink && j == 0) {
    any = true;
    all = true;
    return;
  }
  const int d = i > j ? i - j : j - i;
  const int h = half_width_of(g.hd, g.s, d);
  int gap = l0 - k1;
  if (k0 - l1 > gap) gap = k0 - l1;
  if (gap < 0) gap = 0;
  if (h >= 0) {
    const int span = (k1 - l0) > (l1 - k0) ? (k1 - l0) : (l1 - k0);
    any = gap <= h;
    all = span <= h;
    return;
  }
  const long long period = period_of(g.cd, g.s, d);
  if (d % period == 0) {
    any = gap == 0;
    all = (k0 == k1) && (l0 == l1) && (k0 == l0);
  } else {
    any = false;
    all = false;
  }
}

__device__ uint8_t classify_tile(const MaskGeom& g, int qb, int kb) {
  const int a0 = qb * g.B;
  const int a1 = min(a0 + g.B, g.n);  // exclusive
  const int b0 = kb * g.B;
  const int b1 = min(b0 + g.B, g.n);
  const bool inside = (a0 + g.B <= g.n) && (b0 + g.B <= g.n);
  bool any = false, all = true;
  for (int i = a0 / g.s; i * g.s < a1; ++i) {
    const int k0 = max(a0, i * g.s) - i * g.s;
    const int k1 = min(a1, (i + 1) * g.s) - 1 - i * g.s;
    for (int j = b0 / g.s; j * g.s < b1; ++j) {
      const int l0 = max(b0, j * g.s) - j * g.s;
      const int l1 = min(b1, (j + 1) * g.s) - 1 - j * g.s;
      bool sa, sl;
      segment_pair(g, i, k0, k1, j, l0, l1, sa, sl);
      any |= sa;
      all &= sl;
      if (any && !all) return kTilePartial;
    }
  }
  if (!any) return 0;
  return (all && inside) ? kTileFull : kTilePartial;
}

__global__ void classify_tiles_kernel(MaskGeom g, uint8_t* __restrict__ states) {
  const int kb = blockIdx.x * blockDim.x + threadIdx.x;
  const int qb = blockIdx.y;
  if (kb >= g.nb) return;
  states[static_cast<size_t>(qb) * g.nb + kb] = classify_tile(g, qb, kb);
}

// Coarsen B=64 tile states to 128-token tiles: active if any sub-tile is,
// FULL only if all four sub-tiles exist and are FULL.
__global__ void coarsen_states_kernel(const uint8_t* __restrict__ fine, int nbf,
                                      uint8_t* __restrict__ coarse, int nbc) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (u >= nbc) return;
  bool any = false, all = true;
  for (int dq = 0; dq < 2; ++dq)
    for (int dk = 0; dk < 2; ++dk) {
      const int q = 2 * t + dq, k = 2 * u + dk;
      if (q >= nbf || k >= nbf) {
        all = false;
        continue;
      }
      const uint8_t st = fine[static_cast<size_t>(q) * nbf + k];
      any |= st != 0;
      all &= st == kTileFull;
    }
  coarse[static_cast<size_t>(t) * nbc + u] = any ? (all ? kTileFull : kTilePartial) : 0;
}

// One CTA per row: count active tiles of the row, add each to its column's
// count, and count FULL tiles.
__global__ void count_tiles_kernel(const uint8_t* __restrict__ states, int nb,
                                   int32_t* __restrict__ row_cnt, int32_t* __restrict__ col_cnt,
                                   unsigned long long* __restrict__ n_full) {
  const int r = blockIdx.x;
  int cnt = 0, full = 0;
  for (int c = threadIdx.x; c < nb; c += blockDim.x) {
    const uint8_t st = states[static_cast<size_t>(r) * nb + c];
    if (st) {
      ++cnt;
      atomicAdd(&col_cnt[c], 1);
      full += st == kTileFull;
    }
  }
  __shared__ int s_cnt, s_full;
  if (threadIdx.x == 0) {
    s_cnt = 0;
    s_full = 0;
  }
  __syncthreads();
  for (int o = 16; o > 0; o >>= 1) {
    cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    full += __shfl_xor_sync(0xffffffffu, full, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&s_cnt, cnt);
    atomicAdd(&s_full, full);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    row_cnt[r] = s_cnt;
    atomicAdd(n_full, static_cast<unsigned long long>(s_full));
  }
}

// Exclusive scan of nb counts into ptr[0..nb] by a single CTA of 1024 threads.
__global__ void exclusive_scan_kernel(const int32_t* __restrict__ cnt, int nb,
                                      int32_t* __restrict__ ptr) {
  __shared__ int32_t part[1024];
  const int per = (nb + blockDim.x - 1) / blockDim.x;
  const int beg = min(nb, static_cast<int>(threadIdx.x) * per);
  const int end = min(nb, beg + per);
  int32_t sum = 0;
  for (int i = beg; i < end; ++i) sum += cnt[i];
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int off = 1; off < static_cast<int>(blockDim.x); off <<= 1) {
    int32_t v = threadIdx.x >= static_cast<unsigned>(off) ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int32_t run = part[threadIdx.x] - sum;  // exclusive prefix of this chunk
  for (int i = beg; i < end; ++i) {
    ptr[i] = run;
    run += cnt[i];
  }
  if (threadIdx.x == blockDim.x - 1) ptr[nb] = part[threadIdx.x];
}

// Order-preserving compaction of one row (transpose=false) or one column
// (transpose=true) of the state matrix per CTA of 128 threads.
__global__ void compact_kernel(const uint8_t* __restrict__ states, int nb, bool transpose,
                               const int32_t* __restrict__ ptr, int32_t* __restrict__ idx,
                               uint8_t* __restrict__ kind) {
  const int line = blockIdx.x;
  __shared__ int warp_tot[4];
  int base = ptr[line];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int c0 = 0; c0 < nb; c0 += 128) {
    const int c = c0 + threadIdx.x;
    uint8_t st = 0;
    if (c < nb)
      st = transpose ? states[static_cast<size_t>(c) * nb + line]
                     : states[static_cast<size_t>(line) * nb + c];
    const unsigned ball = __ballot_sync(0xffffffffu, st != 0);
    if (lane == 0) warp_tot[w] = __popc(ball);
    __syncthreads();
    int pre = 0;
    for (int t = 0; t < w; ++t) pre += warp_tot[t];
    const int tot = warp_tot[0] + warp_tot[1] + warp_tot[2] + warp_tot[3];
    if (st) {
      const int pos = base + pre + __popc(ball & ((1u << lane) - 1u));
      idx[pos] = c;
      kind[pos] = st;
    }
    base += tot;
    __syncthreads();
  }
}

// order[rank] = line, ranking by count descending then index ascending.
__global__ void rank_by_count_kernel(const int32_t* __restrict__ ptr, int nb,
                                     int32_t* __restrict__ order) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  extern __shared__ int32_t s_cnt[];
  const int cq = q < nb ? ptr[q + 1] - ptr[q] : 0;
  int rank = 0;
  for (int t0 = 0; t0 < nb; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    s_cnt[threadIdx.x] = t < nb ? ptr[t + 1] - ptr[t] : -1;
    __syncthreads();
    if (q < nb) {
      const int lim = min(static_cast<int>(blockDim.x), nb - t0);
      for (int u = 0; u < lim; ++u) {
        const int cu = s_cnt[u];
        rank += (cu > cq) || (cu == cq && t0 + u < q);
      }
    }
    __syncthreads();
  }
  if (q < nb) order[rank] = q;
}

// ---------------------------------------------------------------------------
// Pair plan: query tiles (2p, 2p+1) processed together by one CTA walk the
// ascending union of their two CSR rows.  Per union entry: the key tile and
// flags (bit 0 / 1: tile 2p / 2p+1 has it; bit 2 / 3: that tile's entry is
// PARTIAL).
// ---------------------------------------------------------------------------
constexpr uint8_t kPairIn0 = 1, kPairIn1 = 2, kPairPart0 = 4, kPairPart1 = 8;

template <bool kFill>
__device__ __forceinline__ int merge_pair(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                                          const uint8_t* __restrict__ kind, int nt, int p,
                                          int32_t* __restrict__ out_col, uint8_t* __restrict__ out_flag) {
  const int t0 = 2 * p, t1 = 2 * p + 1;
  int a = row_ptr[t0], ae = row_ptr[t0 + 1];
  int b = 0, be = 0;
  if (t1 < nt) {
    b = row_ptr[t1];
    be = row_ptr[t1 + 1];
  }
  int n = 0;
  while (a < ae || b < be) {
    const int ca = a < ae ? col_idx[a] : 0x7fffffff;
    const int cb = b < be ? col_idx[b] : 0x7fffffff;
    uint8_t fl = 0;
    int c;
    if (ca <= cb) {
      c = ca;
      fl |= kPairIn0 | (kind[a] != kTileFull ? kPairPart0 : 0);
      ++a;
    } else {
      c = cb;
    }
    if (cb == c) {
      fl |= kPairIn1 | (kind[b] != kTileFull ? kPairPart1 : 0);
      ++b;
    }
    if (kFill) {
      out_col[n] = c;
      out_flag[n] = fl;
    }
    ++n;
  }
  return n;
}

__global__ void pair_count_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                                  const uint8_t* __restrict__ kind, int nt, int np, int32_t* __restrict__ cnt) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= np) return;
  cnt[p] = merge_pair<false>(row_ptr, col_idx, kind, nt, p, nullptr, nullptr);
}

__global__ void pair_fill_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                                 const uint8_t* __restrict__ kind, int nt, int np,
                                 const int32_t* __restrict__ pair_ptr, int32_t* __restrict__ pcol,
                                 uint8_t* __restrict__ pflag) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= np) return;
  merge_pair<true>(row_ptr, col_idx, kind, nt, p, pcol + pair_ptr[p], pflag + pair_ptr[p]);
}

}  // namespace radial
