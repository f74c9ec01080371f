// C ABI of the Radial Attention hot path (declared in include/radial.h).
//
// All device code of the library lives in this one translation unit (the
// kernels are included from the .cuh files beside it), so the shared device
// error word has a single definition.  Host code here only validates,
// allocates the mask's arrays, encodes TMA descriptors and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/radial.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "attn_fwd_pair.cuh"
#include "gemm.cuh"
#include "mask_build.cuh"
#include "sm100_primitives.cuh"

using namespace radial;

namespace radial {
// Failure-detection self-test: one warp waits on an mbarrier that nothing
// will ever complete, with a short limit; the bounded wait must give up,
// set the library's error word and let the kernel return normally.
__global__ void selftest_bounded_wait_kernel(uint64_t limit_ns, int* waited_out) {
  __shared__ uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    abort_s = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_limit(&bar, 0, &abort_s, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0) *waited_out = ok ? 0 : 1;
}

}  // namespace radial

// ---------------------------------------------------------------------------
// errors and instrumentation
// ---------------------------------------------------------------------------
namespace {

thread_local std::string t_last_error;
std::atomic<int64_t> g_launches{0};

radial_status fail(radial_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

#define RADIAL_CUDA(call)                                                                        \
  do {                                                                                           \
    cudaError_t e_ = (call);                                                                     \
    if (e_ != cudaSuccess) {                                                                     \
      return fail(e_ == cudaErrorMemoryAllocation ? RADIAL_ENOMEM : RADIAL_ECUDA, "%s: %s (%s:%d)", \
                  #call, cudaGetErrorString(e_), __FILE__, __LINE__);                            \
    }                                                                                            \
  } while (0)

#define RADIAL_LAUNCHED()                                                                         \
  do {                                                                                            \
    g_launches.fetch_add(1, std::memory_order_relaxed);                                           \
    cudaError_t e_ = cudaGetLastError();                                                          \
    if (e_ != cudaSuccess)                                                                        \
      return fail(RADIAL_ECUDA, "kernel launch: %s (%s:%d)", cudaGetErrorString(e_), __FILE__, __LINE__); \
  } while (0)

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// An NVTX range around each entry point, so that profiler timelines show the
// library's calls by name (no cost unless a profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4D map over a bf16 [B, H, N, D] tensor (D contiguous), box_rows-row x
// 64-column boxes with the 128-byte swizzle; rows past N read as zeros.
radial_status make_bhnd_map(CUtensorMap* map, const void* base, const radial_desc& d, uint32_t box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(RADIAL_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d.head_dim), static_cast<cuuint64_t>(d.n_tokens),
                        static_cast<cuuint64_t>(d.heads), static_cast<cuuint64_t>(d.batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d.stride_n) * 2, static_cast<cuuint64_t>(d.stride_h) * 2,
                           static_cast<cuuint64_t>(d.stride_b) * 2};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RADIAL_ECUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return RADIAL_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// The mask object
// ---------------------------------------------------------------------------
struct TileLists {
  int32_t nb = 0;
  int64_t nnz = 0, n_full = 0;
  int32_t *row_ptr = nullptr, *col_idx = nullptr, *col_ptr = nullptr, *row_idx = nullptr;
  int32_t *row_order = nullptr, *col_order = nullptr;
  uint8_t *kind = nullptr, *kind_t = nullptr;
  void release() {
    cudaFree(row_ptr); cudaFree(col_idx); cudaFree(col_ptr); cudaFree(row_idx);
    cudaFree(row_order); cudaFree(col_order); cudaFree(kind); cudaFree(kind_t);
    *this = TileLists();
  }
};

// Union walk of neighbouring query-tile pairs (2p, 2p+1) of the plan.
struct PairLists {
  int32_t np = 0;
  int64_t nu = 0;
  int32_t *ptr = nullptr, *col = nullptr, *order = nullptr;
  uint8_t* flag = nullptr;
  void release() {
    cudaFree(ptr); cudaFree(col); cudaFree(order); cudaFree(flag);
    *this = PairLists();
  }
};

struct radial_csr {
  int32_t f = 0, s = 0, n = 0, B = 0, sink = 0, dense = 0, device = 0;
  int32_t* hd = nullptr;  // ablation-mask half widths per frame distance (device; nullptr = method's rule)
  int32_t* cd = nullptr;  // ablation-mask sampled-diagonal periods per frame distance
  TileLists user;   // at the caller's block size
  TileLists plan;   // at the kernels' 128-token tile (aliases `user` when B == 128)
  bool plan_owned = false;
  PairLists pairs;  // pairs of plan rows for the two-tile forward
};

namespace {

// From an nb x nb state matrix on the device, build CSR, CSC and orders.
radial_status lists_from_states(const uint8_t* states, int32_t nb, TileLists& L, cudaStream_t st) {
  L.nb = nb;
  int32_t *row_cnt = nullptr, *col_cnt = nullptr;
  unsigned long long* nfull = nullptr;
  RADIAL_CUDA(cudaMalloc(&row_cnt, sizeof(int32_t) * nb));
  RADIAL_CUDA(cudaMalloc(&col_cnt, sizeof(int32_t) * nb));
  RADIAL_CUDA(cudaMalloc(&nfull, sizeof(unsigned long long)));
  RADIAL_CUDA(cudaMalloc(&L.row_ptr, sizeof(int32_t) * (nb + 1)));
  RADIAL_CUDA(cudaMalloc(&L.col_ptr, sizeof(int32_t) * (nb + 1)));
  RADIAL_CUDA(cudaMalloc(&L.row_order, sizeof(int32_t) * nb));
  RADIAL_CUDA(cudaMalloc(&L.col_order, sizeof(int32_t) * nb));
  RADIAL_CUDA(cudaMemsetAsync(col_cnt, 0, sizeof(int32_t) * nb, st));
  RADIAL_CUDA(cudaMemsetAsync(nfull, 0, sizeof(unsigned long long), st));
  count_tiles_kernel<<<nb, 256, 0, st>>>(states, nb, row_cnt, col_cnt, nfull);
  RADIAL_LAUNCHED();
  exclusive_scan_kernel<<<1, 1024, 0, st>>>(row_cnt, nb, L.row_ptr);
  RADIAL_LAUNCHED();
  exclusive_scan_kernel<<<1, 1024, 0, st>>>(col_cnt, nb, L.col_ptr);
  RADIAL_LAUNCHED();
  int32_t nnz32 = 0;
  unsigned long long nf = 0;
  RADIAL_CUDA(cudaMemcpyAsync(&nnz32, L.row_ptr + nb, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  RADIAL_CUDA(cudaMemcpyAsync(&nf, nfull, sizeof(nf), cudaMemcpyDeviceToHost, st));
  RADIAL_CUDA(cudaStreamSynchronize(st));
  L.nnz = nnz32;
  L.n_full = static_cast<int64_t>(nf);
  const size_t m = static_cast<size_t>(nnz32 > 0 ? nnz32 : 1);
  RADIAL_CUDA(cudaMalloc(&L.col_idx, sizeof(int32_t) * m));
  RADIAL_CUDA(cudaMalloc(&L.row_idx, sizeof(int32_t) * m));
  RADIAL_CUDA(cudaMalloc(&L.kind, m));
  RADIAL_CUDA(cudaMalloc(&L.kind_t, m));
  compact_kernel<<<nb, 128, 0, st>>>(states, nb, false, L.row_ptr, L.col_idx, L.kind);
  RADIAL_LAUNCHED();
  compact_kernel<<<nb, 128, 0, st>>>(states, nb, true, L.col_ptr, L.row_idx, L.kind_t);
  RADIAL_LAUNCHED();
  const int rt = 256;
  rank_by_count_kernel<<<(nb + rt - 1) / rt, rt, rt * sizeof(int32_t), st>>>(L.row_ptr, nb, L.row_order);
  RADIAL_LAUNCHED();
  rank_by_count_kernel<<<(nb + rt - 1) / rt, rt, rt * sizeof(int32_t), st>>>(L.col_ptr, nb, L.col_order);
  RADIAL_LAUNCHED();
  RADIAL_CUDA(cudaStreamSynchronize(st));
  cudaFree(row_cnt);
  cudaFree(col_cnt);
  cudaFree(nfull);
  return RADIAL_OK;
}

radial_status pairs_from_plan(const TileLists& P, PairLists& Q, cudaStream_t st) {
  Q.np = (P.nb + 1) / 2;
  int32_t* cnt = nullptr;
  RADIAL_CUDA(cudaMalloc(&cnt, sizeof(int32_t) * Q.np));
  RADIAL_CUDA(cudaMalloc(&Q.ptr, sizeof(int32_t) * (Q.np + 1)));
  RADIAL_CUDA(cudaMalloc(&Q.order, sizeof(int32_t) * Q.np));
  const int t = 128, g = (Q.np + t - 1) / t;
  pair_count_kernel<<<g, t, 0, st>>>(P.row_ptr, P.col_idx, P.kind, P.nb, Q.np, cnt);
  RADIAL_LAUNCHED();
  exclusive_scan_kernel<<<1, 1024, 0, st>>>(cnt, Q.np, Q.ptr);
  RADIAL_LAUNCHED();
  int32_t nu = 0;
  RADIAL_CUDA(cudaMemcpyAsync(&nu, Q.ptr + Q.np, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  RADIAL_CUDA(cudaStreamSynchronize(st));
  Q.nu = nu;
  RADIAL_CUDA(cudaMalloc(&Q.col, sizeof(int32_t) * (nu > 0 ? nu : 1)));
  RADIAL_CUDA(cudaMalloc(&Q.flag, nu > 0 ? nu : 1));
  pair_fill_kernel<<<g, t, 0, st>>>(P.row_ptr, P.col_idx, P.kind, P.nb, Q.np, Q.ptr, Q.col, Q.flag);
  RADIAL_LAUNCHED();
  rank_by_count_kernel<<<(Q.np + 255) / 256, 256, 256 * sizeof(int32_t), st>>>(Q.ptr, Q.np, Q.order);
  RADIAL_LAUNCHED();
  RADIAL_CUDA(cudaStreamSynchronize(st));
  cudaFree(cnt);
  return RADIAL_OK;
}

// Ablation mask rule (see radial_params in radial.h).
struct MaskRule {
  int32_t central_band = 1, num = 2, den = 1, decay = 0;
  bool is_default() const { return central_band == 1 && num == 2 * den && decay == 0; }
};

// h(d), c(d) for d in [0, f) in exact integer arithmetic (128-bit for the
// band boundaries (cb+1) (num/den)^r).  false if the arithmetic would overflow.
bool mask_rule_table(const MaskRule& m, int32_t f, int32_t s, std::vector<int32_t>& H, std::vector<int32_t>& C) {
  typedef unsigned __int128 u128;
  const u128 limit = static_cast<u128>(1) << 120;
  H.assign(f, 0);
  C.assign(f, 1);
  int r = 1;
  u128 P = static_cast<u128>(m.num), Q = static_cast<u128>(m.den);  // num^r, den^r
  for (int32_t d = 0; d < f; ++d) {
    int64_t w;
    int64_t c = 1;
    if (d <= m.central_band) {
      w = s;
    } else if (m.decay == 1) {
      const int64_t e = static_cast<int64_t>(d) - m.central_band + 1;
      w = s / e;
      if (w < 1) c = (e + s - 1) / s;
    } else {
      // advance to the band with dist < (cb+1) sigma^r (bands only grow with d)
      while (!(static_cast<u128>(d) * Q < static_cast<u128>(m.central_band + 1) * P)) {
        P *= static_cast<u128>(m.num);
        Q *= static_cast<u128>(m.den);
        ++r;
        if (P > limit || Q > limit) return false;
      }
      const u128 sQ = static_cast<u128>(s) * Q;
      w = static_cast<int64_t>(sQ / P);
      if (w < 1) {
        const u128 cc = (P + sQ - 1) / sQ;
        c = cc > static_cast<u128>(0x7fffffff) ? 0x7fffffff : static_cast<int64_t>(cc);
      }
    }
    H[d] = static_cast<int32_t>(w - 1);
    C[d] = static_cast<int32_t>(c);
  }
  return true;
}

radial_status build_mask(int32_t f, int32_t s, int32_t B, int32_t sink, int32_t dense, const MaskRule& rule,
                         radial_csr** out, cudaStream_t st) {
  const int64_t n64 = static_cast<int64_t>(f) * s;
  if (n64 > (1LL << 30)) return fail(RADIAL_EINVAL, "frames * tokens_per_frame = %lld exceeds 2^30", (long long)n64);
  const int32_t n = static_cast<int32_t>(n64);
  const int32_t nb = (n + B - 1) / B;
  if (nb > 32768) return fail(RADIAL_EUNSUPPORTED, "%d blocks per side exceeds 32768", nb);
  radial_csr* c = new (std::nothrow) radial_csr();
  if (!c) return fail(RADIAL_ENOMEM, "host allocation failed");
  c->f = f; c->s = s; c->n = n; c->B = B; c->sink = sink; c->dense = dense;
  {
    const cudaError_t e = cudaGetDevice(&c->device);
    if (e != cudaSuccess) {
      delete c;
      return fail(RADIAL_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    }
  }
  if (!rule.is_default()) {
    std::vector<int32_t> H, C;
    if (!mask_rule_table(rule, f, s, H, C)) {
      delete c;
      return fail(RADIAL_EUNSUPPORTED, "band table of width scale %d/%d overflows 128-bit arithmetic", rule.num,
                  rule.den);
    }
    if (cudaMalloc(&c->hd, sizeof(int32_t) * f) != cudaSuccess || cudaMalloc(&c->cd, sizeof(int32_t) * f) != cudaSuccess) {
      cudaFree(c->hd);
      cudaFree(c->cd);
      delete c;
      return fail(RADIAL_ENOMEM, "cannot allocate the distance table");
    }
    cudaMemcpy(c->hd, H.data(), sizeof(int32_t) * f, cudaMemcpyHostToDevice);
    cudaMemcpy(c->cd, C.data(), sizeof(int32_t) * f, cudaMemcpyHostToDevice);
  }
  uint8_t* states = nullptr;
  uint8_t* states128 = nullptr;
  radial_status rs = RADIAL_OK;
  auto cleanup = [&](radial_status r) {
    cudaStreamSynchronize(st);
    cudaFree(states);
    cudaFree(states128);
    if (r != RADIAL_OK) {
      c->pairs.release();
      if (c->plan_owned) c->plan.release();
      c->user.release();
      cudaFree(c->hd);
      cudaFree(c->cd);
      delete c;
    }
    return r;
  };
  if (cudaMalloc(&states, static_cast<size_t>(nb) * nb) != cudaSuccess)
    return cleanup(fail(RADIAL_ENOMEM, "cannot allocate %d x %d tile states", nb, nb));
  MaskGeom g{f, s, n, B, nb, sink, c->hd, c->cd};
  dim3 grid((nb + 127) / 128, nb);
  classify_tiles_kernel<<<grid, 128, 0, st>>>(g, states);
  g_launches.fetch_add(1);
  if (cudaGetLastError() != cudaSuccess) return cleanup(fail(RADIAL_ECUDA, "classify_tiles launch failed"));
  rs = lists_from_states(states, nb, c->user, st);
  if (rs != RADIAL_OK) return cleanup(rs);
  if (B == 128) {
    c->plan = c->user;
    c->plan_owned = false;
  } else {
    const int32_t nt = (n + 127) / 128;
    if (cudaMalloc(&states128, static_cast<size_t>(nt) * nt) != cudaSuccess)
      return cleanup(fail(RADIAL_ENOMEM, "cannot allocate %d x %d tile plan", nt, nt));
    dim3 g2((nt + 127) / 128, nt);
    coarsen_states_kernel<<<g2, 128, 0, st>>>(states, nb, states128, nt);
    g_launches.fetch_add(1);
    if (cudaGetLastError() != cudaSuccess) return cleanup(fail(RADIAL_ECUDA, "coarsen launch failed"));
    c->plan_owned = true;
    rs = lists_from_states(states128, nt, c->plan, st);
    if (rs != RADIAL_OK) return cleanup(rs);
  }
  rs = pairs_from_plan(c->plan, c->pairs, st);
  if (rs != RADIAL_OK) return cleanup(rs);
  *out = c;
  return cleanup(RADIAL_OK);
}

}  // namespace

// ---------------------------------------------------------------------------
// ABI
// ---------------------------------------------------------------------------
extern "C" {

void radial_params_default(radial_params* p) {
  if (!p) return;
  std::memset(p, 0, sizeof(*p));
  p->sink = 1;
  p->central_band = 1;
  p->width_scale_num = 2;
  p->width_scale_den = 1;
  p->decay = 0;
}

radial_status radial_mask_build(int32_t frames, int32_t tokens_per_frame, int32_t block,
                                const radial_params* params, radial_csr** out, void* stream) {
  NvtxRange nvtx_range("radial_mask_build");
  if (!out) return fail(RADIAL_EINVAL, "out is NULL");
  *out = nullptr;
  radial_params def;
  radial_params_default(&def);
  const radial_params* pr = params ? params : &def;
  for (int i = 0; i < 3; ++i)
    if (pr->reserved[i] != 0) return fail(RADIAL_EINVAL, "params.reserved[%d] must be 0", i);
  if (pr->sink != 0 && pr->sink != 1) return fail(RADIAL_EINVAL, "params.sink must be 0 or 1");
  if (pr->central_band < 0 || pr->central_band > (1 << 20))
    return fail(RADIAL_EINVAL, "params.central_band must be in [0, 2^20]");
  if (pr->width_scale_num < 1 || pr->width_scale_num > 64 || pr->width_scale_den < 1 || pr->width_scale_den > 64 ||
      pr->width_scale_num <= pr->width_scale_den)
    return fail(RADIAL_EINVAL, "width scale num/den must be in [1, 64] with num > den");
  if (pr->decay != 0 && pr->decay != 1) return fail(RADIAL_EINVAL, "params.decay must be 0 (radial) or 1 (harmonic)");
  MaskRule rule;
  rule.central_band = pr->central_band;
  rule.num = pr->width_scale_num;
  rule.den = pr->width_scale_den;
  rule.decay = pr->decay;
  if (frames < 1 || tokens_per_frame < 1) return fail(RADIAL_EINVAL, "frames and tokens_per_frame must be >= 1");
  if (block != 64 && block != 128) return fail(RADIAL_EUNSUPPORTED, "block must be 64 or 128");
  return build_mask(frames, tokens_per_frame, block, pr->sink, 0, rule, out, as_stream(stream));
}

radial_status radial_mask_build_dense(int32_t n_tokens, int32_t block, radial_csr** out, void* stream) {
  NvtxRange nvtx_range("radial_mask_build_dense");
  if (!out) return fail(RADIAL_EINVAL, "out is NULL");
  *out = nullptr;
  if (n_tokens < 1) return fail(RADIAL_EINVAL, "n_tokens must be >= 1");
  if (block != 64 && block != 128) return fail(RADIAL_EUNSUPPORTED, "block must be 64 or 128");
  // One frame of n tokens: distance 0 everywhere, so every pair is allowed.
  return build_mask(1, n_tokens, block, 0, 1, MaskRule(), out, as_stream(stream));
}

radial_status radial_csr_info(const radial_csr* c, radial_csr_info_t* info) {
  if (!c || !info) return fail(RADIAL_EINVAL, "NULL argument");
  std::memset(info, 0, sizeof(*info));
  info->frames = c->f;
  info->tokens_per_frame = c->s;
  info->n_tokens = c->n;
  info->block = c->B;
  info->n_blocks = c->user.nb;
  info->sink = c->sink;
  info->dense = c->dense;
  info->nnz = c->user.nnz;
  info->n_full = c->user.n_full;
  return RADIAL_OK;
}

radial_status radial_csr_copy_to_host(const radial_csr* c, int32_t* row_ptr, int32_t* col_idx,
                                      uint8_t* kind, int32_t* col_ptr, int32_t* row_idx,
                                      uint8_t* kind_t, int32_t* row_order, int32_t* col_order) {
  NvtxRange nvtx_range("radial_csr_copy_to_host");
  if (!c) return fail(RADIAL_EINVAL, "csr is NULL");
  const TileLists& L = c->user;
  const size_t nb = static_cast<size_t>(L.nb), nnz = static_cast<size_t>(L.nnz);
  if (row_ptr) RADIAL_CUDA(cudaMemcpy(row_ptr, L.row_ptr, 4 * (nb + 1), cudaMemcpyDeviceToHost));
  if (col_ptr) RADIAL_CUDA(cudaMemcpy(col_ptr, L.col_ptr, 4 * (nb + 1), cudaMemcpyDeviceToHost));
  if (col_idx) RADIAL_CUDA(cudaMemcpy(col_idx, L.col_idx, 4 * nnz, cudaMemcpyDeviceToHost));
  if (row_idx) RADIAL_CUDA(cudaMemcpy(row_idx, L.row_idx, 4 * nnz, cudaMemcpyDeviceToHost));
  if (kind) RADIAL_CUDA(cudaMemcpy(kind, L.kind, nnz, cudaMemcpyDeviceToHost));
  if (kind_t) RADIAL_CUDA(cudaMemcpy(kind_t, L.kind_t, nnz, cudaMemcpyDeviceToHost));
  if (row_order) RADIAL_CUDA(cudaMemcpy(row_order, L.row_order, 4 * nb, cudaMemcpyDeviceToHost));
  if (col_order) RADIAL_CUDA(cudaMemcpy(col_order, L.col_order, 4 * nb, cudaMemcpyDeviceToHost));
  return RADIAL_OK;
}

void radial_csr_free(radial_csr* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  cudaFree(c->hd);
  cudaFree(c->cd);
  c->pairs.release();
  if (c->plan_owned) c->plan.release();
  c->user.release();
  delete c;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// attention validation shared by forward and backward
// ---------------------------------------------------------------------------
namespace {

radial_status check_desc(const radial_csr* c, const radial_desc* d) {
  if (!c || !d) return fail(RADIAL_EINVAL, "NULL csr or desc");
  if (d->batch < 1 || d->heads < 1) return fail(RADIAL_EINVAL, "batch and heads must be >= 1");
  if (d->n_tokens != c->n) return fail(RADIAL_EINVAL, "desc.n_tokens %d != mask n %d", d->n_tokens, c->n);
  if (d->head_dim != 64 && d->head_dim != 128) return fail(RADIAL_EUNSUPPORTED, "head_dim must be 64 or 128");
  if (d->reserved != 0) return fail(RADIAL_EINVAL, "desc.reserved must be 0");
  if (d->stride_n < d->head_dim || d->stride_h < 1 || d->stride_b < 1)
    return fail(RADIAL_EINVAL, "strides must cover head_dim");
  if ((d->stride_n * 2) % 16 || (d->stride_h * 2) % 16 || (d->stride_b * 2) % 16)
    return fail(RADIAL_EINVAL, "strides * 2 bytes must be multiples of 16");
  if (static_cast<int64_t>(d->batch) * d->heads * ((d->n_tokens + 127) / 128) > 0x7fffffffLL)
    return fail(RADIAL_EUNSUPPORTED, "too many work items");
  int dev = 0;
  RADIAL_CUDA(cudaGetDevice(&dev));
  if (dev != c->device) return fail(RADIAL_EINVAL, "mask built on device %d, current device %d", c->device, dev);
  return RADIAL_OK;
}

float softmax_scale(const radial_desc* d) {
  return d->scale > 0.f ? d->scale : 1.0f / std::sqrt(static_cast<float>(d->head_dim));
}

// Work items run head-major and, inside a head, longest row (column) first:
// the order arrays built with the mask.  It balances the tail of each launch.
template <int D>
radial_status launch_fwd_pair(const radial_csr* c, const radial_desc* d, const void* q, const void* k,
                              const void* v, void* o, float* lse, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  radial_status rs;
  if ((rs = make_bhnd_map(&mq, q, *d)) != RADIAL_OK) return rs;
  if ((rs = make_bhnd_map(&mk, k, *d)) != RADIAL_OK) return rs;
  if ((rs = make_bhnd_map(&mv, v, *d)) != RADIAL_OK) return rs;
  FwdPairParams p;
  p.pair_ptr = c->pairs.ptr;
  p.pair_col = c->pairs.col;
  p.pair_flag = c->pairs.flag;
  p.pair_order = c->pairs.order;
  p.hd = c->hd;
  p.cd = c->cd;
  p.np = c->pairs.np;
  p.nt = c->plan.nb;
  p.f = c->f;
  p.s = c->s;
  p.n = c->n;
  p.sink = c->sink;
  p.heads = d->heads;
  p.items = d->batch * d->heads * c->pairs.np;
  p.o_sb = d->stride_b;
  p.o_sh = d->stride_h;
  p.o_sn = d->stride_n;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.scale_log2 = softmax_scale(d) * 1.4426950408889634f;
  const int smem = FwdPairCfg<D>::SMEM_BYTES;
  const int grid = p.items < sm_count() ? p.items : sm_count();
  RADIAL_CUDA(cudaFuncSetAttribute(radial_fwd_pair_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  radial_fwd_pair_kernel<D><<<grid, 384, smem, st>>>(mq, mk, mv, p);
  RADIAL_LAUNCHED();
  return RADIAL_OK;
}

template <int D>
radial_status launch_bwd(const radial_csr* c, const radial_desc* d, const void* dout, const void* q,
                         const void* k, const void* v, const void* o, const float* lse, void* dq, void* dk,
                         void* dv, float* dr, cudaStream_t st) {
  // Everything that can fail on the host (tensor maps, kernel attributes)
  // happens before the first launch: a call that returns an error has
  // launched nothing and left the workspace untouched.
  CUtensorMap mq, mk, mv, mdo;
  radial_status rs;
  if ((rs = make_bhnd_map(&mq, q, *d)) != RADIAL_OK) return rs;
  if ((rs = make_bhnd_map(&mk, k, *d)) != RADIAL_OK) return rs;
  if ((rs = make_bhnd_map(&mv, v, *d)) != RADIAL_OK) return rs;
  if ((rs = make_bhnd_map(&mdo, dout, *d)) != RADIAL_OK) return rs;
  const int smem = BwdCfg<D>::SMEM_BYTES, smem_dq = BwdCfg<D>::DQ_SMEM_BYTES;
  RADIAL_CUDA(cudaFuncSetAttribute(radial_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  RADIAL_CUDA(cudaFuncSetAttribute(radial_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq));
  const int64_t rows = static_cast<int64_t>(d->batch) * d->heads * d->n_tokens;
  {
    const int threads = 256;
    const int64_t blocks = (rows * 16 + threads - 1) / threads;
    bwd_rowdot_kernel<D><<<static_cast<unsigned>(blocks), threads, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(dout), reinterpret_cast<const __nv_bfloat16*>(o), d->heads,
        d->n_tokens, d->stride_b, d->stride_h, d->stride_n, rows, dr);
    RADIAL_LAUNCHED();
  }
  BwdParams p;
  p.row_ptr = c->plan.row_ptr;
  p.col_idx = c->plan.col_idx;
  p.kind = c->plan.kind;
  p.row_order = c->plan.row_order;
  p.col_ptr = c->plan.col_ptr;
  p.row_idx = c->plan.row_idx;
  p.kind_t = c->plan.kind_t;
  p.col_order = c->plan.col_order;
  p.hd = c->hd;
  p.cd = c->cd;
  p.nt = c->plan.nb;
  p.f = c->f;
  p.s = c->s;
  p.n = c->n;
  p.sink = c->sink;
  p.heads = d->heads;
  p.items = d->batch * d->heads * c->plan.nb;
  p.sb = d->stride_b;
  p.sh = d->stride_h;
  p.sn = d->stride_n;
  p.lse = lse;
  p.dr = dr;
  p.dq = reinterpret_cast<__nv_bfloat16*>(dq);
  p.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  p.scale = softmax_scale(d);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  const int grid = p.items < sm_count() ? p.items : sm_count();
  radial_bwd_dkdv_kernel<D><<<grid, 384, smem, st>>>(mq, mk, mv, mdo, p);
  RADIAL_LAUNCHED();
  radial_bwd_dq_kernel<D><<<grid, 384, smem_dq, st>>>(mq, mk, mv, mdo, p);
  RADIAL_LAUNCHED();
  return RADIAL_OK;
}

}  // namespace

extern "C" {

radial_status radial_attn_fwd(const radial_csr* c, const radial_desc* d, const void* q, const void* k,
                              const void* v, void* o, float* lse, void* stream) {
  NvtxRange nvtx_range("radial_attn_fwd");
  radial_status rs = check_desc(c, d);
  if (rs != RADIAL_OK) return rs;
  if (!q || !k || !v || !o || !lse) return fail(RADIAL_EINVAL, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return fail(RADIAL_EINVAL, "tensor pointers must be 16-byte aligned");
  if (d->head_dim == 128) return launch_fwd_pair<128>(c, d, q, k, v, o, lse, as_stream(stream));
  return launch_fwd_pair<64>(c, d, q, k, v, o, lse, as_stream(stream));
}

size_t radial_attn_bwd_workspace_size(const radial_desc* d) {
  if (!d || d->batch < 1 || d->heads < 1 || d->n_tokens < 1 || d->head_dim < 1) return 0;
  const size_t rows = static_cast<size_t>(d->batch) * d->heads * d->n_tokens;
  return (rows * sizeof(float) + 255) & ~size_t(255);
}

radial_status radial_attn_bwd(const radial_csr* c, const radial_desc* d, const void* dout, const void* q,
                              const void* k, const void* v, const void* o, const float* lse, void* dq,
                              void* dk, void* dv, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("radial_attn_bwd");
  radial_status rs = check_desc(c, d);
  if (rs != RADIAL_OK) return rs;
  if (!dout || !q || !k || !v || !o || !lse || !dq || !dk || !dv || !workspace)
    return fail(RADIAL_EINVAL, "NULL tensor or workspace pointer");
  if (!aligned16(dout) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(RADIAL_EINVAL, "tensor pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(RADIAL_EINVAL, "workspace must be 256-byte aligned");
  if (workspace_bytes < radial_attn_bwd_workspace_size(d))
    return fail(RADIAL_EINVAL, "workspace of %zu bytes is below the %zu required", workspace_bytes,
                radial_attn_bwd_workspace_size(d));
  if (d->head_dim == 128)
    return launch_bwd<128>(c, d, dout, q, k, v, o, lse, dq, dk, dv, static_cast<float*>(workspace),
                           as_stream(stream));
  return launch_bwd<64>(c, d, dout, q, k, v, o, lse, dq, dk, dv, static_cast<float*>(workspace),
                        as_stream(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward of host-resident tensors with the copies overlapped
// ---------------------------------------------------------------------------
namespace {

constexpr int kMaxStageGroups = 64;

// Per device: a copy-in and a copy-out stream and the events that order the
// groups of one call (created on first use, kept until exit).
struct StageResources {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in_done[kMaxStageGroups] = {}, comp_done[kMaxStageGroups] = {};
};
std::mutex g_stage_mu;
StageResources g_stage[64];

radial_status stage_resources(StageResources** out) {
  int dev = 0;
  RADIAL_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(RADIAL_EUNSUPPORTED, "device index %d beyond 63", dev);
  std::lock_guard<std::mutex> lock(g_stage_mu);
  StageResources& r = g_stage[dev];
  if (!r.in) {
    RADIAL_CUDA(cudaStreamCreateWithFlags(&r.in, cudaStreamNonBlocking));
    RADIAL_CUDA(cudaStreamCreateWithFlags(&r.out, cudaStreamNonBlocking));
    RADIAL_CUDA(cudaEventCreateWithFlags(&r.start, cudaEventDisableTiming));
    RADIAL_CUDA(cudaEventCreateWithFlags(&r.done, cudaEventDisableTiming));
    for (int i = 0; i < kMaxStageGroups; ++i) {
      RADIAL_CUDA(cudaEventCreateWithFlags(&r.in_done[i], cudaEventDisableTiming));
      RADIAL_CUDA(cudaEventCreateWithFlags(&r.comp_done[i], cudaEventDisableTiming));
    }
  }
  *out = &r;
  return RADIAL_OK;
}

// Copy heads [h0, h1) of batch entry b of one bf16 [B, H, N, D] tensor.
radial_status copy_heads(void* dst, const void* src, const radial_desc& d, int b, int h0, int h1, cudaMemcpyKind kind,
                         cudaStream_t st) {
  const int64_t off = static_cast<int64_t>(b) * d.stride_b + static_cast<int64_t>(h0) * d.stride_h;
  char* dp = static_cast<char*>(dst) + 2 * off;
  const char* sp = static_cast<const char*>(src) + 2 * off;
  if (d.stride_n == d.head_dim && d.stride_h == static_cast<int64_t>(d.n_tokens) * d.head_dim) {
    // heads of one batch entry are one contiguous block
    RADIAL_CUDA(cudaMemcpyAsync(dp, sp, static_cast<size_t>(h1 - h0) * d.stride_h * 2, kind, st));
    return RADIAL_OK;
  }
  for (int h = h0; h < h1; ++h) {
    const int64_t ho = static_cast<int64_t>(h - h0) * d.stride_h * 2;
    RADIAL_CUDA(cudaMemcpy2DAsync(dp + ho, d.stride_n * 2, sp + ho, d.stride_n * 2, static_cast<size_t>(d.head_dim) * 2,
                                  static_cast<size_t>(d.n_tokens), kind, st));
  }
  return RADIAL_OK;
}

}  // namespace

extern "C" radial_status radial_attn_fwd_staged(const radial_csr* c, const radial_desc* d, const void* q_host,
                                                const void* k_host, const void* v_host, void* o_host,
                                                float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                                                float* lse_dev, int32_t chunks, void* stream) {
  NvtxRange nvtx_range("radial_attn_fwd_staged");
  radial_status rs = check_desc(c, d);
  if (rs != RADIAL_OK) return rs;
  if (!q_host || !k_host || !v_host || !o_host || !lse_host || !q_dev || !k_dev || !v_dev || !o_dev || !lse_dev)
    return fail(RADIAL_EINVAL, "NULL tensor pointer");
  if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(v_dev) || !aligned16(o_dev) || !aligned16(lse_dev))
    return fail(RADIAL_EINVAL, "device tensor pointers must be 16-byte aligned");
  if (chunks < 1) return fail(RADIAL_EINVAL, "chunks must be >= 1");
  const int per_b = std::min(chunks, d->heads);
  const int64_t groups = static_cast<int64_t>(d->batch) * per_b;
  if (groups > kMaxStageGroups)
    return fail(RADIAL_EUNSUPPORTED, "batch * chunks = %lld exceeds %d groups", (long long)groups, kMaxStageGroups);
  {
    // the maps of every group are subsets of these: if they encode, so do
    // the groups', and no failure can come after the first copy
    CUtensorMap probe;
    if ((rs = make_bhnd_map(&probe, q_dev, *d)) != RADIAL_OK) return rs;
    if ((rs = make_bhnd_map(&probe, k_dev, *d)) != RADIAL_OK) return rs;
    if ((rs = make_bhnd_map(&probe, v_dev, *d)) != RADIAL_OK) return rs;
  }
  StageResources* R = nullptr;
  if ((rs = stage_resources(&R)) != RADIAL_OK) return rs;
  cudaStream_t st = as_stream(stream);
  // nothing on `stream` before this call may still be using the device buffers
  RADIAL_CUDA(cudaEventRecord(R->start, st));
  RADIAL_CUDA(cudaStreamWaitEvent(R->in, R->start, 0));
  RADIAL_CUDA(cudaStreamWaitEvent(R->out, R->start, 0));
  // Head groups of one batch entry.  The first group's copy-in and the last
  // group's copy-out overlap no attention, so with three or more groups those
  // two are small and the groups between them grow: weights 1, 2, 4, 4, ...,
  // 4 and 1 for the last, rounded to whole heads with at least one per group.
  std::vector<int> bound(per_b + 1, 0);
  {
    std::vector<int64_t> cw(per_b);
    int64_t W = 0;
    for (int k = 0; k < per_b; ++k) {
      const int64_t w = (per_b <= 2 || k == per_b - 1) ? 1 : (int64_t(1) << std::min(k, 2));
      W += w;
      cw[k] = W;
    }
    for (int k = 0; k < per_b; ++k) {
      int x = static_cast<int>((static_cast<int64_t>(d->heads) * cw[k] + W / 2) / W);
      x = std::max(x, bound[k] + 1);
      x = std::min(x, d->heads - (per_b - 1 - k));
      bound[k + 1] = x;
    }
    bound[per_b] = d->heads;
  }
  int g = 0;
  for (int b = 0; b < d->batch; ++b) {
    for (int k = 0; k < per_b; ++k, ++g) {
      const int h0 = bound[k], h1 = bound[k + 1];
      // copy in
      if ((rs = copy_heads(q_dev, q_host, *d, b, h0, h1, cudaMemcpyHostToDevice, R->in)) != RADIAL_OK) return rs;
      if ((rs = copy_heads(k_dev, k_host, *d, b, h0, h1, cudaMemcpyHostToDevice, R->in)) != RADIAL_OK) return rs;
      if ((rs = copy_heads(v_dev, v_host, *d, b, h0, h1, cudaMemcpyHostToDevice, R->in)) != RADIAL_OK) return rs;
      RADIAL_CUDA(cudaEventRecord(R->in_done[g], R->in));
      // attention of this group on the caller's stream
      RADIAL_CUDA(cudaStreamWaitEvent(st, R->in_done[g], 0));
      radial_desc sub = *d;
      sub.batch = 1;
      sub.heads = h1 - h0;
      const int64_t off = static_cast<int64_t>(b) * d->stride_b + static_cast<int64_t>(h0) * d->stride_h;
      const int64_t loff = (static_cast<int64_t>(b) * d->heads + h0) * d->n_tokens;
      const char* qp = static_cast<const char*>(q_dev) + 2 * off;
      const char* kp = static_cast<const char*>(k_dev) + 2 * off;
      const char* vp = static_cast<const char*>(v_dev) + 2 * off;
      char* op = static_cast<char*>(o_dev) + 2 * off;
      rs = d->head_dim == 128 ? launch_fwd_pair<128>(c, &sub, qp, kp, vp, op, lse_dev + loff, st)
                              : launch_fwd_pair<64>(c, &sub, qp, kp, vp, op, lse_dev + loff, st);
      if (rs != RADIAL_OK) return rs;
      RADIAL_CUDA(cudaEventRecord(R->comp_done[g], st));
      // copy out
      RADIAL_CUDA(cudaStreamWaitEvent(R->out, R->comp_done[g], 0));
      if ((rs = copy_heads(o_host, o_dev, *d, b, h0, h1, cudaMemcpyDeviceToHost, R->out)) != RADIAL_OK) return rs;
      RADIAL_CUDA(cudaMemcpyAsync(lse_host + loff, lse_dev + loff, sizeof(float) * (h1 - h0) * d->n_tokens,
                                  cudaMemcpyDeviceToHost, R->out));
    }
  }
  RADIAL_CUDA(cudaEventRecord(R->done, R->out));
  RADIAL_CUDA(cudaStreamWaitEvent(st, R->done, 0));
  return RADIAL_OK;
}

// ---------------------------------------------------------------------------
// Backward without any allocation: the row-sum scratch lives in a fixed
// device array of this module instead of a caller-provided workspace.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocMaxRows = size_t(1) << 22;  // 4,194,304 fp32 row sums = 16 MiB
}  // namespace

// Loaded with the module on every device that uses the library; held until exit.
static __device__ __align__(256) float g_noalloc_rowsum[kNoAllocMaxRows];

namespace {
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[64] = {};

// Device address of g_noalloc_rowsum on the current device, looked up once per
// device (the host-side name of the array is not a device address).
radial_status noalloc_scratch(float** out) {
  int dev = 0;
  RADIAL_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(RADIAL_EUNSUPPORTED, "device index %d beyond 63", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* addr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_rowsum);
    if (e != cudaSuccess || !addr)
      return fail(RADIAL_ECUDA, "cudaGetSymbolAddress of the row-sum scratch: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = static_cast<float*>(addr);
  }
  *out = g_noalloc_ptr[dev];
  return RADIAL_OK;
}
}  // namespace

extern "C" {

radial_status radial_attn_bwd_noalloc(const radial_csr* c, const radial_desc* d, const void* dout,
                                      const void* q, const void* k, const void* v, const void* o,
                                      const float* lse, void* dq, void* dk, void* dv, void* stream) {
  NvtxRange nvtx_range("radial_attn_bwd_noalloc");
  radial_status rs = check_desc(c, d);
  if (rs != RADIAL_OK) return rs;
  if (!dout || !q || !k || !v || !o || !lse || !dq || !dk || !dv)
    return fail(RADIAL_EINVAL, "NULL tensor pointer");
  if (!aligned16(dout) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(RADIAL_EINVAL, "tensor pointers must be 16-byte aligned");
  const size_t rows = static_cast<size_t>(d->batch) * d->heads * d->n_tokens;
  if (rows > kNoAllocMaxRows)
    return fail(RADIAL_EUNSUPPORTED,
                "batch * heads * n_tokens = %zu exceeds the %zu rows of the fixed scratch of "
                "radial_attn_bwd_noalloc; use radial_attn_bwd with a workspace",
                rows, kNoAllocMaxRows);
  float* scratch = nullptr;
  if ((rs = noalloc_scratch(&scratch)) != RADIAL_OK) return rs;
  if (d->head_dim == 128)
    return launch_bwd<128>(c, d, dout, q, k, v, o, lse, dq, dk, dv, scratch, as_stream(stream));
  return launch_bwd<64>(c, d, dout, q, k, v, o, lse, dq, dk, dv, scratch, as_stream(stream));
}

radial_status radial_device_status(void* stream) {
  NvtxRange nvtx_range("radial_device_status");
  RADIAL_CUDA(cudaStreamSynchronize(as_stream(stream)));
  int flag = 0;
  RADIAL_CUDA(cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(int)));
  if (flag != 0) {
    const int zero = 0;
    RADIAL_CUDA(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)));
    if (flag == kErrBounds)
      return fail(RADIAL_EDEVICE, "a kernel read an out-of-range index from the mask's arrays (code %d)", flag);
    if (flag == kErrLayout)
      return fail(RADIAL_EDEVICE, "a kernel found its dynamic shared memory misaligned and did nothing (code %d)", flag);
    return fail(RADIAL_EDEVICE, "a kernel aborted after a bounded wait ran out (code %d)", flag);
  }
  RADIAL_CUDA(cudaGetLastError());
  return RADIAL_OK;
}

radial_status radial_selftest_bounded_wait(uint32_t limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000) return fail(RADIAL_EINVAL, "limit_ms must be in [1, 2000]");
  int* flag = nullptr;
  RADIAL_CUDA(cudaMalloc(&flag, sizeof(int)));
  selftest_bounded_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(limit_ms) * 1000000ull, flag);
  g_launches.fetch_add(1);
  cudaError_t e = cudaGetLastError();
  int h = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, flag, sizeof(int), cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  cudaFree(flag);
  if (e != cudaSuccess) return fail(RADIAL_ECUDA, "self-test: %s", cudaGetErrorString(e));
  if (h != 1) return fail(RADIAL_ECUDA, "self-test: the wait did not time out");
  return RADIAL_OK;
}

const char* radial_status_str(radial_status s) {
  switch (s) {
    case RADIAL_OK: return "ok";
    case RADIAL_EINVAL: return "invalid argument";
    case RADIAL_EUNSUPPORTED: return "unsupported";
    case RADIAL_ENOMEM: return "out of memory";
    case RADIAL_ECUDA: return "CUDA error";
    case RADIAL_EDEVICE: return "device-side abort";
  }
  return "unknown status";
}

const char* radial_last_error(void) { return t_last_error.c_str(); }

int64_t radial_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// LoRA-adapted projections (the fine-tuning layer step around the attention)
// ---------------------------------------------------------------------------
namespace {

// 2D map over a bf16 row-major [rows, cols] matrix with row stride ld
// (elements): 64-column x 128-row boxes, 128-byte swizzle; outside reads 0.
radial_status make_rowmajor_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                                uint32_t box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(RADIAL_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RADIAL_ECUDA, "cuTensorMapEncodeTiled (gemm operand) failed (%d)", static_cast<int>(r));
  return RADIAL_OK;
}

// One operand pair of a GEMM segment: A [M, K] and B [N, K], both K-major.
struct GemmSeg {
  const void* a;
  int64_t lda;
  const void* b;
  int64_t ldb;
  int64_t k;  // 0: no segment
};

template <int BN>
radial_status launch_gemm_bn(int64_t M, int64_t N, const GemmSeg& s0, const GemmSeg& s1, float alpha, float beta,
                             void* c, float* acc, int64_t ldc, int max_splits, cudaStream_t st) {
  CUtensorMap a0, b0, a1, b1;
  radial_status rs;
  if ((rs = make_rowmajor_map(&a0, s0.a, M, s0.k, s0.lda)) != RADIAL_OK) return rs;
  if ((rs = make_rowmajor_map(&b0, s0.b, N, s0.k, s0.ldb, BN)) != RADIAL_OK) return rs;
  if (s1.k > 0) {
    if ((rs = make_rowmajor_map(&a1, s1.a, M, s1.k, s1.lda)) != RADIAL_OK) return rs;
    if ((rs = make_rowmajor_map(&b1, s1.b, N, s1.k, s1.ldb, BN)) != RADIAL_OK) return rs;
  } else {
    a1 = a0;
    b1 = b0;
  }
  GemmParams p;
  p.M = static_cast<int32_t>(M);
  p.N = static_cast<int32_t>(N);
  p.kb0 = static_cast<int32_t>((s0.k + 63) / 64);
  p.kb_total = p.kb0 + static_cast<int32_t>((s1.k + 63) / 64);
  p.tiles_m = static_cast<int32_t>((M + 127) / 128);
  p.tiles_n = static_cast<int32_t>((N + BN - 1) / BN);
  const int tiles = p.tiles_m * p.tiles_n;
  int splits = 1;
  if (acc) {  // split K until the grid fills the device
    splits = std::max(1, std::min({max_splits, p.kb_total, (sm_count() + tiles - 1) / tiles}));
  }
  p.kb_per_split = (p.kb_total + splits - 1) / splits;
  p.splits = (p.kb_total + p.kb_per_split - 1) / p.kb_per_split;  // every slice non-empty
  p.items = tiles * p.splits;
  p.alpha = alpha;
  p.beta = beta;
  p.c = reinterpret_cast<__nv_bfloat16*>(c);
  p.acc = acc;
  p.ldc = ldc;
  RADIAL_CUDA(cudaFuncSetAttribute(radial_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   GemmCfg<BN>::SMEM_BYTES));
  const int grid = p.items < sm_count() ? p.items : sm_count();
  radial_gemm_kernel<BN><<<grid, 256, GemmCfg<BN>::SMEM_BYTES, st>>>(a0, b0, a1, b1, p);
  RADIAL_LAUNCHED();
  return RADIAL_OK;
}

// C[M, N] = alpha (A0 B0^T + A1 B1^T) + beta C (bf16 c) or acc += ... (fp32,
// split over K into up to `max_splits` slices).  Encodes every map first.
// Output tiles are 128 x 256 when N is wider than 128 (half the MMA
// instructions and A re-reads of 128 x 128 tiles), else 128 x 128.
radial_status launch_gemm(int64_t M, int64_t N, const GemmSeg& s0, const GemmSeg& s1, float alpha, float beta,
                          void* c, float* acc, int64_t ldc, int max_splits, cudaStream_t st) {
  if (N > 128) return launch_gemm_bn<256>(M, N, s0, s1, alpha, beta, c, acc, ldc, max_splits, st);
  return launch_gemm_bn<128>(M, N, s0, s1, alpha, beta, c, acc, ldc, max_splits, st);
}

radial_status launch_transpose(const void* in, int64_t ld_in, int64_t R, int64_t Cc, void* out, int64_t ld_out,
                               cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((Cc + 63) / 64), static_cast<unsigned>((R + 63) / 64));
  transpose_bf16_kernel<<<grid, dim3(32, 8), 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(in), ld_in,
                                                      static_cast<int>(R), static_cast<int>(Cc),
                                                      reinterpret_cast<__nv_bfloat16*>(out), ld_out);
  RADIAL_LAUNCHED();
  return RADIAL_OK;
}

int64_t pad8(int64_t x) { return (x + 7) & ~int64_t(7); }
size_t pad256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of radial_lora_bwd, carved in this order.
struct LoraWs {
  size_t wt, bt, at, v, vt, xt, dyt, ut, dA, dB, total;
};
LoraWs lora_ws(int64_t n, int64_t ci, int64_t co, int64_t r) {
  const int64_t ln = pad8(n);
  LoraWs w;
  size_t o = 0;
  w.wt = o; o += pad256(2 * ci * co);
  w.bt = o; o += pad256(2 * r * co);
  w.at = o; o += pad256(2 * ci * r);
  w.v = o; o += pad256(2 * n * r);
  w.vt = o; o += pad256(2 * r * ln);
  w.xt = o; o += pad256(2 * ci * ln);
  w.dyt = o; o += pad256(2 * co * ln);
  w.ut = o; o += pad256(2 * r * ln);
  w.dA = o; o += pad256(4 * r * ci);
  w.dB = o; o += pad256(4 * co * r);
  w.total = o;
  return w;
}

radial_status check_lora(int64_t n, int32_t ci, int32_t co, int32_t r, int64_t ld1, int64_t ld2) {
  if (n < 1 || ci < 1 || co < 1 || r < 1) return fail(RADIAL_EINVAL, "sizes must be >= 1");
  if (n > 0x7fffffffLL) return fail(RADIAL_EUNSUPPORTED, "n_tokens beyond 2^31 - 1");
  if (ci % 8 || co % 8 || r % 8) return fail(RADIAL_EINVAL, "c_in, c_out and rank must be multiples of 8");
  if (ld1 % 8 || ld2 % 8) return fail(RADIAL_EINVAL, "row strides must be multiples of 8 elements");
  return RADIAL_OK;
}

}  // namespace

extern "C" {

radial_status radial_lora_fwd(int64_t n, int32_t c_in, int32_t c_out, int32_t rank, float scale, const void* x,
                              int64_t ldx, const void* W, const void* A, const void* B, void* y, int64_t ldy,
                              void* u, void* stream) {
  NvtxRange nvtx_range("radial_lora_fwd");
  radial_status rs = check_lora(n, c_in, c_out, rank, ldx, ldy);
  if (rs != RADIAL_OK) return rs;
  if (!x || !W || !A || !B || !y || !u) return fail(RADIAL_EINVAL, "NULL pointer");
  if (!aligned16(x) || !aligned16(W) || !aligned16(A) || !aligned16(B) || !aligned16(y) || !aligned16(u))
    return fail(RADIAL_EINVAL, "pointers must be 16-byte aligned");
  if (ldx < c_in || ldy < c_out) return fail(RADIAL_EINVAL, "row strides must cover the rows");
  cudaStream_t st = as_stream(stream);
  // u = s x A^T  [n, r]
  GemmSeg none{nullptr, 0, nullptr, 0, 0};
  if ((rs = launch_gemm(n, rank, GemmSeg{x, ldx, A, c_in, c_in}, none, scale, 0.f, u, nullptr, rank, 1, st)) !=
      RADIAL_OK)
    return rs;
  // y = x W^T + u B^T  [n, c_out]
  return launch_gemm(n, c_out, GemmSeg{x, ldx, W, c_in, c_in}, GemmSeg{u, rank, B, rank, rank}, 1.f, 0.f, y,
                     nullptr, ldy, 1, st);
}

size_t radial_lora_bwd_workspace_size(int64_t n, int32_t c_in, int32_t c_out, int32_t rank) {
  if (n < 1 || c_in < 1 || c_out < 1 || rank < 1) return 0;
  return lora_ws(n, c_in, c_out, rank).total;
}

radial_status radial_lora_bwd(int64_t n, int32_t c_in, int32_t c_out, int32_t rank, float scale, const void* dy,
                              int64_t lddy, const void* x, int64_t ldx, const void* W, const void* A, const void* B,
                              const void* u, void* dx, int64_t lddx, int32_t accumulate_dx, void* dA, void* dB,
                              void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("radial_lora_bwd");
  radial_status rs = check_lora(n, c_in, c_out, rank, lddy, ldx);
  if (rs != RADIAL_OK) return rs;
  if (lddx % 8) return fail(RADIAL_EINVAL, "row strides must be multiples of 8 elements");
  if (!dy || !x || !W || !A || !B || !u || !dx || !dA || !dB || !workspace)
    return fail(RADIAL_EINVAL, "NULL pointer");
  if (!aligned16(dy) || !aligned16(x) || !aligned16(W) || !aligned16(A) || !aligned16(B) || !aligned16(u) ||
      !aligned16(dx) || !aligned16(dA) || !aligned16(dB))
    return fail(RADIAL_EINVAL, "pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(RADIAL_EINVAL, "workspace must be 256-byte aligned");
  if (lddy < c_out || ldx < c_in || lddx < c_in) return fail(RADIAL_EINVAL, "row strides must cover the rows");
  if (accumulate_dx != 0 && accumulate_dx != 1) return fail(RADIAL_EINVAL, "accumulate_dx must be 0 or 1");
  const LoraWs w = lora_ws(n, c_in, c_out, rank);
  if (workspace_bytes < w.total)
    return fail(RADIAL_EINVAL, "workspace of %zu bytes is below the %zu required", workspace_bytes, w.total);
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t ln = pad8(n);
  void* Wt = ws + w.wt;
  void* Bt = ws + w.bt;
  void* At = ws + w.at;
  void* v = ws + w.v;
  void* vt = ws + w.vt;
  void* xt = ws + w.xt;
  void* dyt = ws + w.dyt;
  void* ut = ws + w.ut;
  float* dA32 = reinterpret_cast<float*>(ws + w.dA);
  float* dB32 = reinterpret_cast<float*>(ws + w.dB);
  GemmSeg none{nullptr, 0, nullptr, 0, 0};
  // operands in the orientation the GEMM reads (K contiguous)
  if ((rs = launch_transpose(W, c_in, c_out, c_in, Wt, c_out, st)) != RADIAL_OK) return rs;    // W^T [ci, co]
  if ((rs = launch_transpose(B, rank, c_out, rank, Bt, c_out, st)) != RADIAL_OK) return rs;    // B^T [r, co]
  if ((rs = launch_transpose(A, c_in, rank, c_in, At, rank, st)) != RADIAL_OK) return rs;      // A^T [ci, r]
  // v = s dy B  [n, r]
  if ((rs = launch_gemm(n, rank, GemmSeg{dy, lddy, Bt, c_out, c_out}, none, scale, 0.f, v, nullptr, rank, 1, st)) !=
      RADIAL_OK)
    return rs;
  // dx (+)= dy W + v A  [n, ci]
  if ((rs = launch_gemm(n, c_in, GemmSeg{dy, lddy, Wt, c_out, c_out}, GemmSeg{v, rank, At, rank, rank}, 1.f,
                        accumulate_dx ? 1.f : 0.f, dx, nullptr, lddx, 1, st)) != RADIAL_OK)
    return rs;
  // dA = v^T x  [r, ci] and dB = dy^T u  [co, r]: contractions over all n tokens, split over K
  if ((rs = launch_transpose(v, rank, n, rank, vt, ln, st)) != RADIAL_OK) return rs;
  if ((rs = launch_transpose(x, ldx, n, c_in, xt, ln, st)) != RADIAL_OK) return rs;
  if ((rs = launch_transpose(dy, lddy, n, c_out, dyt, ln, st)) != RADIAL_OK) return rs;
  if ((rs = launch_transpose(u, rank, n, rank, ut, ln, st)) != RADIAL_OK) return rs;
  RADIAL_CUDA(cudaMemsetAsync(dA32, 0, sizeof(float) * rank * c_in, st));
  RADIAL_CUDA(cudaMemsetAsync(dB32, 0, sizeof(float) * c_out * rank, st));
  if ((rs = launch_gemm(rank, c_in, GemmSeg{vt, ln, xt, ln, n}, none, 1.f, 0.f, nullptr, dA32, c_in, 64, st)) !=
      RADIAL_OK)
    return rs;
  if ((rs = launch_gemm(c_out, rank, GemmSeg{dyt, ln, ut, ln, n}, none, 1.f, 0.f, nullptr, dB32, rank, 64, st)) !=
      RADIAL_OK)
    return rs;
  const int64_t na = static_cast<int64_t>(rank) * c_in, nb = static_cast<int64_t>(c_out) * rank;
  f32_to_bf16_kernel<<<static_cast<unsigned>((na + 255) / 256), 256, 0, st>>>(dA32, reinterpret_cast<__nv_bfloat16*>(dA), na);
  RADIAL_LAUNCHED();
  f32_to_bf16_kernel<<<static_cast<unsigned>((nb + 255) / 256), 256, 0, st>>>(dB32, reinterpret_cast<__nv_bfloat16*>(dB), nb);
  RADIAL_LAUNCHED();
  return RADIAL_OK;
}

}  // extern "C"
