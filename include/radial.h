/*
 * radial.h -- C ABI of the B200 (sm_100a) Radial Attention hot path.
 *
 * The operation: masked softmax attention O = softmax(Q K^T * scale + M) V
 * (the sparse-attention equation, Eq.2, of "Paper review: Radial Attention:
 * O(n log n) Sparse Attention with Energy Decay for Long Video Generation",
 * jaehun.me, §3), where M is the static spatiotemporal radial mask of that
 * page's §4.2 (temporal bands, Fig.5a; shrinking spatial diagonal, Fig.5b;
 * the 4D mask Eq.4 flattened to 2D; the attention sink of App. A.1 Eq.8),
 * executed block-sparsely over the active tiles of a block CSR (§4.2: the
 * implementation computes in 128x128 token blocks).  The backward pass is
 * the one the LoRA length-extension fine-tuning of §4.3 needs.
 *
 * Mask reading (the printed formulas were lost; the plain reading, which
 * reproduces the page's worked toy example exactly): tokens a = i*s + k
 * (frame i, row-major position k), b = j*s + l, d = |i - j|,
 * r = floor(log2(max(d,1))), h = floor(s / 2^r) - 1, c = ceil(2^r / s);
 * (a, b) is allowed iff (sink and j == 0) or (h >= 0 and |k - l| <= h) or
 * (h < 0 and d mod c == 0 and k == l).
 *
 * Conventions shared by every call
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) unless its comment says otherwise.
 *  - All arguments are validated on the host before anything is launched; a
 *    call that returns an error has launched nothing.
 *  - No exception crosses the ABI.  CUDA failures map to RADIAL_ECUDA; the
 *    text of the last error on the calling thread is radial_last_error().
 *  - Kernels never wait without bound: a producer/consumer wait that exceeds
 *    its limit (about 2 s) aborts the kernel and records RADIAL_EDEVICE,
 *    which radial_device_status() reports (and clears).
 *  - The caller owns every tensor and workspace buffer; the library owns a
 *    radial_csr from its build call until radial_csr_free().
 */
#ifndef RADIAL_H_
#define RADIAL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum radial_status {
  RADIAL_OK = 0,
  RADIAL_EINVAL = 1,        /* invalid argument: null, misaligned, inconsistent sizes */
  RADIAL_EUNSUPPORTED = 2,  /* well-formed but outside what the kernels implement */
  RADIAL_ENOMEM = 3,        /* a device or host allocation failed */
  RADIAL_ECUDA = 4,         /* a CUDA runtime or driver call failed */
  RADIAL_EDEVICE = 5        /* a kernel aborted after a bounded wait ran out (or, in
                               the bounds-checking debug build, read an out-of-range
                               index from the mask's arrays; or found its dynamic
                               shared memory too misaligned for its layout and did
                               nothing) */
} radial_status;

/* Mask parameters.  sink: 1 = every query also attends to all tokens of frame
 * 0 (App. A.1 Eq.8; default 1).  The remaining fields select the ablation
 * variants of the authors' responses (paperhub.cn: "width of central band",
 * "width scale between consecutive bands") and of the review's App. C.3
 * (harmonic-series decay); their formulas are not printed, the readings are:
 *  central_band (>= 0, default 1): frame distances <= it are dense.
 *  width_scale_num / width_scale_den (sigma = num/den, 1 < sigma, both in
 *    [1, 64], default 2/1): radial decay puts distance dist > cb in band r >= 1
 *    with (cb+1) sigma^(r-1) <= dist < (cb+1) sigma^r and keeps
 *    |k - l| <= floor(s / sigma^r) - 1.
 *  decay (0 radial = the method, default; 1 harmonic): harmonic keeps
 *    |k - l| <= floor(s / (dist - cb + 1)) - 1.
 *  In both decays a width of 0 keeps only k == l, in every c-th frame pair,
 *  c = ceil(sigma^r / s) (radial) or ceil((dist - cb + 1) / s) (harmonic).
 * The defaults reproduce the method's mask exactly.  reserved: must be zero. */
typedef struct radial_params {
  int32_t sink;
  int32_t central_band;
  int32_t width_scale_num;
  int32_t width_scale_den;
  int32_t decay;
  int32_t reserved[3];
} radial_params;

/* Fill *p with the defaults {sink 1, central_band 1, width scale 2/1, decay radial}. */
void radial_params_default(radial_params* p);

/* Opaque block-sparse mask: the block CSR and CSC of active tiles plus the
 * kernels' schedules, all in device memory owned by the library. */
typedef struct radial_csr radial_csr;

typedef struct radial_csr_info_t {
  int32_t frames;            /* f */
  int32_t tokens_per_frame;  /* s */
  int32_t n_tokens;          /* n = f * s */
  int32_t block;             /* B: tile edge in tokens */
  int32_t n_blocks;          /* ceil(n / B): q-blocks = k-blocks */
  int32_t sink;
  int32_t dense;             /* 1 if built by radial_mask_build_dense */
  int32_t reserved;
  int64_t nnz;               /* active tiles */
  int64_t n_full;            /* active tiles with every pair allowed */
  int64_t allowed_pairs;     /* reserved: 0 (not computed by the builder) */
} radial_csr_info_t;

/* Build the block CSR of the radial mask for f frames of s tokens with square
 * B x B tiles (§4.2: block-wise execution).  A tile (qb, kb) is ACTIVE iff it
 * holds at least one allowed pair of tokens < n; FULL (kind 1) iff both
 * blocks lie inside [0, n) and every pair in it is allowed; else PARTIAL
 * (kind 2).  Columns of a row are ascending; the CSC lists, per key block,
 * its active query blocks ascending; row_order / col_order list blocks by
 * active-tile count descending, ties by index ascending.
 * Runs on the device on `stream` and SYNCHRONISES it (the tile count sizes the
 * allocation).  Constraints: f >= 1, s >= 1, f*s <= 2^30, B in {64, 128},
 * ceil(n/B) <= 32768.  On success *out owns device memory until
 * radial_csr_free.  params NULL selects the defaults.  Errors: RADIAL_EINVAL
 * (bad sizes, null out, out-of-range or non-zero reserved parameters),
 * RADIAL_EUNSUPPORTED (other B; a width scale whose band table would
 * overflow 128-bit arithmetic), RADIAL_ENOMEM, RADIAL_ECUDA. */
radial_status radial_mask_build(int32_t frames, int32_t tokens_per_frame, int32_t block,
                                const radial_params* params, radial_csr** out, void* stream);

/* The all-ones mask of n tokens (dense attention, Eq.1 of the same page, run
 * through the same kernels): every tile active, FULL except tail tiles.  It
 * is the dense comparator and the dense-layer / dense-warm-up mode the
 * authors use in their first layers and steps.  Same contract as
 * radial_mask_build. */
radial_status radial_mask_build_dense(int32_t n_tokens, int32_t block, radial_csr** out,
                                      void* stream);

/* Sizes of a built mask.  Host only; no device work. */
radial_status radial_csr_info(const radial_csr* csr, radial_csr_info_t* info);

/* Copy the mask to host arrays (each may be NULL to skip it).  Sizes:
 * row_ptr, col_ptr: n_blocks + 1 int32; col_idx, row_idx: nnz int32;
 * kind, kind_t: nnz uint8 (1 FULL, 2 PARTIAL; kind_t in CSC order);
 * row_order, col_order: n_blocks int32.  Synchronous (blocks the host). */
radial_status radial_csr_copy_to_host(const radial_csr* csr, int32_t* row_ptr, int32_t* col_idx,
                                      uint8_t* kind, int32_t* col_ptr, int32_t* row_idx,
                                      uint8_t* kind_t, int32_t* row_order, int32_t* col_order);

/* Release a mask (waits for the device to be done with it).  NULL is a no-op. */
void radial_csr_free(radial_csr* csr);

/* Shape and layout of the attention tensors.  Q, K, V, O, dO, dQ, dK, dV are
 * bf16 [batch, heads, n_tokens, head_dim] with head_dim contiguous and the
 * element strides given here (shared by all eight tensors); every base
 * pointer and stride * 2 bytes must be 16-byte aligned.  LSE is fp32
 * [batch, heads, n_tokens], contiguous.  head_dim in {64, 128}.
 * scale: softmax scale; <= 0 selects 1/sqrt(head_dim) (Eq.1's scaling). */
typedef struct radial_desc {
  int32_t batch;
  int32_t heads;
  int32_t n_tokens;
  int32_t head_dim;
  int64_t stride_b;
  int64_t stride_h;
  int64_t stride_n;
  float scale;
  int32_t reserved;
} radial_desc;

/* Forward (Eq.2 under the mask): writes O (bf16, rows normalised) and
 * LSE = ln(sum_b exp(scale * q.k_b)) over allowed keys (fp32, natural log) for
 * every (batch, head, token).  The same mask serves every batch entry and
 * head (it depends on positions only, §4.2).  desc->n_tokens must equal the
 * mask's n.  Reads q, k, v; writes o, lse; no workspace; asynchronous. */
radial_status radial_attn_fwd(const radial_csr* csr, const radial_desc* desc, const void* q,
                              const void* k, const void* v, void* o, float* lse, void* stream);

/* Forward of host-resident tensors with the copies overlapped: the same
 * result as copying Q, K, V to the device, calling radial_attn_fwd and copying
 * O and LSE back, but the heads of each batch entry are processed in `chunks`
 * groups (at most batch * chunks = 64 groups), and group g's inputs are copied
 * in while group g-1 is computed and group g-1's outputs copied out, on two
 * internal streams per device created on the first call.  The first group's
 * copy-in and the last group's copy-out overlap no attention, so with three
 * or more groups their sizes follow the weights 1, 2, 4, 4, ..., 4 and 1 for
 * the last group (each group at least one head); one or two groups split the
 * heads evenly.  q_host .. lse_host
 * are host buffers, q_dev .. lse_dev caller-owned device buffers of the full
 * shape; host and device tensors share the layout of `desc`.  The host
 * buffers should be page-locked, or the copies cannot overlap.  Work already
 * queued on `stream` completes before the first copy; `stream` then waits
 * for the last one, so a synchronisation of `stream` covers the whole call.
 * All arguments are validated before the first copy; a CUDA error in a copy
 * itself is reported as RADIAL_ECUDA after earlier groups were issued.  Two
 * calls on one device at once share the internal streams and run one after
 * the other.  Asynchronous. */
radial_status radial_attn_fwd_staged(const radial_csr* csr, const radial_desc* desc, const void* q_host,
                                     const void* k_host, const void* v_host, void* o_host, float* lse_host,
                                     void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_dev,
                                     int32_t chunks, void* stream);

/* Bytes of device workspace radial_attn_bwd needs for this shape: one fp32
 * per (batch, head, token) for the row sums rowsum(dO o O), rounded up to
 * 256 bytes.  Returns 0 for a NULL or empty desc.  Host only. */
size_t radial_attn_bwd_workspace_size(const radial_desc* desc);

/* Backward of Eq.2 under the mask (the gradients LoRA fine-tuning, §4.3,
 * back-propagates through attention): given dO, the forward's inputs, its O
 * and LSE, writes dQ, dK, dV (bf16, same layout).  `workspace` is caller-owned
 * device memory of at least radial_attn_bwd_workspace_size(desc) bytes,
 * 256-byte aligned; its contents on entry do not matter and on exit are
 * unspecified.  Asynchronous. */
radial_status radial_attn_bwd(const radial_csr* csr, const radial_desc* desc, const void* dout,
                              const void* q, const void* k, const void* v, const void* o,
                              const float* lse, void* dq, void* dk, void* dv, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Backward for callers that cannot allocate device memory: the same
 * computation as radial_attn_bwd, with no workspace argument.  The paper has
 * no counterpart to this call; it exists for callers that cannot hand the
 * library a workspace: code running in a plugin or callback interface that
 * gives it no allocator, processes whose device memory is entirely reserved by
 * another framework's pool, and latency-critical loops that must not call
 * cudaMalloc because it can synchronise the device.
 * The per-row scratch (one fp32 per (batch, head, token)) is a fixed array in
 * the library's device memory of 4,194,304 floats (16 MiB), which every GPU
 * that loads the library holds until the process exits.  Calls with
 * batch * heads * n_tokens above 4,194,304 return RADIAL_EUNSUPPORTED and launch
 * nothing.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, once per device, with that
 * device current) and keeps it for the life of the process; make that first
 * call before any stream capture, and do not use this call on a device after
 * cudaDeviceReset (the reset unloads the module, and the kept address would
 * then name memory the library no longer owns).  Every
 * call shares the one array per device, which keeps the last call's contents
 * (each call overwrites every row it reads before reading it), so calls that
 * overlap on the GPU, on different streams or threads, race and must be
 * serialised by the caller.  Arguments, layout and errors otherwise as for
 * radial_attn_bwd.  Asynchronous. */
radial_status radial_attn_bwd_noalloc(const radial_csr* csr, const radial_desc* desc, const void* dout,
                                      const void* q, const void* k, const void* v, const void* o,
                                      const float* lse, void* dq, void* dk, void* dv, void* stream);

/* ---- LoRA-adapted projections (the fine-tuning layer step around the attention)
 * The review's §4.3 extends a pretrained video model to longer videos by
 * training LoRA adapters on the Q/K/V/O projections of its attention layers
 * while the attention runs under the radial mask.  One projection is
 *     y = x W^T + s (x A^T) B^T
 * with W [c_out, c_in] frozen and A [rank, c_in], B [c_out, rank] trained;
 * the pages fix nothing else, and this standard form, with no bias, is the
 * reading taken.  All matrices are bf16, row-major with unit column stride;
 * x, y, dy, dx take a row stride (elements), W, A, B, u, dA, dB are
 * contiguous.  c_in, c_out, rank and every row stride must be multiples of 8,
 * every pointer 16-byte aligned.  The GEMMs run on the tensor cores of this
 * library (fp32 accumulation).  Asynchronous on `stream`; errors as above. */

/* Forward: writes y [n, c_out] and u = s x A^T [n, rank] (bf16), which the
 * backward takes back. */
radial_status radial_lora_fwd(int64_t n_tokens, int32_t c_in, int32_t c_out, int32_t rank, float scale,
                              const void* x, int64_t ldx, const void* W, const void* A, const void* B,
                              void* y, int64_t ldy, void* u, void* stream);

/* Bytes of device workspace radial_lora_bwd needs (transposed operands and
 * fp32 accumulators of the adapter gradients).  Host only. */
size_t radial_lora_bwd_workspace_size(int64_t n_tokens, int32_t c_in, int32_t c_out, int32_t rank);

/* Backward for upstream dy [n, c_out]: dx [n, c_in] = dy W + s (dy B) A
 * (added to the existing dx when accumulate_dx is 1, so the q, k and v
 * projections of one input can share a dx), dA [rank, c_in] = s (dy B)^T x
 * and dB [c_out, rank] = dy^T u (u from the forward).  `workspace`:
 * caller-owned device memory of radial_lora_bwd_workspace_size bytes,
 * 256-byte aligned. */
radial_status radial_lora_bwd(int64_t n_tokens, int32_t c_in, int32_t c_out, int32_t rank, float scale,
                              const void* dy, int64_t lddy, const void* x, int64_t ldx, const void* W,
                              const void* A, const void* B, const void* u, void* dx, int64_t lddx,
                              int32_t accumulate_dx, void* dA, void* dB, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Synchronise `stream` and report whether any kernel of this library aborted
 * on a bounded wait since the last call (RADIAL_EDEVICE, then cleared), or a
 * CUDA error is pending (RADIAL_ECUDA).  RADIAL_OK otherwise. */
radial_status radial_device_status(void* stream);

/* Failure-detection self-test: launches one warp that waits on an mbarrier
 * nothing completes, with a wait limit of limit_ms (1..2000) milliseconds.
 * The bounded wait gives up, the kernel returns normally and records the
 * abort, so a following radial_device_status() reports RADIAL_EDEVICE and
 * the context stays usable.  Synchronous.  RADIAL_OK if the wait timed out
 * as designed. */
radial_status radial_selftest_bounded_wait(uint32_t limit_ms, void* stream);

/* Static text for a status code. */
const char* radial_status_str(radial_status s);

/* Text of the last error raised on the calling thread ("" if none). */
const char* radial_last_error(void);

/* Number of kernel launches this library has issued in this process (all
 * threads, all devices).  Host counter, for instrumentation. */
int64_t radial_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* RADIAL_H_ */
