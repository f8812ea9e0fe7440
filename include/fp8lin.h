/*
 * fp8lin.h -- C ABI of the FP8 linear layer with delayed scaling (sm_100a).
 *
 * Sources: the AstrAI commit logs, cited by the path filter and commit of the
 * page and by the bullet that states the behaviour:
 *   [tests/extension@2eeac02]      ring finalize in the quantize kernel, bias
 *                                  fusion, pre-quantized w8, autograd pair;
 *   [csrc@2eeac02]                 FP8 GEMM kernel history, FP8Params bias;
 *   [astrai/extension/ops@057c0d3] two-primitive API (quantize + mm_fp8),
 *                                  scale snapshot, backward scale reuse;
 *   [astrai@4019dda]               in-kernel fold, fused bias epilogue, dbias
 *                                  only when requested;
 *   [astrai/extension/fp8.py@3e57cc8] amax of raw values, E5M2 gradients.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless marked "host".  The caller allocates
 *     and owns every buffer; the library allocates nothing and keeps no pointer
 *     after a call returns.
 *   - Work is enqueued on `stream` in stream order; no call synchronizes the
 *     host.  A ring (and a workspace) must not be used by two launches that can
 *     run concurrently.
 *   - The library caches a few per-device facts on first use (SM count, the
 *     device address of its status word and of fp8_dbias_noalloc's scratch);
 *     keep one CUDA context per device while it is in use (no
 *     cudaDeviceReset in between).
 *   - Arguments are validated before anything is enqueued.  A failed check
 *     returns a negative fp8_status and enqueues nothing.  A launch failure
 *     returns FP8_ERR_CUDA; fp8_status_string(FP8_ERR_CUDA) then names the CUDA
 *     error.
 *   - Sizes of zero are accepted.  A matrix with no elements is neither read
 *     nor written and its pointer and stride are not checked (NULL is fine):
 *     an empty operand is not quantized and its ring does not step.  An
 *     output that has elements is always written: a GEMM whose contraction
 *     is empty (K = 0 in fp8_mm, N = 0 for dX, M = 0 for dW) writes the bias
 *     alone (zero without one), and dbias over M = 0 rows is zero.
 *   - Matrices are row-major with an explicit row stride `ld` in ELEMENTS.
 *     fp8 matrices (read or written) need ld % 16 == 0 and a 16-byte aligned
 *     base (the GEMMs read them with TMA); bf16/fp16/fp32 inputs may have any
 *     ld >= cols and any element-aligned base.  bf16 outputs need an even-byte
 *     aligned base and ld >= cols.
 */
#ifndef FP8LIN_H
#define FP8LIN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8LIN_API __attribute__((visibility("default")))
#else
#define FP8LIN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fp8_stream_t;  /* = cudaStream_t; NULL = legacy default stream */

typedef enum { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_fmt;

typedef enum {
  FP8_DT_BF16 = 0, FP8_DT_FP16 = 1, FP8_DT_FP32 = 2, FP8_DT_E4M3 = 3, FP8_DT_E5M2 = 4
} fp8_dtype;

typedef enum { FP8_K_MAJOR = 0, FP8_MN_MAJOR = 1 } fp8_major;

/* GEMM output tiles: 128x128 or 128x256 per CTA, or 256x256 per pair of CTAs
 * (2-SM MMA, cluster of 2), or 128x128 tiles each shared by a cluster of S = 2..3
 * CTAs that split K (FP8_TILE_SPLITK_128x128: rank r takes k-blocks
 * [r kb/S, (r+1) kb/S) and rank 0 adds the partial fp32 accumulators in rank
 * order before the epilogue; fp8_mm only -- a two-GEMM launch falls back to
 * 128x128).
 * Stream-K (FP8_TILE_STREAMK, or'ed with FP8_TILE_128x128, FP8_TILE_128x256
 * or FP8_TILE_PAIR_256x256; needs a workspace): one CTA (pair) per SM (pair
 * of SMs); whole waves of tiles run data-parallel and the k-blocks of the
 * remaining tiles are split evenly over the CTAs (pairs), so that no SM idles
 * while others finish a last partial wave.
 * A tile cut between CTAs is finished by the CTA holding its first k-block,
 * which adds the others' fp32 partial accumulators (stored in the workspace)
 * in CTA order: the result is deterministic for a given GPU.
 * FP8_TILE_AUTO chooses per shape with a cost model fitted to B200 timings --
 * split-K when the output has few tiles and K is long; never stream-K, whose
 * fixup latency (flags, then the partials' copies, serialized at the end of
 * the launch) made every stream-K choice of the model slower inside the
 * benchmark steps on a B200.  Results do not depend on the choice beyond the
 * fp32 summation order. */
typedef enum {
  FP8_TILE_AUTO = 0, FP8_TILE_128x128 = 1, FP8_TILE_128x256 = 2, FP8_TILE_PAIR_256x256 = 3,
  FP8_TILE_SPLITK_128x128 = 4, FP8_TILE_STREAMK = 8
} fp8_tile_cfg;

typedef enum {
  FP8_OK = 0,
  FP8_ERR_INVALID_ARG = -1,    /* NULL required pointer, bad enum, ld < cols, ... */
  FP8_ERR_UNSUPPORTED = -2,    /* valid request this library does not implement */
  FP8_ERR_MISALIGNED = -3,     /* fp8 ld % 16 != 0 or base not 16-byte aligned  */
  FP8_ERR_CUDA = -4,           /* a CUDA call failed (see fp8_status_string)    */
  FP8_ERR_DEVICE_TIMEOUT = -5, /* a kernel gave up on a bounded wait            */
  FP8_ERR_WORKSPACE = -6,      /* workspace missing or smaller than required    */
  FP8_ERR_TOO_LARGE = -7       /* beyond the fixed scratch of a no-allocation entry point */
} fp8_status;

/* ------------------------------------------------------------------ rings
 * A scale ring is the delayed-scaling state of one tensor, one device buffer
 * of fp8_ring_bytes(H) bytes, 4-byte aligned (8-byte aligned with an even H
 * lets the in-kernel finalize use one 64-bit atomic on ticket + scratch),
 * laid out as 32-bit words:
 *   [0, H)   hist    fp32 amax history (slot step % H holds the newest)
 *   H        scale   fp32 scale the next quantize multiplies by
 *   H+1      step    u32 number of quantizes folded so far
 *   H+2      ticket  u32 block counter of the in-kernel finalize (0 at rest)
 *   H+3      scratch u32 bits of the running amax of a launch (0 at rest)
 * [tests/extension@2eeac02]: the ring packs history, scale and counter in one
 * buffer; the quantize kernel's last block folds the amax in and publishes
 * the next scale, so a step costs no extra launch.  Checkpointing a ring is
 * copying its bytes between launches.  1 <= H <= 4096. */
FP8LIN_API size_t fp8_ring_bytes(int hist_len);

/* hist = 0, scale = 1.0, ticket = step = scratch = 0.  One tiny kernel. */
FP8LIN_API int fp8_ring_init(void* ring, int hist_len, fp8_stream_t stream);

/* fp8_ring_init, then scale = fp8_max(fmt) / amax when amax (host value) is
 * positive and finite and the quotient is finite; otherwise scale stays 1.0.
 * The history is left at zero ([astrai@4019dda] names seed() on the ring). */
FP8LIN_API int fp8_ring_seed(void* ring, int hist_len, int fmt, float amax, fp8_stream_t stream);

/* ------------------------------------------------------------------ quantize
 * out[r, c] = cast_sat_rne_fmt( fp32(in[r, c]) * s ), s = the ring's scale at
 * launch, for r < rows, c < cols; bytes c in [cols, ld_out) are written 0.
 * In the same launch: amax = max |fp32(in)| over non-NaN elements of the RAW
 * input ([astrai/extension/fp8.py@3e57cc8]: the quantized max pinned the scale
 * at 1); the last block to finish then writes hist[step % H] = amax, takes
 * m = max(hist), publishes scale = fp8_max / m (kept when m is 0 or inf or the
 * quotient overflows), advances step, and rezeroes ticket and scratch.
 *   in        bf16/fp16/fp32 [rows, ld_in]            (in_dtype FP8_DT_BF16/FP16/FP32)
 *   fmt       FP8_E4M3 (max 448) or FP8_E5M2 (max 57344)
 *   ring      fp8_ring_bytes(hist_len) bytes, initialized (delayed scaling); or
 *             NULL for current (dynamic) scaling ([astrai@4019dda] recipe with
 *             a dynamic flag; [astrai/extension/fp8.py@3e57cc8] DynamicScaling:
 *             no rings, scales measured inline): a first launch reduces this
 *             tensor's amax into *amax_out (required then; zeroed first), and
 *             s = fp8_max / amax (1.0 when amax is 0 or not finite or the
 *             quotient overflows); hist_len is ignored.  Reads the input twice
 *             (the second read mostly from L2 for tensors up to ~100 MB).
 *   out       fp8 codes [rows, ld_out], ld_out % 16 == 0, 16-byte aligned
 *   amax_out  optional fp32 (required when ring is NULL): the amax of this launch
 *   scale_out optional fp32: the scale this launch multiplied by (the snapshot
 *             taken before the ring overwrites it, [astrai/extension/ops@057c0d3])
 * NaN inputs give the NaN code and do not enter amax; +-inf saturate to +-max. */
FP8LIN_API int fp8_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld_in,
                 int fmt, void* ring, int hist_len,
                 uint8_t* out, int64_t ld_out,
                 float* amax_out, float* scale_out, fp8_stream_t stream);

/* One quantize operand (the fields of fp8_quantize, as a struct). */
typedef struct fp8_quantize_args {
  const void* in; int in_dtype; int64_t rows, cols, ld_in;
  int fmt; void* ring; int hist_len;
  uint8_t* out; int64_t ld_out;
  float* amax_out; float* scale_out;
} fp8_quantize_args;

/* Two quantizes in ONE launch ([astrai@4019dda] quantize_dual: x and w of a
 * forward).  Each tensor keeps its own ring and last-block finalize, exactly
 * as two fp8_quantize calls would.  Both must share in_dtype and fmt, and use
 * different rings.  Either ring may be NULL (current scaling, amax_out
 * required and distinct); the amax passes of such tensors share one launch. */
FP8LIN_API int fp8_quantize_dual(const fp8_quantize_args* a, const fp8_quantize_args* b, fp8_stream_t stream);

/* fp8_quantize with flags.  FP8_QUANTIZE_DEFER_RING_STEP (ring required):
 * the launch quantizes with the ring's scale and writes scale_out as usual,
 * but only max-reduces this launch's amax into the ring's scratch word
 * (32-bit word hist_len + 3, i.e. byte offset (hist_len + 3) * 4); the
 * history, scale, step and amax_out wait for fp8_ring_finalize.  Between the
 * two, data-parallel ranks all-reduce that word with MAX (non-negative floats
 * order like their bit patterns, so an unsigned or signed 32-bit integer MAX
 * is exact), so every rank's ring takes the same step -- the one exchange the
 * method needs across data-parallel replicas.  Since delayed scaling casts
 * with the previous scale, the all-reduce can overlap the GEMM. */
enum { FP8_QUANTIZE_DEFER_RING_STEP = 1 };
FP8LIN_API int fp8_quantize_ex(const fp8_quantize_args* q, int flags, fp8_stream_t stream);

/* The pending step of a ring left by FP8_QUANTIZE_DEFER_RING_STEP: a = the
 * scratch word (as float), hist[step % H] = a, window max, scale = fp8_max(fmt)
 * / max with the keep-old rule, step + 1, scratch = 0, *amax_out = a (if
 * given) -- exactly the step the quantize's last block would have taken.  One
 * 32-thread launch.  Calling it with no pending step folds an amax of 0. */
FP8LIN_API int fp8_ring_finalize(void* ring, int hist_len, int fmt, float* amax_out, fp8_stream_t stream);

/* fp8_quantize of g [rows, cols] plus, in the same pass over g, its column
 * sums: dbias[c] = bf16( sum_r g[r, c] ) as fp8_dbias computes them (fp32
 * sums in a fixed order).  workspace as fp8_dbias (size from
 * fp8_dbias_workspace_bytes(rows, cols), zero-filled before first use).
 * g->ring NULL: current scaling as in fp8_quantize. */
FP8LIN_API int fp8_quantize_dbias(const fp8_quantize_args* g, void* dbias, void* workspace, size_t workspace_bytes,
                                  fp8_stream_t stream);

/* ------------------------------------------------------------------ mm
 * The GEMM primitive ([astrai/extension/ops@057c0d3] two-primitive API;
 * [astrai@4019dda] fused bias):
 *   D[i, j] = bf16_rne( (sum_k A(i,k) * B(j,k)) / (scale_a * scale_b) + bias[j] )
 * products and sums in fp32 on the tensor cores (tcgen05, kind::f8f6f4), one
 * rounding to bf16.  Operand storage:
 *   a_major FP8_K_MAJOR : A(i,k) = a[i*lda + k]  (a is [m, lda], lda >= k)
 *   a_major FP8_MN_MAJOR: A(i,k) = a[k*lda + i]  (a is [k, lda], lda >= m)
 *   b_major FP8_K_MAJOR : B(j,k) = b[j*ldb + k]  (b is [n, ldb], ldb >= k)
 *   b_major FP8_MN_MAJOR: B(j,k) = b[k*ldb + j]  (b is [k, ldb], ldb >= n)
 * so the forward (X W^T: both K-major), dX (G W: A K-major, B MN-major) and
 * dW (G^T X: both MN-major) run without transposed copies.
 *   scale_a, scale_b  required device fp32 scalars (the quantize snapshots)
 *   bias              optional [n]: bias_dtype FP8_DT_BF16 adds the bf16 value;
 *                     FP8_DT_E4M3/E5M2 adds decode(bias[j]) / *bias_scale
 *                     ([csrc@2eeac02] FP8Params bias bullet: fp8 bias
 *                     dequantized after the operand scaling)
 *   d                 bf16 [m, ldd], ldd >= n
 * Out-of-range rows/columns/k of partial tiles contribute nothing.  k = 0
 * (m, n > 0): every sum is empty, so D = bf16(0 + bias[j]), or 0 without a
 * bias (a small fill launch; the operands and scales are not read). */
typedef struct fp8_mm_args {
  int64_t m, n, k;
  const uint8_t* a; int fmt_a; int a_major; int64_t lda;
  const uint8_t* b; int fmt_b; int b_major; int64_t ldb;
  const float* scale_a; const float* scale_b;
  const void* bias; int bias_dtype; const float* bias_scale;
  void* d; int64_t ldd;
  int tile_cfg;   /* FP8_TILE_AUTO (0, chosen per shape) or one of fp8_tile_cfg */
  /* Stream-K workspace, used only with FP8_TILE_STREAMK (NULL / 0 otherwise):
   * >= fp8_mm_workspace_bytes(m, n, k) bytes, 16-byte aligned, ZERO-FILLED
   * before its first use; every call leaves its flags at zero again, so it
   * may be reused by later calls of the same sizes that are ordered after
   * this one (same stream).  FP8_TILE_STREAMK without it returns
   * FP8_ERR_WORKSPACE. */
  void* workspace; size_t workspace_bytes;
} fp8_mm_args;
FP8LIN_API int fp8_mm(const fp8_mm_args* args, fp8_stream_t stream);

/* Bytes of the stream-K workspace of an m x n x k GEMM (or of a two-GEMM
 * launch: the larger of the two): a fixed block of 1280 zero-at-rest flags,
 * then one 128 x 256 fp32 partial accumulator per CTA that can hold a cut
 * tile (at most 160, and at most one per 128 x 128 x 128 block of work).
 * 0 when m, n or k is 0. */
FP8LIN_API size_t fp8_mm_workspace_bytes(int64_t m, int64_t n, int64_t k);

/* A batch of GEMMs of one shape in one launch ([astrai@4019dda] mm_fp8 bullet:
 * 3-D operands through the same signature, batches sliced by strides, a
 * size-1 batch broadcast with stride 0, transposed views folded into the
 * layout tag at zero copy):
 *   D_b = args applied to A_b = a + b*stride_a, B_b = b + b*stride_b,
 *         D_b = d + b*stride_d, for b < batch (strides in ELEMENTS)
 * stride_a / stride_b 0 shares that operand across the batch; other operand
 * strides must be multiples of 16 bytes (FP8_ERR_MISALIGNED); stride_d >=
 * (m - 1) * ldd + n so that outputs do not overlap (FP8_ERR_INVALID_ARG).
 * Scales and bias are shared by the batch.  The tile configuration counts
 * batch x per-matrix tiles; split-K is not used for batch > 1 (the batch
 * already fills the SMs).  batch == 0 is a no-op; batch == 1 equals fp8_mm. */
FP8LIN_API int fp8_mm_batched(const fp8_mm_args* args, int64_t batch, int64_t stride_a, int64_t stride_b,
                              int64_t stride_d, fp8_stream_t stream);

/* Two independent GEMMs (the backward's dX and dW) in ONE launch over one
 * persistent tile schedule.  Same results as two fp8_mm calls; the tile
 * configuration (a->tile_cfg, or chosen for the pair when AUTO) and, for
 * FP8_TILE_STREAMK, the workspace (a->workspace, >= fp8_mm_workspace_bytes of
 * either problem) are shared. */
FP8LIN_API int fp8_mm_pair(const fp8_mm_args* a, const fp8_mm_args* b, fp8_stream_t stream);

/* The tile configuration fp8_mm (b == NULL) or fp8_mm_pair (b != NULL) would
 * choose for these arguments on a GPU with num_sms SMs -- host arithmetic
 * only: nothing is launched, the GPU is not touched and the operands are not
 * read, so it works without a device.  The arguments are validated as
 * fp8_mm validates them (same status codes).  Split-K, which FP8_TILE_AUTO
 * may also pick for a single few-tile, long-K problem, depends on the
 * device's cluster occupancy and is not considered here.  Output (host
 * pointer):
 *   tile_cfg  the fp8_tile_cfg value (a forced a->tile_cfg comes back as given;
 *             FP8_TILE_AUTO when every problem is empty);
 *   tiles     output tiles of that configuration over the problem(s);
 *   units     CTAs (CTA pairs for FP8_TILE_PAIR_256x256) the launch keeps
 *             busy: min(tiles, num_sms) (pairs: num_sms / 2; stream-K: all);
 *   est_us    the cost model's estimate of the launch in microseconds (fitted
 *             to B200 timings; 0 for a forced configuration). */
typedef struct {
  int tile_cfg;
  int64_t tiles;
  int units;
  double est_us;
  int stream_k_ctas;   /* CTAs sharing the stream-K k-blocks (0: no stream-K) */
  int64_t dp_tiles;    /* tiles run whole before the stream-K part */
} fp8_mm_plan_info;
FP8LIN_API int fp8_mm_plan(const fp8_mm_args* a, const fp8_mm_args* b, int num_sms, fp8_mm_plan_info* out);

/* ------------------------------------------------------------------ dbias
 * dbias[n] = bf16_rne( sum_m g(m, n) ), fp32 sums, for n < N.  g is bf16,
 * fp16 or fp32 [M, ldg], or fp8 (E4M3/E5M2) [M, ldg] with g_scale required:
 * then each element is dequantized, decode(g8) / *g_scale, before the sum
 * ([astrai/extension/ops@057c0d3]: a pre-quantized g dequantizes before the
 * bias sum).  The result is deterministic for a given (M, N) (fixed partial
 * order).  workspace: >= fp8_dbias_workspace_bytes(M, N) bytes, 16-byte
 * aligned, ZERO-FILLED before its first use; every call leaves it ready for
 * the next (its counters back at zero). */
FP8LIN_API size_t fp8_dbias_workspace_bytes(int64_t M, int64_t N);
FP8LIN_API int fp8_dbias(const void* g, int g_dtype, int64_t M, int64_t N, int64_t ldg,
              const float* g_scale, void* dbias,
              void* workspace, size_t workspace_bytes, fp8_stream_t stream);

/* fp8_dbias without a workspace argument.  No page of the source describes
 * this entry point; it exists for callers that cannot allocate device memory
 * themselves (code running under a memory manager it does not control, such as
 * a plugin inside a serving runtime with a fixed device-memory budget, or a C
 * caller with no access to the framework's allocator) and therefore have no
 * workspace to pass.  The same kernel and arguments as fp8_dbias; its scratch
 * is a 1 MiB array compiled into the library, which every GPU that loads the
 * library holds until the process exits.
 *   - Requests needing more than 1 MiB of scratch (fp8_dbias_workspace_bytes(M,
 *     N) > 1048576; every N <= 131072 fits, whatever M) return
 *     FP8_ERR_TOO_LARGE and enqueue nothing.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on a device looks up the array's device address (once
 *     per device, under a lock); make that first call before any stream
 *     capture.  The address is kept for the life of the process, so the
 *     device must keep one CUDA context meanwhile: no cudaDeviceReset (or
 *     other context teardown) while the library is in use.
 *   - All calls share the one array: calls that can overlap on the GPU (other
 *     streams, other host threads) race and must be serialized by the caller.
 *     Each call clears the tile counters it needs before its kernel. */
FP8LIN_API int fp8_dbias_noalloc(const void* g, int g_dtype, int64_t M, int64_t N, int64_t ldg,
                      const float* g_scale, void* dbias, fp8_stream_t stream);

/* ------------------------------------------------------------------ linear
 * Forward of the FP8 linear ([tests/extension@2eeac02], [astrai/extension/ops@057c0d3]):
 *   x [M, K] and w [N, K] (PyTorch out x in) are each either bf16/fp16/fp32,
 *   quantized here with their own ring (x with fmt_x into x8, w with fmt_w into
 *   w8), or already fp8 in the matching format, in which case the quantize is
 *   skipped, the operand is used in place, its scale is *x_scale_in /
 *   *w_scale_in and its amax output is 0 ([tests/extension@2eeac02], w8 bullet).
 *   Then y = bf16( X8 W8^T / (sx sw) + bias ), as fp8_mm.
 * Outputs: y (bf16 [M, ldy]); x8/w8 (fp8, kept by the caller for the
 * backward; unused when that operand arrives fp8); sx_out/sw_out (required:
 * the scales the GEMM dequantized with); amax_x_out/amax_w_out (optional).
 * A NULL ring_x / ring_w selects current scaling for that operand, as in
 * fp8_quantize (its amax output is then required; one extra amax launch for
 * one or both).  Inside this call a ring's step is completed by the GEMM
 * launch, not by the quantize's last block (same ring words; one launch
 * fewer on the critical path).  2 to 4 launches.  hist_len is the H of both
 * rings. */
typedef struct fp8_linear_fwd_args {
  int64_t M, N, K;
  const void* x; int x_dtype; int64_t ldx; const float* x_scale_in;
  const void* w; int w_dtype; int64_t ldw; const float* w_scale_in;
  const void* bias; int bias_dtype; const float* bias_scale;
  int fmt_x, fmt_w, hist_len;
  void* ring_x; void* ring_w;
  uint8_t* x8; int64_t ldx8;
  uint8_t* w8; int64_t ldw8;
  float* sx_out; float* sw_out; float* amax_x_out; float* amax_w_out;
  void* y; int64_t ldy;
} fp8_linear_fwd_args;
FP8LIN_API int fp8_linear_forward(const fp8_linear_fwd_args* args, fp8_stream_t stream);

/* Backward of the FP8 linear ([astrai/extension/ops@057c0d3]):
 *   g [M, N] is bf16/fp16/fp32, quantized with ring_g (fmt_g, normally E5M2)
 *   into g8 (ring_g NULL: current scaling, amax_g_out required), or already
 *   fp8 (then *g_scale_in is its scale, amax_g_out = 0).
 *   dx = bf16( G8 W8 / (sg sw) )    [M, K]  when need_dx
 *   dw = bf16( G8^T X8 / (sg sx) )  [N, K]  when need_dw
 *   dbias = bf16( sum_m g )         [N]     when need_dbias ([astrai@4019dda]:
 *                                           only when the bias needs a grad)
 * sx, sw, x8, w8 are the FORWARD's snapshots and quantized operands: the
 * backward reuses the forward's scales.  Outputs are bf16 whatever the input
 * dtypes.  workspace: as fp8_dbias, needed only when need_dbias (size from
 * fp8_linear_workspace_bytes).  Up to 4 launches. */
typedef struct fp8_linear_bwd_args {
  int64_t M, N, K;
  const void* g; int g_dtype; int64_t ldg; const float* g_scale_in;
  int fmt_g, hist_len; void* ring_g;
  uint8_t* g8; int64_t ldg8;
  float* sg_out; float* amax_g_out;
  const uint8_t* x8; int64_t ldx8; const float* sx; int fmt_x;
  const uint8_t* w8; int64_t ldw8; const float* sw; int fmt_w;
  int need_dx, need_dw, need_dbias;
  void* dx; int64_t lddx;
  void* dw; int64_t lddw;
  void* dbias;
  void* workspace; size_t workspace_bytes;
} fp8_linear_bwd_args;
FP8LIN_API int fp8_linear_backward(const fp8_linear_bwd_args* args, fp8_stream_t stream);

/* Workspace bytes fp8_linear_backward needs for need_dbias (0 when M or N is
 * 0).  Equal to fp8_dbias_workspace_bytes(M, N): one size covers the row
 * splits of fp8_dbias and of the column-sum quantize (fp8_quantize_dbias and
 * the backward's g).  Zero-fill it once before first use, like fp8_dbias's
 * workspace; every call leaves it ready for the next call of the same sizes.
 * K does not enter. */
FP8LIN_API size_t fp8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* ------------------------------------------------------------------ status
 * Kernels never wait without a bound: a wait that runs out records
 * FP8_ERR_DEVICE_TIMEOUT in a device word and the kernel returns.  This call
 * reads that word (synchronizing the device) and clears it; FP8_OK if clear. */
FP8LIN_API int fp8_get_device_status(void);

/* The bounded waits themselves, exercised on purpose (a diagnostic, not a
 * step of the path): one tiny kernel waits, with a time limit of limit_ns
 * nanoseconds (1 ns .. 2 s), on the 32-bit device word *flag becoming
 * non-zero (the stream-K flag protocol) and on an mbarrier that nothing ever
 * arrives on (the GEMM pipeline protocol).  results (device, 2 ints): 1 where
 * the wait was satisfied, 0 where it ran out.  A wait that runs out records
 * FP8_ERR_DEVICE_TIMEOUT for fp8_get_device_status; the kernel then returns,
 * and the context stays usable.  flag and results 4-byte aligned, else
 * FP8_ERR_INVALID_ARG. */
FP8LIN_API int fp8_wait_selftest(const void* flag, uint64_t limit_ns, int* results, fp8_stream_t stream);

/* Static description of a status code (for FP8_ERR_CUDA: the last CUDA error
 * this library saw, on the calling host thread). */
FP8LIN_API const char* fp8_status_string(int status);

/* Library version string, e.g. "fp8lin 0.1 sm_100a". */
FP8LIN_API const char* fp8_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FP8LIN_H */
