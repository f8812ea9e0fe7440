// internal.h -- launchers shared between the translation units of libfp8lin.
// Host-side only types; no CUDA device code.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fp8lin {

enum : int { kE4M3 = 0, kE5M2 = 1 };
enum : int { kBF16 = 0, kFP16 = 1, kFP32 = 2, kDtE4M3 = 3, kDtE5M2 = 4 };

// Ring word offsets (in 32-bit words) for history length H:
// [hist (H) | scale | step | ticket | scratch].  With H even (and the ring
// 8-byte aligned) ticket and scratch form one aligned 8-byte word, which the
// in-kernel finalize updates with one 64-bit atomic per block.
__host__ __device__ constexpr int ring_scale(int H) { return H; }
__host__ __device__ constexpr int ring_step(int H) { return H + 1; }
__host__ __device__ constexpr int ring_ticket(int H) { return H + 2; }
__host__ __device__ constexpr int ring_scratch(int H) { return H + 3; }

struct QuantizeParams {
  const void* in;
  int64_t rows, cols, ld_in;  // rows == 1 with cols = total for contiguous data
  uint8_t* out;
  int64_t ld_out;
  int64_t chunks_per_row;     // ceil(cols / 16)
  int64_t total_chunks;
  float* ring;                // [hist | scale | step | ticket | scratch]
  int H;
  float fp8_max;
  float* amax_out;
  float* scale_out;
  int vec_ok;                 // 16-byte vector loads are legal for full chunks
  int defer_finalize;         // 1: only fold block maxima into the ring's scratch
                              // word; the GEMM that consumes the output finalizes
  const float* dyn_amax;      // current scaling: ring unused, s = fp8_max / *dyn_amax
                              // (the amax pass reduced it there before this launch)
};

// One or two tensors quantized by one launch: blocks [0, blocks0) work on
// t[0], the rest on t[1] (each with its own ring and last-block finalize).
struct QuantizePair {
  QuantizeParams t[2];
  int blocks0;
  int pf_blocks;              // the first pf_blocks blocks prefetch the inputs into L2
};

// Quantize of a [rows, cols] tensor (not flattened) that also produces its
// column sums: grid (ceil(cols / 256), R), partial [R, cols] fp32 and one
// counter per column tile in a caller workspace.
struct ColsumParams {
  QuantizeParams q;
  float* partial;
  unsigned* counters;
  void* dbias;                // bf16 [cols]
  int64_t rows_per_split;
  int R;
  int defer_sum;              // 1: only write the partials; the GEMM that
                              // follows sums them (DbiasFinish)
};

// Side writes a GEMM launch performs once (block 0), for operands that arrive
// pre-quantized: dst = *src for the scale snapshot, zero for its amax.
struct SideWrites {
  const float* copy_src[2];
  float* copy_dst[2];
  float* zero_dst[2];
};

// A scale ring whose quantize ran with defer_finalize: the GEMM launch that
// reads the quantized output completes the ring step (fold the scratch max
// into the history, publish the next scale, advance step, clear scratch).
struct RingFinalize {
  float* ring;
  int H;
  float fp8_max;
  float* amax_out;
};

// The bias gradient of a quantize whose column sums ran with defer_sum: the
// GEMM launch that follows turns the R x cols partials into dbias (bf16),
// each column summed in the same fixed order as the quantize's own last
// block would have.
struct DbiasFinish {
  const float* partial;
  void* dbias;
  int64_t cols;
  int R;
};

// One GEMM problem of a launch (a launch runs one or two of them over one
// persistent tile schedule: the backward's dX and dW share a launch).
struct GemmProblem {
  int m, n, k;
  int tiles_m, tiles_n, num_tiles, k_blocks;
  int raster_group;           // M-tiles per raster group
  uint32_t idesc;
  int a_major, b_major;
  const float* scale_a;
  const float* scale_b;
  const void* bias;
  int bias_kind;              // 0 none, 1 bf16, 2 e4m3, 3 e5m2
  const float* bias_scale;
  void* d;
  int64_t ldd;
  int tma_store;              // D is addressable by TMA (16-byte aligned base, pitch and row end)
  int batch;                  // independent GEMMs of this shape; tiles enumerate batch x tiles_m x tiles_n
  int bcast_a, bcast_b;       // operand shared by every batch (batch stride 0): batch coordinate 0
  int64_t stride_d;           // elements between consecutive batches of D
};

struct GemmParams {
  GemmProblem pr[2];
  int nprob;
  int tiles0;                 // tiles of pr[0]; tile t >= tiles0 belongs to pr[1]
  int total_tiles;
  int any_tma_store;
  int* status;
  SideWrites side;
  RingFinalize fin[2];
  int nfin;
  DbiasFinish dbias;          // partial == nullptr: none
  int split;                  // split-K launches: CTAs per tile (cluster size)
  // Tile schedule.  CTA (or pair) u runs slots u, u + units, u + 2 units, ...
  // below nslots; with use_order, slot s holds tile order[s] (kNoTile: none),
  // else tile s.
  int nslots;
  int use_order;
  // Stream-K (single-CTA tiles; sk_ctas = 0: off).  The slots above cover the
  // whole tiles [0, dp_tiles); the k-blocks of tiles [dp_tiles, total_tiles),
  // sk_total of them in tile order (sk_u0 belong to problem 0), are split
  // into sk_ctas contiguous ranges, range c = [c sk_total / sk_ctas,
  // (c + 1) sk_total / sk_ctas) for CTA c.  A tile cut by range boundaries
  // is finished by the CTA whose range holds its first k-block: the CTAs
  // holding its later k-blocks store their fp32 partial accumulators in
  // sk_part (one slot per CTA) and raise one flag per epilogue warp in
  // sk_flag; the finishing CTA adds them in CTA order and clears the flags.
  int sk_ctas;
  int dp_tiles;
  int64_t sk_total;
  int64_t sk_u0;
  float* sk_part;             // [sk_ctas][BN / 4][128][4]
  unsigned* sk_flag;          // [sk_ctas][8]
  uint16_t order[1024];
};
constexpr int kMaxOrder = 1024;
constexpr uint16_t kNoTile = 0xFFFF;

// D = bias broadcast over the rows (bf16, or fp8 / bias_scale), or zero: the
// GEMM of an empty contraction (K = 0), where every accumulator is 0.
struct FillParams {
  void* d;
  int64_t ldd, stride_d;      // elements
  int64_t m, n, batch;
  const void* bias;
  int bias_kind;              // 0 none, 1 bf16, 2 e4m3, 3 e5m2
  const float* bias_scale;
};

struct DbiasParams {
  const void* g;
  int dtype;
  int64_t M, N, ldg;
  const float* g_scale;
  void* dbias;
  float* partial;             // [R, N] fp32
  unsigned* counters;         // [col_tiles]
  int64_t rows_per_split;
  int R;
  int vec_ok;
};

int num_sms(int device);
// Keeps e's name for fp8_status_string(FP8_ERR_CUDA) on this host thread and
// returns FP8_ERR_CUDA.
int record_cuda_error(cudaError_t e);

// b may be NULL (one tensor); both tensors share in_dtype and fmt.
cudaError_t launch_quantize(int in_dtype, int fmt, const QuantizeParams* a, const QuantizeParams* b, cudaStream_t s);
cudaError_t launch_quantize_colsum(int in_dtype, int fmt, const ColsumParams& cp, cudaStream_t s);
// Current scaling's first pass: max |x| of one or two tensors (b may be NULL)
// reduced into each one's dyn_amax word, which must be zero beforehand.
cudaError_t launch_amax(int in_dtype, const QuantizeParams* a, const QuantizeParams* b, cudaStream_t s);
cudaError_t launch_ring_set(float* ring, int H, float scale, cudaStream_t s);
cudaError_t launch_side_writes(const SideWrites& w, cudaStream_t s);
cudaError_t launch_ring_finalize(const RingFinalize& f, cudaStream_t s);
// GEMM tile configurations: 128x128 and 128x256 on one CTA, 256x256 on a pair
// of CTAs (2-SM MMA).
enum : int { kGemm128 = 1, kGemm256 = 2, kGemmPair256 = 3, kGemmSplit128 = 4 };
// Split factor (2..3, or 1 for none) for a 128 x 128-tile problem: the largest
// S with every rank given >= 4 k-blocks and all tiles' clusters resident in
// one wave; forced: the largest S <= min(3, k_blocks) fitting one wave, else 2.
int gemm_split_factor(int tiles, int k_blocks, int sms, bool forced);
// CTA pairs (256x256 tiles) that can be resident at once on the device.
int gemm_pair_capacity(int device);
// maps[0..2]: A, B, D of pr[0]; maps[3..5]: those of pr[1] (zeroed if unused).
cudaError_t launch_gemm(const CUtensorMap* maps, const GemmParams& p, int cfg, cudaStream_t s);
cudaError_t launch_dbias(const DbiasParams& p, cudaStream_t s);
cudaError_t launch_fill(const FillParams& p, cudaStream_t s);
cudaError_t launch_wait_selftest(const uint32_t* flag, int* status, int* results, uint64_t limit_ns,
                                 cudaStream_t s);

// Column-sum geometry (R row splits of rows_per_split rows over 256-column
// tiles) shared by the size queries and the launchers: dbias_geometry for the
// dbias kernel, colsum_geometry for the column-sum quantize (standalone, or
// in the linear backward with its sums finished by the GEMM launch).
// Workspaces hold the per-tile counters first (16-byte rounded), then R x N
// fp32 partials for the larger R of the two, so one workspace serves both.
constexpr int kDbiasColsPerTile = 256;
void dbias_geometry(int64_t M, int64_t N, int* R, int64_t* rows_per_split);
void colsum_geometry(int64_t M, int64_t N, int* R, int64_t* rows_per_split);

}  // namespace fp8lin
