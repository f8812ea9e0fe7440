// quantize.cu -- HBM-bound fp8 quantize with in-kernel delayed-scaling finalize.
//
// One launch per tensor, or per pair of tensors (AstrAI commit log,
// tests/extension @2eeac02, bullets on finalizing scale rings inside the
// quantize kernels; astrai @4019dda, quantize_dual bullet):
//   1. every thread reads its ring's current scale s (the first block of the
//      tensor also stores it to scale_out: the snapshot the GEMM dequantizes
//      with, astrai/extension/ops @057c0d3 snapshot bullet);
//   2. a grid-stride loop over 16-element chunks streams the input with
//      16-byte loads (the next iteration's loads are issued before the
//      current chunks are converted), keeps a running max of |x| over the RAW
//      values (NaN ignored), multiplies by s in fp32 and casts pairs with
//      cvt.rn.satfinite.{e4m3,e5m2}x2, storing 16 fp8 codes per 16-byte store;
//   3. warp max (redux.sync) -> block max -> one relaxed red.max on the ring's
//      scratch word (non-negative floats order like their bit patterns);
//   4. a fetch-add on the ring's ticket: the block that draws the tensor's
//      last ticket sees every block's max, folds the launch's amax into
//      hist[step % H], reduces the window, and publishes fp8_max / max as the
//      next scale (kept when the max is 0 or inf or the quotient overflows),
//      then rezeroes ticket and scratch.  When ticket and scratch share an
//      aligned 8-byte word (even H), the ticket is one relaxed 64-bit add whose
//      return value already carries the max: one round trip, no fence.
//      Otherwise an acquire-release add, then an exchange of the scratch word.
//      History and step are prefetched into shared memory at kernel start.
//   4'. with defer_finalize (the fused linear entry points, where a GEMM that
//      reads the output always follows) step 4 is skipped: each block's max
//      goes to the scratch word and the GEMM -- which starts reading only after
//      this grid has completed -- does the finalize in one warp while its
//      mainloop runs.  That takes the ticket round trip and the last block's
//      ring update off every quantize launch.
// The column-sum variant (quantize of g with the bias gradient) walks 2-D
// tiles of 256 columns instead -- a warp spans a tile row, 8 columns a lane,
// eight rows' loads in flight per lane before any is cast -- so each thread
// also accumulates the column sums of its 8 columns (0.52 -> 0.77 of HBM at
// 4096 x 11008 against 16 columns and four rows a lane); per-tile partials
// meet in a workspace and the last
// block of each column tile (its own ticket) sums them in a fixed order
// (astrai @4019dda: the column sum runs only when the bias needs a gradient).
// With defer_sum (a GEMM follows in the fused backward) the blocks stop after
// writing their partials and the GEMM's idle epilogue warps do the fixed-order
// sums, as they do the deferred ring finalize.
// No block ever waits on another, so nothing here can hang.
#include <type_traits>

#include "device.cuh"
#include "internal.h"
#include "launch.h"
#include "partials.cuh"
#include "ring.cuh"

namespace fp8lin {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 16;
constexpr int kHistCache = 64;  // ring histories up to this length are prefetched
constexpr uint64_t kPrefetchMaxBytes = uint64_t(48) << 20;  // early L2 prefetch only up to this input size

// ---------------------------------------------------------------- raw chunks

// 16 consecutive input elements, kept as raw bits until converted.
template <typename T>
struct Raw {
  static constexpr int kWords = static_cast<int>(sizeof(T)) * kChunk / 16;
  uint4 w[kWords];
};

template <typename T>
__device__ __forceinline__ uint32_t elem_bits(const void* base, int64_t idx) {
  if constexpr (sizeof(T) == 2) return static_cast<uint32_t>(__ldg(static_cast<const unsigned short*>(base) + idx));
  else return __float_as_uint(__ldg(static_cast<const float*>(base) + idx));
}

// Load the chunk starting at (r, col): 16-byte loads when the whole chunk is
// inside the row and the rows are 16-byte aligned, else element loads with
// zeros past the row end.
template <typename T>
__device__ __forceinline__ void load_raw(const QuantizeParams& p, int64_t r, int64_t col, Raw<T>& raw) {
  const int64_t base = r * p.ld_in + col;
  if (p.vec_ok && col + kChunk <= p.cols) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.in) + base);
    #pragma unroll
    for (int i = 0; i < Raw<T>::kWords; ++i) raw.w[i] = __ldg(src + i);
  } else {
    const int64_t left = p.cols - col;
    uint32_t b[kChunk];
    #pragma unroll
    for (int j = 0; j < kChunk; ++j) b[j] = (j < left) ? elem_bits<T>(p.in, base + j) : 0u;
    #pragma unroll
    for (int i = 0; i < Raw<T>::kWords; ++i) {
      if constexpr (sizeof(T) == 2)
        raw.w[i] = make_uint4(b[8 * i] | (b[8 * i + 1] << 16), b[8 * i + 2] | (b[8 * i + 3] << 16),
                              b[8 * i + 4] | (b[8 * i + 5] << 16), b[8 * i + 6] | (b[8 * i + 7] << 16));
      else
        raw.w[i] = make_uint4(b[4 * i], b[4 * i + 1], b[4 * i + 2], b[4 * i + 3]);
    }
  }
}

template <typename T>
__device__ __forceinline__ void to_floats(const Raw<T>& raw, float (&v)[16]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(raw.w);
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else if constexpr (std::is_same<T, __half>::value) {
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
    #pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(w[i]);
  }
}

template <int FMT>
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) {
  return FMT == kE4M3 ? cvt_e4m3x2(lo, hi) : cvt_e5m2x2(lo, hi);
}

// amax, scale, cast and one 16-byte store of the chunk at (r, col); bytes past
// cols (row padding up to ld_out) are written as zero.
template <int FMT>
__device__ __forceinline__ void cast_store(const QuantizeParams& p, int64_t r, int64_t col, const float (&v)[16],
                                           float s, float& amax) {
  uint32_t w[4];
  #pragma unroll
  for (int i = 0; i < 8; ++i) {
    amax = fmaxf(amax, fabsf(v[2 * i]));
    amax = fmaxf(amax, fabsf(v[2 * i + 1]));
    const uint32_t h = cvt2<FMT>(v[2 * i] * s, v[2 * i + 1] * s);
    if (i & 1) w[i >> 1] |= h << 16;
    else w[i >> 1] = h;
  }
  const int64_t left = p.cols - col;
  if (left < kChunk) {
    #pragma unroll
    for (int j = 0; j < kChunk; ++j)
      if (j >= left) w[j >> 2] &= ~(0xFFu << (8 * (j & 3)));
  }
  *reinterpret_cast<uint4*>(p.out + r * p.ld_out + col) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void chunk_pos(const QuantizeParams& p, int64_t c, int64_t& r, int64_t& col) {
  if (p.rows == 1) {
    r = 0;
    col = c * kChunk;
  } else {
    r = c / p.chunks_per_row;
    col = (c - r * p.chunks_per_row) * kChunk;
  }
}

// ---------------------------------------------------------------- ring finalize

// Thread 0: the block's max goes to the ring; the tensor's last block folds
// the launch amax into the ring and publishes the next scale.
__device__ __forceinline__ void ring_finalize(const QuantizeParams& p, uint32_t bits, uint32_t nblocks, float s,
                                              uint32_t step, const float* hist_s) {
  uint32_t* words = reinterpret_cast<uint32_t*>(p.ring);
  uint32_t* ticket = words + ring_ticket(p.H);
  uint32_t* scratch = words + ring_scratch(p.H);
  if (bits) red_max_u32(scratch, bits);
  float a;
  const bool paired = (reinterpret_cast<uintptr_t>(ticket) & 7u) == 0;
  if (paired) {
    // ticket (low half) and scratch (high half) are one 8-byte word.  The red
    // above and this add both write bytes of it, so program order puts this
    // block's max before its ticket in that word's coherence order; the add
    // that draws the last ticket therefore returns every block's max in its
    // high half.  No fence and no second round trip.
    const uint64_t old = atom_add_relaxed_u64(ticket, 1ull);
    if (static_cast<uint32_t>(old) != nblocks - 1) return;
    a = __uint_as_float(static_cast<uint32_t>(old >> 32));
  } else {
    // The release orders the red above before the ticket; the block that draws
    // the last ticket acquires every earlier block's red.
    if (atom_add_acq_rel(ticket, 1u) != nblocks - 1) return;
    a = __uint_as_float(atomicExch(scratch, 0u));
  }
  const uint32_t slot = step % static_cast<uint32_t>(p.H);
  float m = a;
  if (p.H <= kHistCache) {
    for (int i = 0; i < p.H; ++i)
      if (static_cast<uint32_t>(i) != slot) m = fmaxf(m, hist_s[i]);
  } else {
    for (int i = 0; i < p.H; ++i)
      if (static_cast<uint32_t>(i) != slot) m = fmaxf(m, p.ring[i]);
  }
  const float snew = next_scale(s, m, p.fp8_max);
  p.ring[slot] = a;
  p.ring[p.H] = snew;
  words[ring_step(p.H)] = step + 1;
  if (paired) *reinterpret_cast<volatile unsigned long long*>(ticket) = 0ull;  // ticket and scratch
  else atomicExch(ticket, 0u);
  if (p.amax_out) *p.amax_out = a;
}

// The scale a launch multiplies by: the ring's current scale (delayed), or
// fp8_max / this tensor's amax (current scaling; 1.0 when amax is 0 or not
// finite or the quotient overflows -- the ring's keep rule with 1.0 kept).
__device__ __forceinline__ float scale_of(const QuantizeParams& p) {
  return p.dyn_amax ? next_scale(1.0f, *p.dyn_amax, p.fp8_max) : p.ring[p.H];
}

// Thread 0's end of a block: with a deferred finalize only the block's max
// goes to the ring's scratch word (the consuming GEMM, which starts reading
// only after this grid completed, finishes the step); else the last-block
// finalize above.
__device__ __forceinline__ void ring_tail(const QuantizeParams& p, uint32_t bits, uint32_t nblocks, float s,
                                          uint32_t step, const float* hist_s) {
  if (p.defer_finalize) {
    if (bits) red_max_u32(reinterpret_cast<uint32_t*>(p.ring) + ring_scratch(p.H), bits);
    return;
  }
  ring_finalize(p, bits, nblocks, s, step, hist_s);
}

__device__ __forceinline__ uint32_t block_max_bits(float amax, uint32_t* warp_max) {
  uint32_t bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = bits;
  cta_sync();
  #pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) bits = max(bits, warp_max[w]);
  return bits;
}

// ---------------------------------------------------------------- flat kernel

// chunks per thread per iteration (plus as many prefetched): 64 bytes of input
constexpr int unroll_for(int bytes) { return bytes == 2 ? 2 : 1; }

// Before the dependency wait: the blocks that become resident first (one per
// SM fits beside a GEMM CTA still running) prefetch the contiguous inputs into
// L2, each a 1/pf_blocks slice of every tensor, so the DRAM latency overlaps
// the previous kernel's tail.  Safe whatever that kernel writes: a prefetch
// only warms L2, the loads come after the wait.
template <typename T>
__device__ __forceinline__ void prefetch_inputs(const QuantizePair& pair) {
  if (threadIdx.x == 0 && blockIdx.x < static_cast<unsigned>(pair.pf_blocks)) {
    const int ntensors = pair.blocks0 < static_cast<int>(gridDim.x) ? 2 : 1;
    for (int i = 0; i < ntensors; ++i) {
      const QuantizeParams& q = pair.t[i];
      if (q.rows != 1 || !q.vec_ok) continue;  // strided rows: no single range
      const uint64_t bytes = (static_cast<uint64_t>(q.cols) * sizeof(T)) & ~uint64_t(15);
      // large inputs stream at full bandwidth anyway; there the early lines
      // only compete with the loads (measured on a B200: 90 MB 0.80 -> 0.76 of
      // HBM with the prefetch, 28-32 MB 3-6 % faster)
      if (bytes > kPrefetchMaxBytes) continue;
      const uint64_t span = (bytes / static_cast<uint64_t>(pair.pf_blocks) + 15) & ~uint64_t(15);
      const uint64_t off = static_cast<uint64_t>(blockIdx.x) * span;
      if (span > 0 && off < bytes)
        prefetch_l2_bulk(static_cast<const uint8_t*>(q.in) + off, static_cast<uint32_t>(min(span, bytes - off)));
    }
  }
}

template <typename T, int FMT>
__global__ void __launch_bounds__(kThreads, 4) quantize_kernel(const __grid_constant__ QuantizePair pair) {
  __shared__ uint32_t warp_max[kThreads / 32];
  __shared__ float hist_s[kHistCache];
  constexpr int U = unroll_for(sizeof(T));
  prefetch_inputs<T>(pair);
  pdl_wait();
  pdl_trigger();
  const bool second = blockIdx.x >= pair.blocks0;
  const QuantizeParams& p = second ? pair.t[1] : pair.t[0];
  const uint32_t bid = second ? blockIdx.x - pair.blocks0 : blockIdx.x;
  const uint32_t nblocks = second ? gridDim.x - pair.blocks0 : pair.blocks0;

  const float s = scale_of(p);
  const bool do_step = p.ring && !p.defer_finalize;  // this launch finalizes the ring
  uint32_t step = 0;
  if (threadIdx.x == 0) {
    if (do_step) step = reinterpret_cast<const uint32_t*>(p.ring)[ring_step(p.H)];
    if (bid == 0 && p.scale_out) *p.scale_out = s;
  }
  // Only the tensor's last block writes its ring, after every block read it.
  if (do_step && p.H <= kHistCache && threadIdx.x < p.H) hist_s[threadIdx.x] = p.ring[threadIdx.x];

  float amax = 0.0f;
  const int64_t stride = static_cast<int64_t>(nblocks) * kThreads;
  int64_t c = static_cast<int64_t>(bid) * kThreads + threadIdx.x;
  Raw<T> cur[U];
  #pragma unroll
  for (int u = 0; u < U; ++u) {
    const int64_t cu = c + u * stride;
    if (cu < p.total_chunks) {
      int64_t r, col;
      chunk_pos(p, cu, r, col);
      load_raw<T>(p, r, col, cur[u]);
    }
  }
  // Every round but the last: the next round's loads are issued before the
  // current chunks are converted and stored.
  #pragma unroll 1
  while (c + U * stride < p.total_chunks) {
    const int64_t cn = c + U * stride;
    Raw<T> nxt[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t cu = cn + u * stride;
      if (cu < p.total_chunks) {
        int64_t r, col;
        chunk_pos(p, cu, r, col);
        load_raw<T>(p, r, col, nxt[u]);
      }
    }
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t cu = c + u * stride;
      if (cu < p.total_chunks) {
        int64_t r, col;
        chunk_pos(p, cu, r, col);
        float v[16];
        to_floats<T>(cur[u], v);
        cast_store<FMT>(p, r, col, v, s, amax);
      }
    }
    #pragma unroll
    for (int u = 0; u < U; ++u) cur[u] = nxt[u];
    c = cn;
  }
  // Last round: its amax first, then the block's ring tail, then its stores.
  // The tail's release (the last-block ticket) then waits only for the
  // stores of earlier rounds, which drain while these loads are in flight,
  // and the finalize runs beside the other blocks' last stores.
  #pragma unroll
  for (int u = 0; u < U; ++u) {
    if (c + u * stride < p.total_chunks) {
      float v[16];
      to_floats<T>(cur[u], v);
      #pragma unroll
      for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    }
  }
  if (p.ring) {  // current scaling: amax was reduced by the amax pass
    const uint32_t bits = block_max_bits(amax, warp_max);
    if (threadIdx.x == 0) ring_tail(p, bits, nblocks, s, step, hist_s);
  }
  float unused = 0.0f;
  #pragma unroll
  for (int u = 0; u < U; ++u) {
    const int64_t cu = c + u * stride;
    if (cu < p.total_chunks) {
      int64_t r, col;
      chunk_pos(p, cu, r, col);
      float v[16];
      to_floats<T>(cur[u], v);
      cast_store<FMT>(p, r, col, v, s, unused);
    }
  }
}

// ---------------------------------------------------------------- amax pass

// Current scaling's first pass: the same chunk walk as the quantize, max |x|
// only (NaN ignored), one red.max per block into the tensor's dyn_amax word.
template <typename T>
__global__ void __launch_bounds__(kThreads, 4) amax_kernel(const __grid_constant__ QuantizePair pair) {
  __shared__ uint32_t warp_max[kThreads / 32];
  constexpr int U = unroll_for(sizeof(T));
  prefetch_inputs<T>(pair);
  pdl_wait();
  pdl_trigger();
  const bool second = blockIdx.x >= pair.blocks0;
  const QuantizeParams& p = second ? pair.t[1] : pair.t[0];
  const uint32_t bid = second ? blockIdx.x - pair.blocks0 : blockIdx.x;
  const uint32_t nblocks = second ? gridDim.x - pair.blocks0 : pair.blocks0;
  float amax = 0.0f;
  const int64_t stride = static_cast<int64_t>(nblocks) * kThreads;
  #pragma unroll 1
  for (int64_t c = static_cast<int64_t>(bid) * kThreads + threadIdx.x; c < p.total_chunks; c += U * stride) {
    Raw<T> raw[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t cu = c + u * stride;
      if (cu < p.total_chunks) {
        int64_t r, col;
        chunk_pos(p, cu, r, col);
        load_raw<T>(p, r, col, raw[u]);
      }
    }
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      if (c + u * stride < p.total_chunks) {
        float v[16];
        to_floats<T>(raw[u], v);
        #pragma unroll
        for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
      }
    }
  }
  const uint32_t bits = block_max_bits(amax, warp_max);
  if (threadIdx.x == 0 && bits) red_max_u32(reinterpret_cast<uint32_t*>(const_cast<float*>(p.dyn_amax)), bits);
}

// ---------------------------------------------------------------- column-sum kernel


constexpr int kColTile = kDbiasColsPerTile;        // 256 columns
constexpr int kCsChunk = 8;                        // columns per thread
constexpr int kChunkLanes = kColTile / kCsChunk;   // 32: one warp spans the tile's 256 columns
constexpr int kRowLanes = kThreads / kChunkLanes;  // 8: one warp per row lane

// 8 consecutive input elements of one row, as raw bits (the vector path).
template <typename T>
struct Raw8 {
  uint4 w[sizeof(T) == 4 ? 2 : 1];
};

template <typename T>
__device__ __forceinline__ Raw8<T> load_raw8(const QuantizeParams& p, int64_t r, int64_t col) {
  Raw8<T> raw;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.in) + r * p.ld_in + col);
  raw.w[0] = __ldg(src);
  if constexpr (sizeof(T) == 4) raw.w[1] = __ldg(src + 1);
  return raw;
}

// The 8 elements at (r, col) as floats, element loads with zeros past the row end.
template <typename T>
__device__ __forceinline__ void load8_elems(const QuantizeParams& p, int64_t r, int64_t col, float (&v)[8]) {
  const int64_t base = r * p.ld_in + col;
  #pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (col + j < p.cols) {
      const uint32_t b = elem_bits<T>(p.in, base + j);
      if constexpr (std::is_same<T, __nv_bfloat16>::value) v[j] = __uint_as_float(b << 16);
      else if constexpr (std::is_same<T, __half>::value) v[j] = __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
      else v[j] = __uint_as_float(b);
    } else {
      v[j] = 0.0f;
    }
  }
}

template <typename T>
__device__ __forceinline__ void to_floats8(const Raw8<T>& raw, float (&v)[8]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(raw.w);
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else if constexpr (std::is_same<T, __half>::value) {
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
    #pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(w[i]);
  }
}

// amax, scale, cast and one 8-byte store of the 8 codes at (r, col); codes
// past cols (row padding up to ld_out) are written as zero.
template <int FMT>
__device__ __forceinline__ void cast_store8(const QuantizeParams& p, int64_t r, int64_t col, const float (&v)[8],
                                            float s, float& amax) {
  uint32_t w[2];
  #pragma unroll
  for (int i = 0; i < 4; ++i) {
    amax = fmaxf(amax, fabsf(v[2 * i]));
    amax = fmaxf(amax, fabsf(v[2 * i + 1]));
    const uint32_t h = cvt2<FMT>(v[2 * i] * s, v[2 * i + 1] * s);
    if (i & 1) w[i >> 1] |= h << 16;
    else w[i >> 1] = h;
  }
  const int64_t left = p.cols - col;
  if (left < kCsChunk) {
    #pragma unroll
    for (int j = 0; j < kCsChunk; ++j)
      if (j >= left) w[j >> 2] &= ~(0xFFu << (8 * (j & 3)));
  }
  *reinterpret_cast<uint2*>(p.out + r * p.ld_out + col) = make_uint2(w[0], w[1]);
}

template <typename T, int FMT>
__global__ void __launch_bounds__(kThreads, 3) quantize_colsum_kernel(const __grid_constant__ ColsumParams cp) {
  __shared__ uint32_t warp_max[kThreads / 32];
  __shared__ float hist_s[kHistCache];
  __shared__ __align__(16) float red[kRowLanes][kColTile];
  __shared__ int last_tile;
  // Before the dependency wait: the first block of each row split prefetches
  // its band of rows into L2 (one contiguous range when the rows are 16-byte
  // aligned), so the DRAM latency overlaps the previous kernel's tail; as in
  // the flat kernel, only inputs up to kPrefetchMaxBytes.
  if (threadIdx.x == 0 && blockIdx.x == 0 && cp.q.vec_ok) {
    const QuantizeParams& q = cp.q;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * cp.rows_per_split;
    const int64_t r1 = min(q.rows, r0 + cp.rows_per_split);
    const uint64_t total = static_cast<uint64_t>(q.rows) * static_cast<uint64_t>(q.ld_in) * sizeof(T);
    if (r1 > r0 && total <= kPrefetchMaxBytes) {
      const uint64_t bytes =
          (static_cast<uint64_t>((r1 - r0 - 1) * q.ld_in + q.cols) * sizeof(T)) & ~uint64_t(15);
      if (bytes > 0)
        prefetch_l2_bulk(static_cast<const T*>(q.in) + r0 * q.ld_in, static_cast<uint32_t>(bytes));
    }
  }
  pdl_wait();
  pdl_trigger();
  const QuantizeParams& p = cp.q;
  const uint32_t nblocks = gridDim.x * gridDim.y;
  const uint32_t bid = blockIdx.y * gridDim.x + blockIdx.x;
  const float s = scale_of(p);
  const bool do_step = p.ring && !p.defer_finalize;
  uint32_t step = 0;
  if (threadIdx.x == 0) {
    if (do_step) step = reinterpret_cast<const uint32_t*>(p.ring)[ring_step(p.H)];
    if (bid == 0 && p.scale_out) *p.scale_out = s;
  }
  if (do_step && p.H <= kHistCache && threadIdx.x < p.H) hist_s[threadIdx.x] = p.ring[threadIdx.x];

  // warp rl is row lane rl; its 32 lanes cover the tile's 256 columns, 8 each,
  // so one row of a warp is 512 contiguous bytes of bf16 input
  const int cl = threadIdx.x % kChunkLanes;
  const int rl = threadIdx.x / kChunkLanes;
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kColTile + cl * kCsChunk;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * cp.rows_per_split;
  const int64_t r1 = min(p.rows, r0 + cp.rows_per_split);
  float amax = 0.0f;
  float csum[kCsChunk];
  #pragma unroll
  for (int j = 0; j < kCsChunk; ++j) csum[j] = 0.0f;
  if (col < p.cols) {
    // U rows of this lane in flight at once, then summed and cast in row
    // order (the column sums of a lane add its rows in ascending order)
    constexpr int U = sizeof(T) == 4 ? 4 : 8;
    int64_t r = r0 + rl;
    const bool vec = p.vec_ok && col + kCsChunk <= p.cols;
    #pragma unroll 1
    for (; vec && r + (U - 1) * kRowLanes < r1; r += U * kRowLanes) {
      Raw8<T> raw[U];
      #pragma unroll
      for (int u = 0; u < U; ++u) raw[u] = load_raw8<T>(p, r + u * kRowLanes, col);
      #pragma unroll
      for (int u = 0; u < U; ++u) {
        float v[kCsChunk];
        to_floats8<T>(raw[u], v);
        #pragma unroll
        for (int j = 0; j < kCsChunk; ++j) csum[j] += v[j];
        cast_store8<FMT>(p, r + u * kRowLanes, col, v, s, amax);
      }
    }
    #pragma unroll 1
    for (; r < r1; r += kRowLanes) {
      float v[kCsChunk];
      if (vec) {
        const Raw8<T> raw = load_raw8<T>(p, r, col);
        to_floats8<T>(raw, v);
      } else {
        load8_elems<T>(p, r, col, v);
      }
      #pragma unroll
      for (int j = 0; j < kCsChunk; ++j) csum[j] += v[j];
      cast_store8<FMT>(p, r, col, v, s, amax);
    }
  } else if (col < ((p.cols + 15) & ~int64_t(15)) && col < p.ld_out) {
    // a chunk wholly in the row padding (the 16-byte rounding of cols): zeros
    for (int64_t r = r0 + rl; r < r1; r += kRowLanes)
      *reinterpret_cast<uint2*>(p.out + r * p.ld_out + col) = make_uint2(0u, 0u);
  }
  // column partials of this block: row lanes summed in lane order
  #pragma unroll
  for (int j = 0; j < kCsChunk; j += 4)
    *reinterpret_cast<float4*>(&red[rl][cl * kCsChunk + j]) =
        make_float4(csum[j], csum[j + 1], csum[j + 2], csum[j + 3]);
  const uint32_t bits = block_max_bits(amax, warp_max);  // includes a CTA barrier
  const int64_t ccol = static_cast<int64_t>(blockIdx.x) * kColTile + threadIdx.x;
  float part = 0.0f;
  #pragma unroll
  for (int y = 0; y < kRowLanes; ++y) part += red[y][threadIdx.x];
  if (ccol < p.cols) cp.partial[static_cast<int64_t>(blockIdx.y) * p.cols + ccol] = part;
  if (cp.defer_sum) {  // the GEMM that follows sums the partials
    if (threadIdx.x == 0 && p.ring) ring_tail(p, bits, nblocks, s, step, hist_s);
    return;
  }
  cta_sync();
  // Two independent tails run side by side: thread 0 the ring's, thread 32
  // the column tile's ticket.
  if (threadIdx.x == 0 && p.ring) ring_tail(p, bits, nblocks, s, step, hist_s);
  if (threadIdx.x == 32) {
    // the barrier above ordered every thread's partial before this fence
    __threadfence();
    last_tile = atomicAdd(&cp.counters[blockIdx.x], 1u) == gridDim.y - 1;
    if (last_tile) __threadfence();
  }
  cta_sync();
  if (!last_tile) return;
  if (ccol < p.cols)
    static_cast<__nv_bfloat16*>(cp.dbias)[ccol] =
        __float2bfloat16_rn(sum_partials(cp.partial + ccol, p.cols, static_cast<int>(gridDim.y)));
  if (threadIdx.x == 0) atomicExch(&cp.counters[blockIdx.x], 0u);
}

// ---------------------------------------------------------------- small kernels

__global__ void ring_set_kernel(float* ring, int H, float scale) {
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < H; i += blockDim.x) ring[i] = 0.0f;
  if (threadIdx.x == 0) {
    uint32_t* w = reinterpret_cast<uint32_t*>(ring);
    ring[ring_scale(H)] = scale;
    w[ring_step(H)] = 0u;
    w[ring_ticket(H)] = 0u;
    w[ring_scratch(H)] = 0u;
  }
}

// The pending ring step of one ring (fp8_ring_finalize): one warp.
__global__ void ring_finalize_kernel(const RingFinalize f) {
  pdl_wait();
  pdl_trigger();
  ring_finalize_warp(f, static_cast<int>(threadIdx.x));
}

__global__ void side_writes_kernel(const SideWrites w) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  for (int i = 0; i < 2; ++i) {
    if (w.copy_dst[i]) *w.copy_dst[i] = *w.copy_src[i];
    if (w.zero_dst[i]) *w.zero_dst[i] = 0.0f;
  }
}

// ---------------------------------------------------------------- launchers

// Resident blocks per SM (registers allow four); measured on a B200, four
// blocks of 2 chunks (plus the next 2 in flight) per thread stream ~18% faster
// than two blocks of 4.
constexpr int kBlocksPerSm = 4;

int64_t blocks_for(const QuantizeParams& p, int sms) {
  const int64_t want = (p.total_chunks + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sms) * kBlocksPerSm;
  return want < 1 ? 1 : (want > cap ? cap : want);
}

template <typename T, int FMT>
cudaError_t launch_q(const QuantizePair& pair, int grid, cudaStream_t s) {
  return launch_pdl(quantize_kernel<T, FMT>, dim3(grid), dim3(kThreads), 0, s, pair);
}

template <typename T, int FMT>
cudaError_t launch_cs(const ColsumParams& cp, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((cp.q.cols + kColTile - 1) / kColTile), static_cast<unsigned>(cp.R));
  return launch_pdl(quantize_colsum_kernel<T, FMT>, grid, dim3(kThreads), 0, s, cp);
}

}  // namespace

// One or two tensors over one resident wave of blocks, shared in proportion to
// their chunks; returns the grid size.
static int make_pair(const QuantizeParams* a, const QuantizeParams* b, QuantizePair* pair) {
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = num_sms(dev);
  pair->t[0] = *a;
  pair->t[1] = b ? *b : *a;
  int64_t g0 = blocks_for(*a, sms);
  int64_t g1 = b ? blocks_for(*b, sms) : 0;
  const int64_t cap = static_cast<int64_t>(sms) * kBlocksPerSm;  // one resident wave
  if (g0 + g1 > cap) {  // share the wave in proportion to the chunks
    const double f = static_cast<double>(a->total_chunks) / static_cast<double>(a->total_chunks + b->total_chunks);
    g0 = static_cast<int64_t>(f * static_cast<double>(cap) + 0.5);
    g0 = g0 < 1 ? 1 : (g0 > cap - 1 ? cap - 1 : g0);
    g1 = cap - g0;
  }
  pair->blocks0 = static_cast<int>(g0);
  const int grid = static_cast<int>(g0 + g1);
  pair->pf_blocks = sms < grid ? sms : grid;
  return grid;
}

cudaError_t launch_quantize(int in_dtype, int fmt, const QuantizeParams* a, const QuantizeParams* b,
                            cudaStream_t s) {
  QuantizePair pair;
  const int grid = make_pair(a, b, &pair);
  if (fmt == kE4M3) {
    if (in_dtype == kBF16) return launch_q<__nv_bfloat16, kE4M3>(pair, grid, s);
    if (in_dtype == kFP16) return launch_q<__half, kE4M3>(pair, grid, s);
    return launch_q<float, kE4M3>(pair, grid, s);
  }
  if (in_dtype == kBF16) return launch_q<__nv_bfloat16, kE5M2>(pair, grid, s);
  if (in_dtype == kFP16) return launch_q<__half, kE5M2>(pair, grid, s);
  return launch_q<float, kE5M2>(pair, grid, s);
}

cudaError_t launch_amax(int in_dtype, const QuantizeParams* a, const QuantizeParams* b, cudaStream_t s) {
  QuantizePair pair;
  const int grid = make_pair(a, b, &pair);
  if (in_dtype == kBF16) return launch_pdl(amax_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, s, pair);
  if (in_dtype == kFP16) return launch_pdl(amax_kernel<__half>, dim3(grid), dim3(kThreads), 0, s, pair);
  return launch_pdl(amax_kernel<float>, dim3(grid), dim3(kThreads), 0, s, pair);
}

cudaError_t launch_quantize_colsum(int in_dtype, int fmt, const ColsumParams& cp, cudaStream_t s) {
  if (fmt == kE4M3) {
    if (in_dtype == kBF16) return launch_cs<__nv_bfloat16, kE4M3>(cp, s);
    if (in_dtype == kFP16) return launch_cs<__half, kE4M3>(cp, s);
    return launch_cs<float, kE4M3>(cp, s);
  }
  if (in_dtype == kBF16) return launch_cs<__nv_bfloat16, kE5M2>(cp, s);
  if (in_dtype == kFP16) return launch_cs<__half, kE5M2>(cp, s);
  return launch_cs<float, kE5M2>(cp, s);
}

cudaError_t launch_ring_set(float* ring, int H, float scale, cudaStream_t s) {
  return launch_pdl(ring_set_kernel, dim3(1), dim3(128), 0, s, ring, H, scale);
}

cudaError_t launch_ring_finalize(const RingFinalize& f, cudaStream_t s) {
  return launch_pdl(ring_finalize_kernel, dim3(1), dim3(32), 0, s, f);
}

cudaError_t launch_side_writes(const SideWrites& w, cudaStream_t s) {
  return launch_pdl(side_writes_kernel, dim3(1), dim3(32), 0, s, w);
}

}  // namespace fp8lin
