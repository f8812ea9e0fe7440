// dbias.cu -- bias gradient: dbias[n] = bf16( sum_m g[m, n] ), fp32 sums.
//
// Computed only when the bias needs a gradient (AstrAI commit log, astrai
// @4019dda, bullet on the unconditional column sum).  A pre-quantized g is
// dequantized element by element before the sum (astrai/extension/ops
// @057c0d3, grad dtype bullet).
//
// HBM-bound: one read of g.  Grid (column tiles of 256, R row splits); a
// block of 8 x 32 threads streams rows of its split with 16-byte loads (8
// columns per thread, eight rows' loads in flight before any is summed --
// one row at a time left HBM at 0.31 of its bandwidth at 4096 x 11008, eight
// reach 0.71 on a B200), reduces its 8 row lanes in shared memory in a fixed
// order and writes 256 fp32 partials.  The block that draws the last ticket
// of its column tile sums the R partials in a fixed order (partials.cuh), so
// the result does not depend on block scheduling, and rezeroes the tile's
// counter.
#include <cstring>

#include "device.cuh"
#include "internal.h"
#include "launch.h"
#include "partials.cuh"

namespace fp8lin {
namespace {

constexpr int kCols = kDbiasColsPerTile;  // 256 = 32 lanes x 8 columns
constexpr int kRowLanes = 8;

template <int DT>
__device__ __forceinline__ void load8(const DbiasParams& p, int64_t r, int64_t c, float inv, float (&v)[8]) {
  const int64_t idx = r * p.ldg + c;
  const bool full = c + 8 <= p.N;
  if constexpr (DT == kBF16) {
    const uint16_t* g = static_cast<const uint16_t*>(p.g);
    if (p.vec_ok && full) {
      uint4 q = __ldg(reinterpret_cast<const uint4*>(g + idx));
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&q);
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
      #pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = (c + j < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(g + idx + j)) << 16) : 0.0f;
    }
  } else if constexpr (DT == kFP16) {
    const __half* g = static_cast<const __half*>(p.g);
    if (p.vec_ok && full) {
      uint4 q = __ldg(reinterpret_cast<const uint4*>(g + idx));
      const __half2* h = reinterpret_cast<const __half2*>(&q);
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
    } else {
      #pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (c + j < p.N) ? __half2float(g[idx + j]) : 0.0f;
    }
  } else if constexpr (DT == kFP32) {
    const float* g = static_cast<const float*>(p.g);
    if (p.vec_ok && full) {
      float4 a = __ldg(reinterpret_cast<const float4*>(g + idx));
      float4 b = __ldg(reinterpret_cast<const float4*>(g + idx) + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
      #pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (c + j < p.N) ? __ldg(g + idx + j) : 0.0f;
    }
  } else {
    const uint8_t* g = static_cast<const uint8_t*>(p.g);
    uint32_t w[2];
    if (p.vec_ok && full) {
      uint2 q = __ldg(reinterpret_cast<const uint2*>(g + idx));
      w[0] = q.x;
      w[1] = q.y;
    } else {
      w[0] = w[1] = 0;
      #pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c + j < p.N) w[j >> 2] |= static_cast<uint32_t>(__ldg(g + idx + j)) << (8 * (j & 3));
    }
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t pair = static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1)));
      const float2 f = DT == kDtE4M3 ? dec_e4m3x2(pair) : dec_e5m2x2(pair);
      v[2 * i] = f.x * inv;
      v[2 * i + 1] = f.y * inv;
    }
  }
}

// The raw bytes of 8 columns of one row (vector path), and their values.
template <int DT>
struct Raw8 {
  uint4 w[DT == kFP32 ? 2 : 1];
};

// Vector path only (p.vec_ok and 8 whole columns from c).
template <int DT>
__device__ __forceinline__ Raw8<DT> load_raw8(const DbiasParams& p, int64_t r, int64_t c) {
  Raw8<DT> raw;
  const int64_t idx = r * p.ldg + c;
  if constexpr (DT == kFP32) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(p.g) + idx);
    raw.w[0] = __ldg(src);
    raw.w[1] = __ldg(src + 1);
  } else if constexpr (DT == kBF16 || DT == kFP16) {
    raw.w[0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.g) + idx));
  } else {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(p.g) + idx));
    raw.w[0] = make_uint4(q.x, q.y, 0u, 0u);
  }
  return raw;
}

template <int DT>
__device__ __forceinline__ void to_floats8(const Raw8<DT>& raw, float inv, float (&v)[8]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(raw.w);
  if constexpr (DT == kFP32) {
    #pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(w[j]);
  } else if constexpr (DT == kBF16) {
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else if constexpr (DT == kFP16) {
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t pair = static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1)));
      const float2 f = DT == kDtE4M3 ? dec_e4m3x2(pair) : dec_e5m2x2(pair);
      v[2 * i] = f.x * inv;
      v[2 * i + 1] = f.y * inv;
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(kRowLanes * 32) dbias_kernel(const DbiasParams p) {
  __shared__ float red[kRowLanes][kCols];
  __shared__ int last;
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x & 31;
  const int ty = threadIdx.x >> 5;
  const int64_t c_base = static_cast<int64_t>(blockIdx.x) * kCols;
  const int64_t c = c_base + tx * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * p.rows_per_split;
  const int64_t r1 = min(p.M, r0 + p.rows_per_split);
  const float inv = (DT == kDtE4M3 || DT == kDtE5M2) ? 1.0f / *p.g_scale : 1.0f;

  float acc[8];
  #pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
  if (c < p.N) {
    // U rows of this lane in flight at once (their loads issued before any is
    // summed: a lone 16-byte load per row leaves HBM mostly idle), then summed
    // in row order -- the same order as one row at a time
    constexpr int U = DT == kFP32 ? 4 : 8;
    int64_t r = r0 + ty;
    const bool vec = p.vec_ok && c + 8 <= p.N;
    #pragma unroll 1
    for (; vec && r + (U - 1) * kRowLanes < r1; r += U * kRowLanes) {
      Raw8<DT> raw[U];
      #pragma unroll
      for (int u = 0; u < U; ++u) raw[u] = load_raw8<DT>(p, r + u * kRowLanes, c);
      #pragma unroll
      for (int u = 0; u < U; ++u) {
        float v[8];
        to_floats8<DT>(raw[u], inv, v);
        #pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += v[j];
      }
    }
    for (; r < r1; r += kRowLanes) {
      float v[8];
      load8<DT>(p, r, c, inv, v);
      #pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += v[j];
    }
  }
  #pragma unroll
  for (int j = 0; j < 8; ++j) red[ty][tx * 8 + j] = acc[j];
  cta_sync();

  const int64_t col = c_base + threadIdx.x;
  float s = 0.0f;
  #pragma unroll
  for (int y = 0; y < kRowLanes; ++y) s += red[y][threadIdx.x];
  if (col < p.N) p.partial[static_cast<int64_t>(blockIdx.y) * p.N + col] = s;
  cta_sync();
  if (threadIdx.x == 0) {
    // the barrier above ordered every thread's partial before this fence
    __threadfence();
    last = atomicAdd(&p.counters[blockIdx.x], 1u) == static_cast<unsigned>(p.R - 1);
    if (last) __threadfence();
  }
  cta_sync();
  if (!last) return;
  if (col < p.N)
    static_cast<__nv_bfloat16*>(p.dbias)[col] = __float2bfloat16_rn(sum_partials(p.partial + col, p.N, p.R));
  if (threadIdx.x == 0) atomicExch(&p.counters[blockIdx.x], 0u);
}

}  // namespace

namespace {

// Row splits of an [M, N] column sum over 256-column tiles: about `blocks`
// (col tile, row split) blocks in total (at most `blocks` with at_most, the
// row splits rounded down instead of up), each split at least min_rows rows.
void split_geometry(int64_t M, int64_t N, int64_t blocks, int64_t min_rows, bool at_most, int* R,
                    int64_t* rows_per_split) {
  const int64_t col_tiles = (N + kCols - 1) / kCols;
  const int64_t ct = col_tiles > 0 ? col_tiles : 1;
  int64_t r = at_most ? blocks / ct : (blocks + ct - 1) / ct;
  const int64_t rmax = (M + min_rows - 1) / min_rows;
  if (r > rmax) r = rmax;
  if (r < 1) r = 1;
  int64_t rps = (M + r - 1) / r;
  if (rps < 1) rps = 1;
  r = (M + rps - 1) / rps;
  if (r < 1) r = 1;
  *R = static_cast<int>(r);
  *rows_per_split = rps;
}

}  // namespace

// The dbias kernel: at most 444 blocks (three per SM of a B200; its 48
// registers would allow five), at least 64 rows each.  Measured on a B200
// (bf16 g): 0.75 / 0.50 / 0.32 of HBM at 4096x11008 / 2048x6912 / 2048x4096
// against 0.72 / 0.40 / 0.28 with about 296 blocks; at most 592 or 740
// blocks of >= 32 rows were slower than 444 on every shape.
void dbias_geometry(int64_t M, int64_t N, int* R, int64_t* rows_per_split) {
  split_geometry(M, N, 444, 64, true, R, rows_per_split);
}

// The column-sum quantize (standalone, or in the linear backward where a GEMM
// launch finishes its sums): at most 444 blocks (one resident wave: three per SM), at least
// 32 rows each.  Measured on a B200 in the dim1024 and production steps: 592
// blocks (1.33 waves) were 0.7 % slower in the dim1024 step; 16-row or
// 1184-block splits were slower with the kernel's earlier form.
void colsum_geometry(int64_t M, int64_t N, int* R, int64_t* rows_per_split) {
  split_geometry(M, N, 444, 32, true, R, rows_per_split);
}

cudaError_t launch_dbias(const DbiasParams& p, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((p.N + kCols - 1) / kCols), static_cast<unsigned>(p.R));
  const int threads = kRowLanes * 32;
  switch (p.dtype) {
    case kBF16: return launch_pdl(dbias_kernel<kBF16>, grid, dim3(threads), 0, s, p);
    case kFP16: return launch_pdl(dbias_kernel<kFP16>, grid, dim3(threads), 0, s, p);
    case kFP32: return launch_pdl(dbias_kernel<kFP32>, grid, dim3(threads), 0, s, p);
    case kDtE4M3: return launch_pdl(dbias_kernel<kDtE4M3>, grid, dim3(threads), 0, s, p);
    default: return launch_pdl(dbias_kernel<kDtE5M2>, grid, dim3(threads), 0, s, p);
  }
}

}  // namespace fp8lin

// ---------------------------------------------------------------- no-allocation variant
//
// fp8_dbias_noalloc: the same bias-gradient kernel with its scratch (the R x N
// fp32 partials and the per-tile counters) in a fixed array compiled into this
// library instead of a caller workspace.  For callers that cannot allocate
// device memory themselves -- code running under a memory manager it does not
// control (a plugin inside a serving runtime with a fixed device-memory
// budget, a C caller with no access to the framework's caching allocator) --
// and so have no workspace to pass.

#include <mutex>

#include "fp8lin.h"

namespace fp8lin {
namespace {

// 1 MiB, held by every GPU that loads this library until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;
static __device__ __align__(256) unsigned char g_dbias_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
unsigned char* g_noalloc_ptr[64] = {};

// Device address of g_dbias_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
cudaError_t noalloc_scratch(int dev, unsigned char** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_dbias_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace fp8lin

extern "C" int fp8_dbias_noalloc(const void* g, int g_dtype, int64_t M, int64_t N, int64_t ldg, const float* g_scale,
                                 void* dbias, fp8_stream_t stream) {
  using namespace fp8lin;
  const bool fp8_in = g_dtype == FP8_DT_E4M3 || g_dtype == FP8_DT_E5M2;
  const bool wide = g_dtype == FP8_DT_BF16 || g_dtype == FP8_DT_FP16 || g_dtype == FP8_DT_FP32;
  const int64_t kMax = (int64_t(1) << 31) - 1;
  if (M < 0 || N < 0 || M > kMax || N > kMax) return FP8_ERR_INVALID_ARG;
  if (!fp8_in && !wide) return FP8_ERR_INVALID_ARG;
  const size_t esz = g_dtype == FP8_DT_FP32 ? 4 : (fp8_in ? 1 : 2);
  if (!g || !dbias || ldg < N || reinterpret_cast<uintptr_t>(g) % esz || reinterpret_cast<uintptr_t>(dbias) % 2)
    return FP8_ERR_INVALID_ARG;
  if (fp8_in && !g_scale) return FP8_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FP8_OK;
  const size_t need = fp8_dbias_workspace_bytes(M, N);
  if (need > kNoAllocScratchBytes) return FP8_ERR_TOO_LARGE;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  unsigned char* scratch = nullptr;
  if ((e = noalloc_scratch(dev, &scratch)) != cudaSuccess) return record_cuda_error(e);
  DbiasParams p;
  std::memset(&p, 0, sizeof(p));
  p.g = g;
  p.dtype = g_dtype;
  p.M = M;
  p.N = N;
  p.ldg = ldg;
  p.g_scale = g_scale;
  p.dbias = dbias;
  dbias_geometry(M, N, &p.R, &p.rows_per_split);
  const size_t part = (static_cast<size_t>(p.R) * static_cast<size_t>(N) * 4u + 15u) & ~size_t(15);
  p.partial = reinterpret_cast<float*>(scratch);
  p.counters = reinterpret_cast<unsigned*>(scratch + part);
  p.vec_ok = fp8_in ? (reinterpret_cast<uintptr_t>(g) % 8 == 0 && ldg % 8 == 0)
                    : (reinterpret_cast<uintptr_t>(g) % 16 == 0 && (static_cast<size_t>(ldg) * esz) % 16 == 0);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the tile counters must start
  // at zero (the kernel also leaves them at zero when it completes).
  const size_t tiles = static_cast<size_t>((N + kDbiasColsPerTile - 1) / kDbiasColsPerTile);
  if ((e = cudaMemsetAsync(p.counters, 0, tiles * sizeof(unsigned), st)) != cudaSuccess) return record_cuda_error(e);
  if ((e = launch_dbias(p, st)) != cudaSuccess) return record_cuda_error(e);
  return FP8_OK;
}
