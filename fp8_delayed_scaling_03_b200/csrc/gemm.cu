// gemm.cu -- dense FP8 GEMM with fused dequant + bias epilogue, sm_100a.
//
//   D[i, j] = bf16_rne( (sum_k A(i,k) B(j,k)) * 1/(scale_a scale_b) + bias[j] )
//
// The pages' kernel (AstrAI commit log, csrc @2eeac02: 128x128 CTA of
// mma.sync warps fed by cp.async, PRMT byte transposes for the "crosswise"
// operands of dX/dW) is prior art for sm_89; this is the Blackwell design:
//   * one persistent CTA per SM, tiles in a grouped raster so the CTAs working
//     at the same time share operand stripes in L2 (astrai @4019dda and csrc
//     @2eeac02 describe grouped rasterization for the same reason);
//   * warp 0 lane 0: TMA producer.  128x128-byte boxes with 128-byte swizzle
//     land in a STAGES-deep shared-memory ring; out-of-range rows, columns and
//     k come back as zeros, so no tail predication exists in the mainloop;
//   * warp 1 lane 0: tcgen05.mma.cta_group::1.kind::f8f6f4 issuer, M=128,
//     N=BN, K=32 per instruction, fp32 accumulator in TMEM (two accumulators
//     of BN columns, so the epilogue of tile t overlaps the mainloop of t+1);
//   * the transposed ("crosswise") operands of dX and dW are read in place:
//     the smem descriptor and instruction descriptor mark them MN-major, which
//     tcgen05 supports for E4M3/E5M2 -- no transpose pass, no copy;
//   * warps 2-9: epilogue, two warps per TMEM lane quadrant splitting the
//     tile's columns.  Per 32-column step: tcgen05.ld 32 lanes x 32 columns,
//     multiply by the dequant factor, add the bias in fp32 (bf16, or fp8 /
//     bias_scale; one load per lane, broadcast by shuffle), one RNE rounding
//     to bf16 (astrai @4019dda fused-bias bullet), then the 32x32 bf16 block is
//     staged in a 64-byte-swizzled shared slab and written by a TMA store
//     (coalesced, asynchronous, clipped at the matrix edge) -- the pages'
//     kernel also staged its epilogue through shared memory for write
//     efficiency (astrai @4019dda, epilogue bullet).  The accumulator is handed
//     back to the MMA warp right after its last TMEM read.  Output strides that
//     TMA cannot address (row pitch not a multiple of 16 bytes) take guarded
//     per-element stores instead.
// Every mbarrier wait is bounded (see device.cuh); a timeout records
// FP8_ERR_DEVICE_TIMEOUT and the CTA winds down instead of hanging.
#include "device.cuh"
#include "internal.h"
#include "launch.h"

namespace fp8lin {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 128;  // fp8 elements (= bytes) of k per stage
constexpr int kUmmaK = 32;
constexpr int kThreads = 320;       // 10 warps: TMA, MMA, 8 epilogue
constexpr int kEpiWarps = 8;
constexpr int kEpiCols = 32;        // columns per epilogue step
constexpr int kEpiSlab = 32 * kEpiCols * 2;  // one 32x32 bf16 staging slab

template <int BN>
struct Cfg {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kEpiBytes = kEpiWarps * 2 * kEpiSlab;  // two slabs per epilogue warp
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kStages * kStageBytes + kEpiBytes + kBarBytes + 1024;
  static_assert(BN == 128 || BN == 256, "BN");
};

__device__ __forceinline__ void tile_coords(const GemmParams& p, int t, int& tm, int& tn) {
  const int per_group = p.raster_group * p.tiles_n;
  const int g = t / per_group;
  const int first_m = g * p.raster_group;
  const int gm = min(p.raster_group, p.tiles_m - first_m);
  const int r = t - g * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float bias_value(const GemmParams& p, int j, float binv) {
  if (p.bias_kind == 1)
    return __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const unsigned short*>(p.bias) + j)) << 16);
  const uint16_t b = __ldg(static_cast<const uint8_t*>(p.bias) + j);
  const float2 f = p.bias_kind == 2 ? dec_e4m3x2(b) : dec_e5m2x2(b);
  return f.x * binv;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                    const __grid_constant__ CUtensorMap tma_d, const GemmParams p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint8_t* sEpi = sB + C::kStages * C::kBBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::kEpiBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    if (p.k_blocks > 0) {
      prefetch_tmap(&tma_a);
      prefetch_tmap(&tma_b);
    }
    if (p.tma_store) prefetch_tmap(&tma_d);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  // Everything above overlaps the previous kernel on the stream; from here on
  // its results (operands, scales) are read.
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 64) {
    for (int i = 0; i < 2; ++i) {
      if (p.side.copy_dst[i]) *p.side.copy_dst[i] = *p.side.copy_src[i];
      if (p.side.zero_dst[i]) *p.side.zero_dst[i] = 0.0f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < p.num_tiles && !*abort_flag; t += gridDim.x) {
        int tm, tn;
        tile_coords(p, t, tm, tn);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag)) break;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          uint8_t* a_dst = sA + stage * C::kABytes;
          uint8_t* b_dst = sB + stage * C::kBBytes;
          if (p.a_major == 0) tma_load_2d(a_dst, &tma_a, &full[stage], kb * kBK, tm * kBM);
          else                tma_load_2d(a_dst, &tma_a, &full[stage], tm * kBM, kb * kBK);
          if (p.b_major == 0) {
            tma_load_2d(b_dst, &tma_b, &full[stage], kb * kBK, tn * BN);
          } else {
            #pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              tma_load_2d(b_dst + h * 128 * kBK, &tma_b, &full[stage], tn * BN + h * 128, kb * kBK);
          }
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < p.num_tiles && !*abort_flag; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_base = smem_u32(sB + stage * C::kBBytes);
          #pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            // K-major: advance 32 bytes along the swizzled 128-byte row.
            // MN-major: advance 32 k-rows of 128 bytes (4 swizzle atoms).
            const uint64_t ad = p.a_major == 0
                                    ? smem_desc_sw128(a_base + kk * kUmmaK, 16, 1024)
                                    : smem_desc_sw128(a_base + kk * kUmmaK * 128, 128 * kBK, 1024);
            const uint64_t bd = p.b_major == 0
                                    ? smem_desc_sw128(b_base + kk * kUmmaK, 16, 1024)
                                    : smem_desc_sw128(b_base + kk * kUmmaK * 128, 128 * kBK, 1024);
            umma_f8f6f4(d_tmem, ad, bd, p.idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0..7
    const int q = warp & 3;                  // TMEM lane quadrant this warp may access
    const int half = ew >> 2;                // which half of the tile's columns
    const int row_in_tile = q * 32 + lane;
    const float inv = 1.0f / (*p.scale_a * *p.scale_b);
    const float binv = (p.bias_kind >= 2) ? 1.0f / *p.bias_scale : 1.0f;
    const bool have_k = p.k_blocks > 0;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* slabs = sEpi + ew * 2 * kEpiSlab;
    int slab = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    __nv_bfloat16* D = static_cast<__nv_bfloat16*>(p.d);
    constexpr int kSteps = BN / 2 / kEpiCols;
    for (int t = blockIdx.x; t < p.num_tiles && !*abort_flag; t += gridDim.x) {
      int tm, tn;
      tile_coords(p, t, tm, tn);
      if (!mbar_wait(&tfull[acc], acc_phase, p.status, abort_flag)) break;
      tc_fence_after();
      const int row = tm * kBM + row_in_tile;
      const int col_half = tn * BN + half * (BN / 2);
      const int live_steps = min(kSteps, max(0, (p.n - col_half + kEpiCols - 1) / kEpiCols));
      #pragma unroll 1
      for (int st = 0; st < kSteps; ++st) {
        const int col0 = col_half + st * kEpiCols;
        uint32_t r[32];
        if (st < live_steps) {
          __syncwarp();  // tcgen05.ld is .sync.aligned
          tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(acc * BN + half * (BN / 2) + st * kEpiCols), r);
          tmem_ld_wait();
        }
        if (st == kSteps - 1) {  // last TMEM read of this accumulator: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (st >= live_steps) continue;
        float bl = 0.0f;
        if (p.bias_kind && col0 + lane < p.n) bl = bias_value(p, col0 + lane, binv);
        float v[32];
        #pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = (have_k ? __uint_as_float(r[j]) : 0.0f) * inv;
          if (p.bias_kind) v[j] += __shfl_sync(0xFFFFFFFFu, bl, j);
        }
        if (p.tma_store) {
          uint8_t* buf = slabs + slab * kEpiSlab;
          if (lane == 0) bulk_wait_read<1>();  // the store that last read this slab is done
          __syncwarp();
          // row `lane` of the 32x32 block, 4 chunks of 16 bytes, 64-byte swizzle
          #pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 o = make_uint4(pack_bf16x2(v[8 * c + 0], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                 pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
            const int phys = c ^ ((lane >> 1) & 3);
            *reinterpret_cast<uint4*>(buf + lane * 64 + phys * 16) = o;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tma_d, buf, col0, tm * kBM + q * 32);
            bulk_commit();
          }
          slab ^= 1;
        } else if (row < p.m) {
          __nv_bfloat16* drow = D + static_cast<int64_t>(row) * p.ldd;
          #pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < p.n) drow[col0 + j] = __float2bfloat16_rn(v[j]);
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (p.tma_store && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td, const GemmParams& p,
                      cudaStream_t s) {
  using C = Cfg<BN>;
  int dev = 0;
  cudaGetDevice(&dev);
  static bool configured[64] = {};
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(fp8_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int sms = num_sms(dev);
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  return launch_pdl(fp8_gemm_kernel<BN>, dim3(grid), dim3(kThreads), C::kSmem, s, ta, tb, td, p);
}

}  // namespace

cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td, GemmParams p, int bn,
                        cudaStream_t s) {
  if (bn == 256) return launch_bn<256>(ta, tb, td, p, s);
  return launch_bn<128>(ta, tb, td, p, s);
}

}  // namespace fp8lin
