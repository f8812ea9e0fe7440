// gemm.cu -- dense FP8 GEMM with fused dequant + bias epilogue, sm_100a.
//
//   D[i, j] = bf16_rne( (sum_k A(i,k) B(j,k)) * 1/(scale_a scale_b) + bias[j] )
//
// The pages' kernel (AstrAI commit log, csrc @2eeac02: 128x128 CTA of
// mma.sync warps fed by cp.async, PRMT byte transposes for the "crosswise"
// operands of dX/dW) is prior art for sm_89; this is the Blackwell design:
//   * persistent CTAs (or CTA pairs), tiles in a grouped raster so the CTAs
//     working at the same time share operand stripes in L2 (astrai @4019dda
//     and csrc @2eeac02 describe grouped rasterization for the same reason);
//   * warp 0 lane 0: TMA producer.  128x128-byte boxes with 128-byte swizzle
//     land in a STAGES-deep shared-memory ring; out-of-range rows, columns and
//     k come back as zeros, so no tail predication exists in the mainloop;
//   * warp 1 lane 0: tcgen05.mma kind::f8f6f4 issuer, K=32 per instruction,
//     fp32 accumulators in TMEM (two of them, so the epilogue of tile t
//     overlaps the mainloop of t+1);
//   * single-CTA tiles are 128 x BN.  Pair tiles (kPair) are 256 x 256 over a
//     cluster of two CTAs: each CTA loads its 128 rows of A and 128 rows of B,
//     the even CTA issues 2-SM MMAs (cta_group::2, M=256) that read both CTAs'
//     shared memory, and each CTA's TMEM holds its 128 x 256 accumulator
//     slice.  Per MMA cycle a CTA then moves 2/3 of the operand bytes of a
//     128x256 single-CTA tile through shared memory and L2;
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
//     back to the MMA warp right after its last TMEM read.  Output rows that
//     TMA cannot address (row pitch or row end not on 16 bytes) take guarded
//     per-element stores instead.
// Every mbarrier wait is bounded (see device.cuh); a timeout records
// FP8_ERR_DEVICE_TIMEOUT and the CTA winds down instead of hanging.
#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "launch.h"
#include "partials.cuh"
#include "ring.cuh"

namespace fp8lin {
namespace {

constexpr int kBM = 128;              // accumulator rows per CTA
constexpr int kBK = 128;              // fp8 elements (= bytes) of k per stage
constexpr int kUmmaK = 32;
constexpr int kThreads = 320;         // 10 warps: TMA, MMA, 8 epilogue
constexpr int kEpiWarps = 8;
constexpr int kEpiCols = 32;          // columns per epilogue step
constexpr int kEpiSlab = 32 * kEpiCols * 2;  // one 32x32 bf16 staging slab
constexpr int kRingBytes = 192 * 1024;       // operand stages
// A split-K partial: 128 x 128 fp32 as [column / 4][row][4] (a warp's 16-byte
// accesses for one column quad are 512 contiguous bytes, conflict-free).  The
// split kernel gives the top (S - 1) partials' worth of the operand ring to a
// partial region: rank r > 0 parks its partial in slot 0 of its own region
// and one bulk copy moves it to slot r - 1 of rank 0's, completing on rank 0's
// barrier; the ring keeps (192 KB - (S - 1) 64 KB) / 32 KB stages (4 for S = 2,
// 2 for S = 3).
constexpr int kPartBytes = kBM * 128 * 4;
constexpr int kMaxSplit = 3;
// Stream-K fixup: the finishing CTA's epilogue warps stage the partials of a
// cut tile in the operand ring (free by then: the owner part is the CTA's
// last work item), kSkStageBytes per warp, one 4 KB block per 32-column step
// and partial; at most kSkMaxParts partials per tile (the planner's bound).
constexpr int kSkBlock = 32 * kEpiCols * 4;
constexpr int kSkStageBytes = kRingBytes / kEpiWarps;
constexpr int kSkMaxParts = kSkStageBytes / kSkBlock;
static_assert(kSkMaxParts == 6, "stream-K stage: 24 KB per epilogue warp");
static_assert((kMaxSplit - 1) * kPartBytes < kRingBytes, "partials leave room for operand stages");

template <int BN, bool kPair>
struct Cfg {
  static constexpr int kTileM = kPair ? 2 * kBM : kBM;    // rows of a (pair) tile
  static constexpr int kBRows = kPair ? BN / 2 : BN;      // rows of B this CTA loads
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = kBRows * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = kRingBytes / kStageBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kEpiBytes = kEpiWarps * 2 * kEpiSlab;  // two slabs per epilogue warp
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kStages * kStageBytes + kEpiBytes + kBarBytes + 1024;
  static constexpr int kTempty = kPair ? 2 * kEpiWarps : kEpiWarps;
  static_assert(BN == 128 || BN == 256, "BN");
  static_assert(!kPair || BN == 256, "pair tiles are 256 x 256");
};

// Global tile index -> (problem, tile row, tile column).  Problem 0's tiles
// come first; within a problem the tiles go in groups of raster_group tile
// rows, column by column.
// Fields of the problem a tile belongs to are read as pi ? pr[1].f : pr[0].f:
// two fixed-offset parameter reads instead of one at a run-time offset.
#define FP8_PR(f) (pi ? p.pr[1].f : p.pr[0].f)

__device__ __forceinline__ int tile_coords(const GemmParams& p, int t, int& tb, int& tm, int& tn) {
  const int pi = t >= p.tiles0 ? 1 : 0;
  if (pi) t -= p.tiles0;
  // batches one after another, each with its own raster
  const int per_batch = FP8_PR(tiles_m) * FP8_PR(tiles_n);
  tb = t / per_batch;
  t -= tb * per_batch;
  const int raster_group = FP8_PR(raster_group);
  const int per_group = raster_group * FP8_PR(tiles_n);
  const int g = t / per_group;
  const int first_m = g * raster_group;
  const int gm = min(raster_group, FP8_PR(tiles_m) - first_m);
  const int r = t - g * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
  return pi;
}

// The tile a schedule slot holds (-1: none).
__device__ __forceinline__ int slot_tile(const GemmParams& p, int slot) {
  if (!p.use_order) return slot;
  const uint16_t t = p.order[slot];
  return t == kNoTile ? -1 : static_cast<int>(t);
}

// ---------------------------------------------------------------- work items
// One work item of a CTA (or pair): k-blocks [kb_lo, kb_hi) of tile t.
//   kFull    the whole tile: its own epilogue;
//   kPartial a later part of a stream-K tile: the fp32 accumulator goes to
//            this CTA's partial slot, then its epilogue warps raise their flags;
//   kOwner   the part holding a stream-K tile's first k-block: the partials of
//            CTAs part0 .. part0 + nparts - 1 (the ranges right after this
//            CTA's, which start with them) are added, in CTA order, before the
//            epilogue.
// A CTA's stream-K range runs [tail of one tile][whole tiles][head of another]:
// its one partial (the tail) is stored first and its owner part (the head)
// comes last, so an owner only waits for partials written at the start of
// later CTAs' ranges, and no CTA waits while holding a partial -- no cycle.
enum : int { kFull = 0, kOwner = 1, kPartial = 2 };
struct Work {
  int t, kb_lo, kb_hi, kind, part0, nparts;
};
struct Sched {
  int slot;        // next data-parallel slot
  int64_t u, ue;   // next stream-K k-block unit, end of this CTA's range
};

__device__ __forceinline__ int64_t sk_begin(const GemmParams& p, int c) {
  return static_cast<int64_t>(c) * p.sk_total / p.sk_ctas;
}
// The CTA whose stream-K range holds unit u: the largest c with
// floor(c total / ctas) <= u, i.e. c = ceil((u + 1) ctas / total) - 1.
__device__ __forceinline__ int sk_cta_of(const GemmParams& p, int64_t u) {
  return static_cast<int>(((u + 1) * p.sk_ctas + p.sk_total - 1) / p.sk_total) - 1;
}

template <bool kSk>
__device__ __forceinline__ void sched_init(const GemmParams& p, int unit, Sched& s) {
  s.slot = unit;
  s.u = s.ue = 0;
  if (kSk && unit < p.sk_ctas) {
    s.u = sk_begin(p, unit);
    s.ue = sk_begin(p, unit + 1);
  }
}

template <bool kSk>
__device__ __forceinline__ bool sched_next(const GemmParams& p, int unit, int units, Sched& s, Work& w) {
  while (s.slot < p.nslots) {
    const int t = slot_tile(p, s.slot);
    s.slot += units;
    if (t < 0) continue;
    w.t = t;
    w.kb_lo = 0;
    w.kb_hi = t >= p.tiles0 ? p.pr[1].k_blocks : p.pr[0].k_blocks;
    w.kind = kFull;
    w.part0 = 0;
    w.nparts = 0;
    return true;
  }
  if (!kSk || s.u >= s.ue) return false;
  // stream-K unit -> (tile, k-block); problem 0's stream-K tiles come first
  int t, kbt;
  int64_t ut;  // the tile's first unit
  if (s.u < p.sk_u0) {
    kbt = p.pr[0].k_blocks;
    t = p.dp_tiles + static_cast<int>(s.u / kbt);
    ut = static_cast<int64_t>(t - p.dp_tiles) * kbt;
  } else {
    kbt = p.pr[1].k_blocks;
    const int t1 = max(p.dp_tiles, p.tiles0);
    t = t1 + static_cast<int>((s.u - p.sk_u0) / kbt);
    ut = p.sk_u0 + static_cast<int64_t>(t - t1) * kbt;
  }
  const int kb = static_cast<int>(s.u - ut);
  const int take = static_cast<int>(min(static_cast<int64_t>(kbt - kb), s.ue - s.u));
  s.u += take;
  w.t = t;
  w.kb_lo = kb;
  w.kb_hi = kb + take;
  w.part0 = unit + 1;
  w.nparts = 0;
  if (kb > 0) {
    w.kind = kPartial;
  } else if (take == kbt) {
    w.kind = kFull;
  } else {
    w.kind = kOwner;
    w.nparts = sk_cta_of(p, ut + kbt - 1) - unit;
  }
  return true;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// a[i] for a register array and a run-time i, without indexing (which would
// move the array to local memory).
template <int N>
__device__ __forceinline__ float pick(const float (&a)[N], int i) {
  float r = a[0];
  #pragma unroll
  for (int k = 1; k < N; ++k) r = (i == k) ? a[k] : r;
  return r;
}

__device__ __forceinline__ float bias_value(const void* bias, int bias_kind, int j, float binv) {
  if (bias_kind == 1)
    return __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const unsigned short*>(bias) + j)) << 16);
  const uint16_t b = __ldg(static_cast<const uint8_t*>(bias) + j);
  const float2 f = bias_kind == 2 ? dec_e4m3x2(b) : dec_e5m2x2(b);
  return f.x * binv;
}

// dbias[c] = bf16(fixed-order sum of the R partials of column c) for the
// columns c = 32 * (blockIdx.x + k * gridDim.x) + lane: one warp per CTA,
// 32 consecutive columns (coalesced rows of partials) at a time.
__device__ __forceinline__ void dbias_finish_warp(const DbiasFinish& f, int lane) {
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * 32 + lane; c < f.cols;
       c += static_cast<int64_t>(gridDim.x) * 32)
    static_cast<__nv_bfloat16*>(f.dbias)[c] = __float2bfloat16_rn(sum_partials(f.partial + c, f.cols, f.R));
}

// kSk: the stream-K build (its work items, partial slots and fixup); the
// data-parallel build carries none of that code.
template <int BN, bool kPair, bool kSplit, bool kSk>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap tb0,
                    const __grid_constant__ CUtensorMap td0, const __grid_constant__ CUtensorMap ta1,
                    const __grid_constant__ CUtensorMap tb1, const __grid_constant__ CUtensorMap td1,
                    const __grid_constant__ GemmParams p) {
  static_assert(!kSplit || (BN == 128 && !kPair), "split-K runs 128 x 128 single-CTA tiles");
  using C = Cfg<BN, kPair>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nsplit = kSplit ? p.split : 1;
  const int nstages = kSplit ? (kRingBytes - (nsplit - 1) * kPartBytes) / C::kStageBytes : C::kStages;
  uint8_t* sA = smem;
  uint8_t* sB = smem + nstages * C::kABytes;
  uint8_t* sPart = smem + nstages * C::kStageBytes;   // split-K partial region
  uint8_t* sEpi = smem + C::kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::kEpiBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* pbar = drain + 1;  // split-K rank 0: partials landed (bytes); rank r > 0: partial parked (warps)
  uint64_t* skbar = pbar + 1;  // stream-K: one per epilogue warp, its staged partials landed (bytes)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(skbar + kEpiWarps);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Pair: rank 0 issues the 2-SM MMAs, rank 1 holds the tile's lower half.
  // Split-K: the cluster's S CTAs share one tile, rank r taking k-blocks
  // [r kb / S, (r + 1) kb / S); rank 0 sums the partials and stores.
  const uint32_t rank = (kPair || kSplit) ? cluster_rank() : 0u;
  const uint32_t prank = kPair ? rank : 0u;            // rank in the tile's row geometry
  const int per_unit = kPair ? 2 : nsplit;            // CTAs per unit of work
  const int unit = static_cast<int>(blockIdx.x) / per_unit;
  const int units = static_cast<int>(gridDim.x) / per_unit;

  // Barrier set-up (warp 2), TMEM allocation (warp 1) and the producer's
  // first tile coordinates (warp 0) proceed side by side.
  int first_tb = 0, first_tm = 0, first_tn = 0, first_pi = 0;
  const int first_t = unit < p.nslots ? slot_tile(p, unit) : -1;
  if (threadIdx.x == 0 && first_t >= 0) first_pi = tile_coords(p, first_t, first_tb, first_tm, first_tn);
  if (threadIdx.x == 64) {
    for (int s = 0; s < nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], C::kTempty);
    }
    mbar_init(drain, 1);
    if constexpr (kSplit) mbar_init(pbar, rank == 0 ? 1u : static_cast<uint32_t>(kEpiWarps));
    if constexpr (!kSplit)
      for (int i = 0; i < kEpiWarps; ++i) mbar_init(&skbar[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    // split-K rank 0: its partial region fills with (S - 1) bulk copies
    if (kSplit && rank == 0) mbar_arrive_expect_tx(pbar, static_cast<uint32_t>((nsplit - 1) * kPartBytes));
    for (int i = 0; i < p.nprob; ++i) {
      if (p.pr[i].k_blocks > 0) {
        prefetch_tmap(i ? &ta1 : &ta0);
        prefetch_tmap(i ? &tb1 : &tb0);
      }
      if (p.pr[i].tma_store) prefetch_tmap(i ? &td1 : &td0);
    }
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (kPair) {
    cluster_sync();  // both CTAs' barriers exist before either signals the other
  } else {
    cta_sync();
    // Split-K: the first remote access comes at the end of the mainloop, so
    // the cluster barrier's wait (every CTA's barriers initialized) is taken
    // there (epilogue) or at teardown (the other warps), not here.
    if constexpr (kSplit) cluster_arrive();
  }
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next kernel on the stream may start its own set-up now; it reads what
  // this one writes only after its own griddepcontrol.wait, which waits for
  // this grid to complete.  Each role below waits for the previous kernel
  // (griddepcontrol.wait) only before it first touches global memory: the
  // producer before its first TMA load, the epilogue before reading scales
  // and writing D; the MMA warp reads shared memory and TMEM only.
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const int a_row0 = static_cast<int>(prank) * kBM;      // this CTA's rows within the tile
      const int b_row0 = static_cast<int>(prank) * C::kBRows;
      bool dep_done = false;
      int issued = 0;  // k-blocks loaded so far; the first kStages find their stage free
      Sched sc;
      sched_init<kSk>(p, unit, sc);
      Work w;
      while (!*abort_flag && sched_next<kSk>(p, unit, units, sc, w)) {
        const int t = w.t;
        int tb = first_tb, tm = first_tm, tn = first_tn;
        const int pi = t == first_t ? first_pi : tile_coords(p, t, tb, tm, tn);
        const int za = FP8_PR(bcast_a) ? 0 : tb, zb = FP8_PR(bcast_b) ? 0 : tb;  // batch coordinates
        const CUtensorMap* tma_a = pi ? &ta1 : &ta0;
        const CUtensorMap* tma_b = pi ? &tb1 : &tb0;
        const int am = tm * C::kTileM + a_row0;
        const int bn0 = tn * BN + b_row0;
        const int k_blocks = FP8_PR(k_blocks);
        const bool a_mn = FP8_PR(a_major) != 0, b_mn = FP8_PR(b_major) != 0;
        const int kb_lo = kSplit ? static_cast<int>(rank) * k_blocks / nsplit : w.kb_lo;
        const int kb_hi = kSplit ? (static_cast<int>(rank) + 1) * k_blocks / nsplit : w.kb_hi;
        for (int kb = kb_lo; kb < kb_hi; ++kb, ++issued) {
          if (issued >= nstages && !mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag)) break;
          if (!dep_done) {  // operands are the previous kernel's output
            pdl_wait();
            dep_done = true;
          }
          uint8_t* a_dst = sA + stage * C::kABytes;
          uint8_t* b_dst = sB + stage * C::kBBytes;
          if constexpr (kPair) {
            // both CTAs' bytes are counted on the even CTA's full barrier
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
            if (!a_mn) tma_load_3d_pair(a_dst, tma_a, bar, kb * kBK, am, za);
            else       tma_load_3d_pair(a_dst, tma_a, bar, am, kb * kBK, za);
            if (!b_mn) tma_load_3d_pair(b_dst, tma_b, bar, kb * kBK, bn0, zb);
            else       tma_load_3d_pair(b_dst, tma_b, bar, bn0, kb * kBK, zb);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
            if (!a_mn) tma_load_3d(a_dst, tma_a, &full[stage], kb * kBK, am, za);
            else       tma_load_3d(a_dst, tma_a, &full[stage], am, kb * kBK, za);
            if (!b_mn) {
              tma_load_3d(b_dst, tma_b, &full[stage], kb * kBK, bn0, zb);
            } else {
              #pragma unroll
              for (int h = 0; h < C::kBRows / 128; ++h)
                tma_load_3d(b_dst + h * 128 * kBK, tma_b, &full[stage], bn0 + h * 128, kb * kBK, zb);
            }
          }
          if (++stage == nstages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && (!kPair || rank == 0)) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      Sched sc;
      sched_init<kSk>(p, unit, sc);
      Work w;
      while (!*abort_flag && sched_next<kSk>(p, unit, units, sc, w)) {
        const int t = w.t;
        const int pi = t >= p.tiles0 ? 1 : 0;
        const int k_blocks = FP8_PR(k_blocks);
        const bool a_mn = FP8_PR(a_major) != 0, b_mn = FP8_PR(b_major) != 0;
        const uint32_t idesc = FP8_PR(idesc);
        const int kb_lo = kSplit ? static_cast<int>(rank) * k_blocks / nsplit : w.kb_lo;
        const int kb_hi = kSplit ? (static_cast<int>(rank) + 1) * k_blocks / nsplit : w.kb_hi;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_base = smem_u32(sB + stage * C::kBBytes);
          #pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            // K-major: advance 32 bytes along the swizzled 128-byte row.
            // MN-major: advance 32 k-rows of 128 bytes (4 swizzle atoms); the
            // leading offset steps between 128-element MN chunks of B.
            const uint64_t ad = !a_mn ? smem_desc_sw128(a_base + kk * kUmmaK, 16, 1024)
                                      : smem_desc_sw128(a_base + kk * kUmmaK * 128, 128 * kBK, 1024);
            const uint64_t bd = !b_mn ? smem_desc_sw128(b_base + kk * kUmmaK, 16, 1024)
                                      : smem_desc_sw128(b_base + kk * kUmmaK * 128, 128 * kBK, 1024);
            const uint32_t accum = (kb != kb_lo || kk != 0) ? 1u : 0u;
            if constexpr (kPair) umma_f8f6f4_pair(d_tmem, ad, bd, idesc, accum);
            else                 umma_f8f6f4(d_tmem, ad, bd, idesc, accum);
          }
          if constexpr (kPair) {
            const uint32_t e = smem_u32(&empty[stage]);
            umma_commit_pair(e);
            umma_commit_pair(mapa_shared(e, 1));
          } else {
            umma_commit(&empty[stage]);
          }
          if (++stage == nstages) { stage = 0; phase ^= 1u; }
        }
        if constexpr (kPair) {
          const uint32_t f = smem_u32(&tfull[acc]);
          umma_commit_pair(f);
          umma_commit_pair(mapa_shared(f, 1));
        } else {
          umma_commit(&tfull[acc]);
        }
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // Whatever path led here (a bounded wait may have given up), no MMA may
      // still read shared memory or TMEM when the CTAs tear down.
      if constexpr (kPair) umma_commit_pair(smem_u32(drain));
      else umma_commit(drain);
      mbar_wait(drain, 0, nullptr, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0..7
    const int qd = warp & 3;                 // TMEM lane quadrant this warp may access
    const int half = ew >> 2;                // which half of the tile's columns
    const int row_in_tile = static_cast<int>(prank) * kBM + qd * 32 + lane;
    // split-K: this thread's row in slot 0 of the partial region; column quad
    // c4 of row i is float4 c4 * 128 + i of a slot
    float4* const part_row = reinterpret_cast<float4*>(sPart) + (qd * 32 + lane);
    bool cluster_ready = !kSplit;  // split-K: the start-up cluster barrier's wait is taken
    pdl_wait();
    if (blockIdx.x == 0 && threadIdx.x == 64) {
      for (int i = 0; i < 2; ++i) {
        if (p.side.copy_dst[i]) *p.side.copy_dst[i] = *p.side.copy_src[i];
        if (p.side.zero_dst[i]) *p.side.zero_dst[i] = 0.0f;
      }
    }
    if (blockIdx.x == 0 && ew == 1)  // warp 3 of CTA 0; the mainloop runs meanwhile
      for (int i = 0; i < p.nfin; ++i) ring_finalize_warp(p.fin[i], lane);
    if (p.dbias.partial && ew == 2) dbias_finish_warp(p.dbias, lane);  // warp 4 of every CTA
    const float inv0 = 1.0f / (*p.pr[0].scale_a * *p.pr[0].scale_b);
    const float binv0 = (p.pr[0].bias_kind >= 2) ? 1.0f / *p.pr[0].bias_scale : 1.0f;
    float inv1 = 1.0f, binv1 = 1.0f;
    if (p.nprob > 1) {
      inv1 = 1.0f / (*p.pr[1].scale_a * *p.pr[1].scale_b);
      binv1 = (p.pr[1].bias_kind >= 2) ? 1.0f / *p.pr[1].bias_scale : 1.0f;
    }
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    uint8_t* slabs = sEpi + ew * 2 * kEpiSlab;
    int slab = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    constexpr int kSteps = BN / 2 / kEpiCols;
    // stream-K partial slots, one per CTA: [epilogue warp][32-column step]
    // [column quad][lane] float4s, so each (warp, step) block is 4 KB of
    // contiguous fp32 (one bulk copy) and a warp's stores of one column quad
    // are 512 contiguous bytes
    float4* const sk_part = reinterpret_cast<float4*>(p.sk_part);
    uint8_t* const sk_stage = sA + ew * kSkStageBytes;
    uint32_t sk_phase = 0;
    // the slot (and flag block) of a work unit's CTA of this rank: a pair tile
    // keeps one partial per CTA, its 128-row half
    auto sk_slot = [&](int u) { return kPair ? 2 * u + static_cast<int>(prank) : u; };
    auto sk_block = [&](int slot, int st) {
      return sk_part + ((static_cast<int64_t>(slot) * kEpiWarps + ew) * kSteps + st) * (kSkBlock / 16);
    };
    Sched sc;
    sched_init<kSk>(p, unit, sc);
    Work w;
    while (!*abort_flag && sched_next<kSk>(p, unit, units, sc, w)) {
      const int t = w.t;
      int tb, tm, tn;
      const int pi = tile_coords(p, t, tb, tm, tn);
      // The tile's constants go to registers and its bias values are fetched
      // BEFORE the wait for the accumulator, so that no parameter read and no
      // global-memory latency sits between the TMEM read and the store.
      const int qm = FP8_PR(m), qn = FP8_PR(n), bias_kind = FP8_PR(bias_kind);
      const bool tma_store = FP8_PR(tma_store) != 0;
      const bool have_k = kSplit ? (static_cast<int>(rank) + 1) * FP8_PR(k_blocks) / nsplit >
                                       static_cast<int>(rank) * FP8_PR(k_blocks) / nsplit
                                 : w.kb_hi > w.kb_lo;
      void* const qd_ptr = static_cast<__nv_bfloat16*>(FP8_PR(d)) + static_cast<int64_t>(tb) * FP8_PR(stride_d);
      const int64_t ldd = FP8_PR(ldd);
      const void* const bias = FP8_PR(bias);
      const CUtensorMap* tma_d = pi ? &td1 : &td0;
      const float tinv = pi ? inv1 : inv0;
      const int col_half = tn * BN + half * (BN / 2);
      const int live_steps = min(kSteps, max(0, (qn - col_half + kEpiCols - 1) / kEpiCols));
      float bl[kSteps];
      #pragma unroll
      for (int st = 0; st < kSteps; ++st) {
        const int j = col_half + st * kEpiCols + lane;
        bl[st] = (bias_kind && j < qn) ? bias_value(bias, bias_kind, j, pi ? binv1 : binv0) : 0.0f;
      }
      if (!mbar_wait(&tfull[acc], acc_phase, p.status, abort_flag)) break;
      tc_fence_after();
      if constexpr (kSplit) {
        if (!cluster_ready) { cluster_wait(); cluster_ready = true; }
        // rank 0: the other ranks' partials have landed in its partial region
        if (rank == 0 && !mbar_wait(pbar, 0, p.status, abort_flag)) break;
      }
      // owner: the later parts' partials are in their slots; they are staged
      // `spr` steps at a time in this warp's share of the (now idle) operand ring
      int spr = kSteps;
      if (kSk && w.kind == kOwner) {
        bool ok = w.nparts >= 1 && w.nparts <= kSkMaxParts;
        if (!ok && lane == 0 && p.status) atomicExch(p.status, kDevTimeout);  // outside the planner's bound: give up
        for (int q = 0; q < w.nparts && ok; ++q)
          ok = flag_wait_warp(p.sk_flag + static_cast<int64_t>(sk_slot(w.part0 + q)) * kEpiWarps + ew, p.status,
                              abort_flag);
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        spr = min(kSteps, kSkMaxParts / w.nparts);
        fence_proxy_async_global();  // the acquires above come before the bulk copies' reads
      }
      const int row = tm * C::kTileM + row_in_tile;
      #pragma unroll 1
      for (int st = 0; st < kSteps; ++st) {
        const int col0 = col_half + st * kEpiCols;
        if (kSk && w.kind == kOwner && st % spr == 0) {  // stage the partials of steps [st, st + spr)
          const int nst = min(spr, kSteps - st);
          fence_proxy_async_smem();  // this warp's reads of the previous round come first
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_expect_tx(&skbar[ew], static_cast<uint32_t>(w.nparts * nst * kSkBlock));
            for (int q = 0; q < w.nparts; ++q)
              bulk_copy_g2s(sk_stage + q * nst * kSkBlock, sk_block(sk_slot(w.part0 + q), st),
                            static_cast<uint32_t>(nst * kSkBlock), &skbar[ew]);
          }
          if (!mbar_wait(&skbar[ew], sk_phase, p.status, abort_flag)) break;
          sk_phase ^= 1u;
        }
        uint32_t r[32];
        if (st < live_steps) {
          if (have_k) {
            __syncwarp();  // tcgen05.ld is .sync.aligned
            tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(acc * BN + half * (BN / 2) + st * kEpiCols), r);
            tmem_ld_wait();
          } else {  // K = 0: the MMA never wrote this accumulator
            #pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = 0u;
          }
        }
        if (st == kSteps - 1) {  // last TMEM read of this accumulator: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
            else mbar_arrive(&tempty[acc]);
          }
        }
        if (st >= live_steps) continue;
        if constexpr (kSplit) {
          const int pq = (half * (BN / 2) + st * kEpiCols) / 4;  // column quad of r[0..3]
          if (rank != 0) {  // park the partial; rank 0 finishes the tile
            #pragma unroll
            for (int j = 0; j < 32; j += 4)
              part_row[(pq + j / 4) * kBM] = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                         __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
            continue;
          }
          // rank order: ((p0 + p1) + p2) + ..., the same for every launch
          for (int q = 1; q < nsplit; ++q) {
            const float4* src = part_row + (q - 1) * (kPartBytes / 16) + pq * kBM;
            #pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 o = src[(j / 4) * kBM];
              r[j] = __float_as_uint(__uint_as_float(r[j]) + o.x);
              r[j + 1] = __float_as_uint(__uint_as_float(r[j + 1]) + o.y);
              r[j + 2] = __float_as_uint(__uint_as_float(r[j + 2]) + o.z);
              r[j + 3] = __float_as_uint(__uint_as_float(r[j + 3]) + o.w);
            }
          }
        }
        if (kSk && w.kind != kFull) {
          if (w.kind == kPartial) {  // this part's accumulator goes to the CTA's slot
            float4* dst = sk_block(sk_slot(unit), st) + lane;
            #pragma unroll
            for (int j = 0; j < 32; j += 4)
              __stcg(dst + (j / 4) * 32, make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                     __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])));
            continue;
          }
          // owner: ((acc + p[part0]) + p[part0 + 1]) + ..., the same for every launch
          const int nst = min(spr, kSteps - (st - st % spr));
          for (int q = 0; q < w.nparts; ++q) {
            const float4* src =
                reinterpret_cast<const float4*>(sk_stage + (q * nst + st % spr) * kSkBlock) + lane;
            #pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 o = src[(j / 4) * 32];
              r[j] = __float_as_uint(__uint_as_float(r[j]) + o.x);
              r[j + 1] = __float_as_uint(__uint_as_float(r[j + 1]) + o.y);
              r[j + 2] = __float_as_uint(__uint_as_float(r[j + 2]) + o.z);
              r[j + 3] = __float_as_uint(__uint_as_float(r[j + 3]) + o.w);
            }
          }
        }
        // One uniform branch per step, none per element: a shuffle under a
        // per-element condition costs a reconvergence point each.
        float v[32];
        if (bias_kind) {
          const float bst = pick(bl, st);
          #pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) * tinv + __shfl_sync(0xFFFFFFFFu, bst, j);
        } else {
          #pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) * tinv;
        }
        if (tma_store) {
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
            tma_store_3d(tma_d, buf, col0, tm * C::kTileM + static_cast<int>(prank) * kBM + qd * 32, tb);
            bulk_commit();
          }
          slab ^= 1;
        } else if (row < qm) {
          __nv_bfloat16* drow = static_cast<__nv_bfloat16*>(qd_ptr) + static_cast<int64_t>(row) * ldd;
          #pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < qn) drow[col0 + j] = __float2bfloat16_rn(v[j]);
        }
      }
      if (kSk && w.kind == kPartial) {  // this warp's share of the partial is written: raise its flag
        warp_release_flag(p.sk_flag + static_cast<int64_t>(sk_slot(unit)) * kEpiWarps + ew, 1u);
      } else if (kSk && w.kind == kOwner) {  // every lane has read the partials: clear their flags
        __syncwarp();
        if (lane == 0)
          for (int q = 0; q < w.nparts; ++q) p.sk_flag[static_cast<int64_t>(sk_slot(w.part0 + q)) * kEpiWarps + ew] = 0u;
      }
      if (kSplit && rank != 0) {  // partial parked: one bulk copy into rank 0's region
        fence_proxy_async_smem();  // this thread's parked bytes, visible to the copy engine
        __syncwarp();
        if (lane == 0) mbar_arrive(pbar);
        if (ew == 0 && lane == 0 && mbar_wait(pbar, 0, p.status, abort_flag))  // all eight warps parked
          bulk_copy_to_cluster(mapa_shared(smem_u32(sPart + (rank - 1) * kPartBytes), 0), sPart, kPartBytes,
                               mapa_shared(smem_u32(pbar), 0));
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    // The stores' global writes complete on their own; the CTA only has to
    // outlive their reads of its shared memory.
    if (p.any_tma_store && lane == 0) bulk_wait_read<0>();
    if (!cluster_ready) cluster_wait();
  }
  if constexpr (kSplit) {
    if (warp < 2) cluster_wait();  // producer and MMA warps close the start-up cluster barrier
  }

  tc_fence_before();
  if constexpr (kPair || kSplit) cluster_sync();  // no CTA leaves while another still signals or reads it
  else cta_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Pairs (clusters of two 256x256-tile CTAs) that can be resident at once
// (cached per device; 0 on failure).
int pair_capacity_impl(int dev) {
  using C = Cfg<256, true>;
  static int cache[64] = {};
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  if (cudaFuncSetAttribute(fp8_gemm_kernel<256, true, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmem) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.gridDim = dim3(2 * (num_sms(dev) / 2));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, fp8_gemm_kernel<256, true, false, false>, &cfg) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cache[dev] = clusters;
  return clusters;
}

int pair_capacity(int dev) { return pair_capacity_impl(dev); }

template <int BN, bool kPair>
cudaError_t launch_cfg(const CUtensorMap* mp, const GemmParams& p, cudaStream_t s) {
  using C = Cfg<BN, kPair>;
  int dev = 0;
  cudaGetDevice(&dev);
  // the stream-K build for launches with stream-K ranges, else the plain one
  auto kernel = p.sk_ctas > 0 ? fp8_gemm_kernel<BN, kPair, false, true> : fp8_gemm_kernel<BN, kPair, false, false>;
  static bool configured[64] = {};
  if (dev < 64 && !configured[dev]) {
    for (auto k : {fp8_gemm_kernel<BN, kPair, false, false>, fp8_gemm_kernel<BN, kPair, false, true>}) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
      if (e != cudaSuccess) return e;
    }
    configured[dev] = true;
  }
  const int sms = num_sms(dev);
  if (!kPair) {
    // stream-K: the whole-tile waves use one CTA per SM (at most 160, the
    // planner's CTA count), the k-block ranges the first sk_ctas of them
    int grid = p.total_tiles < sms ? p.total_tiles : sms;
    if (p.sk_ctas > 0) grid = p.dp_tiles > 0 ? (sms < 160 ? sms : 160) : p.sk_ctas;
    return launch_pdl(kernel, dim3(grid), dim3(kThreads), C::kSmem, s, mp[0], mp[1], mp[2], mp[3],
                      mp[4], mp[5], p);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // persistent grid: no more pairs than can be resident at once
  const int cap = pair_capacity(dev);
  if (cap <= 0) return cudaErrorInvalidConfiguration;
  int pairs = p.total_tiles < cap ? p.total_tiles : cap;
  // stream-K: the planner's pair count (its whole-tile waves use sms / 2
  // pairs, at most 80); every pair must be resident at once
  if (p.sk_ctas > 0) {
    const int sk_pairs = sms / 2 < 80 ? sms / 2 : 80;
    pairs = p.dp_tiles > 0 ? sk_pairs : p.sk_ctas;
    if (pairs > cap) return cudaErrorInvalidConfiguration;
  }
  cfg.gridDim = dim3(2 * pairs);
  return cudaLaunchKernelEx(&cfg, kernel, mp[0], mp[1], mp[2], mp[3], mp[4], mp[5], p);
}

// Largest number of clusters of `split` CTAs of the split-K kernel that can be
// resident at once (cached per device and split factor).
int split_clusters(int dev, int split) {
  static int cache[64][kMaxSplit + 1] = {};
  if (split < 2 || split > kMaxSplit) return 0;
  if (dev < 64 && cache[dev][split]) return cache[dev][split];
  using C = Cfg<128, false>;
  cudaError_t e = cudaFuncSetAttribute(fp8_gemm_kernel<128, false, true, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.gridDim = dim3(split * (num_sms(dev) / split));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(split);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, fp8_gemm_kernel<128, false, true, false>, &cfg) != cudaSuccess) return 0;
  if (dev < 64) cache[dev][split] = clusters;
  return clusters;
}

// Split-K launch: one cluster of p.split CTAs per 128 x 128 tile.
cudaError_t launch_split(const CUtensorMap* mp, const GemmParams& p, cudaStream_t s) {
  using C = Cfg<128, false>;
  int dev = 0;
  cudaGetDevice(&dev);
  if (split_clusters(dev, p.split) <= 0) return cudaErrorInvalidConfiguration;  // also sets the smem limit
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cfg.gridDim = dim3(static_cast<unsigned>(p.total_tiles * p.split));
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.split);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, fp8_gemm_kernel<128, false, true, false>, mp[0], mp[1], mp[2], mp[3], mp[4], mp[5], p);
}

// The output of an empty contraction: every accumulator is zero, so each
// element is 0 + bias[j] rounded once to bf16 (the epilogue's arithmetic with
// acc = 0), or zero without a bias.  Grid-stride over batch x m x n.
__global__ void __launch_bounds__(256) fill_kernel(const FillParams p) {
  pdl_wait();
  pdl_trigger();
  const float binv = p.bias_kind >= 2 ? 1.0f / *p.bias_scale : 1.0f;
  const int64_t per = p.m * p.n;
  const int64_t total = per * p.batch;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / per, r = (i - b * per) / p.n, c = i - b * per - r * p.n;
    const float v = 0.0f + (p.bias_kind ? bias_value(p.bias, p.bias_kind, static_cast<int>(c), binv) : 0.0f);
    static_cast<__nv_bfloat16*>(p.d)[b * p.stride_d + r * p.ldd + c] = __float2bfloat16_rn(v);
  }
}

}  // namespace

cudaError_t launch_fill(const FillParams& p, cudaStream_t s) {
  const int64_t total = p.m * p.n * p.batch;
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t cap = static_cast<int64_t>(num_sms(dev) > 0 ? num_sms(dev) : 1) * 8;
  const int64_t blocks = std::min<int64_t>(cap, std::max<int64_t>(1, (total + 255) / 256));
  return launch_pdl(fill_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p);
}

int gemm_pair_capacity(int dev) { return pair_capacity(dev); }

int gemm_split_factor(int tiles, int k_blocks, int sms, bool forced) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || tiles <= 0 || k_blocks < 2) return 1;
  int best = 1;
  for (int s = 2; s <= kMaxSplit; ++s) {
    if (s > k_blocks) break;
    if (!forced && k_blocks / s < 4) break;  // at least 4 k-blocks a rank
    const int clusters = split_clusters(dev, s);
    if (clusters <= 0) break;
    if (tiles > clusters) {  // a second wave of clusters: never worth it
      if (forced && best == 1) best = s;
      break;
    }
    best = s;
  }
  return best;
}

cudaError_t launch_gemm(const CUtensorMap* maps, const GemmParams& p, int cfg, cudaStream_t s) {
  if (cfg == kGemmSplit128) return launch_split(maps, p, s);
  if (cfg == kGemmPair256) return launch_cfg<256, true>(maps, p, s);
  if (cfg == kGemm256) return launch_cfg<256, false>(maps, p, s);
  return launch_cfg<128, false>(maps, p, s);
}

}  // namespace fp8lin
