// api.cu -- the extern "C" boundary of libfp8lin (see include/fp8lin.h).
//
// Validation happens before anything is enqueued; the library allocates no
// memory and never synchronizes the host (fp8_get_device_status excepted).
// TMA tensor maps are encoded on the host per call (cuTensorMapEncodeTiled,
// fetched through the runtime's driver entry point so the shared object loads
// on machines without a GPU driver) and passed as __grid_constant__ kernel
// parameters.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <functional>
#include <queue>
#include <vector>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "device.cuh"
#include "fp8lin.h"
#include "internal.h"

namespace fp8lin {

__device__ int g_device_status;

namespace {

thread_local char g_err[256] = "";

int cuda_fail(cudaError_t e) {
  snprintf(g_err, sizeof(g_err), "CUDA error %d: %s", static_cast<int>(e), cudaGetErrorString(e));
  return FP8_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
int g_sms[64] = {};
int* g_status_ptr[64] = {};

EncodeTiledFn encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

int* status_ptr(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) == cudaSuccess) g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool is_fmt(int f) { return f == FP8_E4M3 || f == FP8_E5M2; }
bool is_wide(int dt) { return dt == FP8_DT_BF16 || dt == FP8_DT_FP16 || dt == FP8_DT_FP32; }
bool is_fp8(int dt) { return dt == FP8_DT_E4M3 || dt == FP8_DT_E5M2; }
int esize(int dt) { return dt == FP8_DT_FP32 ? 4 : (is_fp8(dt) ? 1 : 2); }
float fp8_max(int fmt) { return fmt == FP8_E4M3 ? 448.0f : 57344.0f; }
bool ring_len_ok(int H) { return H >= 1 && H <= 4096; }
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

// An fp8 matrix [rows, ld] the kernels read or write with TMA or 16-byte
// accesses.  An empty one (no rows or no columns) is never touched, so its
// pointer and stride are not checked.
int check_fp8_matrix(const void* p, int64_t ld, int64_t rows, int64_t cols) {
  if (rows == 0 || cols == 0) return FP8_OK;
  if (!p) return FP8_ERR_INVALID_ARG;
  if (ld < cols) return FP8_ERR_INVALID_ARG;
  if (ld % 16 != 0 || !aligned(p, 16)) return FP8_ERR_MISALIGNED;
  return FP8_OK;
}

// 2-D tensor map with zero fill out of bounds (loads) / clipping (stores).
// Every GEMM tensor map is 3-D: (inner, outer, batch) with a box one batch
// deep.  An unbatched or broadcast operand has batch extent 1 (its batch
// stride is then only formal: one matrix, rounded up to 16 bytes).
int make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
             uint64_t ld_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz,
             uint64_t batch = 1, uint64_t batch_bytes = 0) {
  EncodeTiledFn enc = encoder();
  if (!enc) {
    snprintf(g_err, sizeof(g_err), "cuTensorMapEncodeTiled unavailable");
    return FP8_ERR_CUDA;
  }
  if (batch <= 1) batch_bytes = (ld_bytes * outer + 15) / 16 * 16;
  cuuint64_t dims[3] = {inner, outer, batch};
  cuuint64_t strides[2] = {ld_bytes, batch_bytes};
  cuuint32_t box[3] = {box_inner, box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_err, sizeof(g_err), "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return FP8_ERR_CUDA;
  }
  return FP8_OK;
}

// fp8 operand map: 128-byte rows of a 128 x `rows` box, 128-byte swizzle.
int make_fp8_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld, uint32_t box_rows,
                 uint64_t batch = 1, uint64_t batch_stride = 0) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, inner, outer, ld, 128, box_rows, CU_TENSOR_MAP_SWIZZLE_128B,
                  batch, batch_stride);
}

struct MmCall {
  int64_t m, n, k;
  const uint8_t* a; int fmt_a; int a_major; int64_t lda;
  const uint8_t* b; int fmt_b; int b_major; int64_t ldb;
  const float* scale_a; const float* scale_b;
  const void* bias; int bias_dtype; const float* bias_scale;
  void* d; int64_t ldd;
  int tile_cfg;
  // batched GEMMs (fp8_mm_batched): element strides between batches; a zero
  // operand stride shares that operand across the batch
  int64_t batch = 1, stride_a = 0, stride_b = 0, stride_d = 0;
  // stream-K workspace (optional): zero-at-rest flags, then partial slots
  void* ws = nullptr;
  size_t ws_bytes = 0;
};

// Stream-K scratch: a fixed block of flags (one per epilogue warp of up to
// kSkMaxCtas CTAs, zero at rest), then one partial accumulator slot per CTA.
constexpr int kSkMaxCtas = 160;
constexpr int kSkWarps = 8;
constexpr size_t kSkFlagBytes = static_cast<size_t>(kSkMaxCtas) * kSkWarps * 4;
constexpr size_t kSkSlotBytes = 128 * 256 * 4;   // the largest tile's fp32 accumulator
constexpr int64_t kSkMinUnits = 4;               // k-blocks per CTA below which stream-K is not used
constexpr int64_t kSkMaxParts = 6;               // partials a finishing CTA stages (24 KB per epilogue warp)

// Slots a stream-K launch of this size can use: at most one per CTA and per
// 128 x 128 x 128 block of work.
int64_t sk_slots_for(int64_t m, int64_t n, int64_t k) {
  if (m <= 0 || n <= 0 || k <= 0) return 0;
  const int64_t blocks = ((m + 127) / 128) * ((n + 127) / 128) * ((k + 127) / 128);
  return std::min<int64_t>(kSkMaxCtas, blocks);
}

size_t sk_bytes_for(int64_t m, int64_t n, int64_t k) {
  const int64_t slots = sk_slots_for(m, n, k);
  return slots ? kSkFlagBytes + static_cast<size_t>(slots) * kSkSlotBytes : 0;
}

int validate_mm(const MmCall& c) {
  if (c.m < 0 || c.n < 0 || c.k < 0 || c.m > kMaxDim || c.n > kMaxDim || c.k > kMaxDim) return FP8_ERR_INVALID_ARG;
  if (!is_fmt(c.fmt_a) || !is_fmt(c.fmt_b)) return FP8_ERR_INVALID_ARG;
  if ((c.a_major != FP8_K_MAJOR && c.a_major != FP8_MN_MAJOR) ||
      (c.b_major != FP8_K_MAJOR && c.b_major != FP8_MN_MAJOR))
    return FP8_ERR_INVALID_ARG;
  if (!c.scale_a || !c.scale_b) return FP8_ERR_INVALID_ARG;
  int s = c.a_major == FP8_K_MAJOR ? check_fp8_matrix(c.a, c.lda, c.m, c.k) : check_fp8_matrix(c.a, c.lda, c.k, c.m);
  if (s) return s;
  s = c.b_major == FP8_K_MAJOR ? check_fp8_matrix(c.b, c.ldb, c.n, c.k) : check_fp8_matrix(c.b, c.ldb, c.k, c.n);
  if (s) return s;
  if (c.m > 0 && c.n > 0 && (!c.d || c.ldd < c.n || !aligned(c.d, 2))) return FP8_ERR_INVALID_ARG;
  const int base_cfg = c.tile_cfg & ~FP8_TILE_STREAMK;
  if (base_cfg < FP8_TILE_AUTO || base_cfg > FP8_TILE_SPLITK_128x128) return FP8_ERR_INVALID_ARG;
  if ((c.tile_cfg & FP8_TILE_STREAMK) && (base_cfg < FP8_TILE_128x128 || base_cfg > FP8_TILE_PAIR_256x256))
    return FP8_ERR_INVALID_ARG;
  if (c.ws_bytes && (!c.ws || !aligned(c.ws, 16))) return FP8_ERR_WORKSPACE;
  if (c.bias) {
    if (c.bias_dtype != FP8_DT_BF16 && !is_fp8(c.bias_dtype)) return FP8_ERR_INVALID_ARG;
    if (is_fp8(c.bias_dtype) && !c.bias_scale) return FP8_ERR_INVALID_ARG;
    if (c.bias_dtype == FP8_DT_BF16 && !aligned(c.bias, 2)) return FP8_ERR_INVALID_ARG;
  }
  return FP8_OK;
}

// The call an fp8_mm_args describes (tile configuration and workspace from
// `lead`, the first GEMM of a launch).
MmCall mm_call(const fp8_mm_args* x, const fp8_mm_args* lead) {
  MmCall c{x->m, x->n, x->k, x->a, x->fmt_a, x->a_major, x->lda, x->b, x->fmt_b, x->b_major, x->ldb,
           x->scale_a, x->scale_b, x->bias, x->bias_dtype, x->bias_scale, x->d, x->ldd, lead->tile_cfg};
  c.ws = lead->workspace;
  c.ws_bytes = lead->workspace_bytes;
  return c;
}

// Per-tile cost, in k-blocks, of the schedule models: the mainloop plus the
// part of the epilogue a following tile does not hide.
constexpr int kTileFixedKb = 2;

// Longest-processing-time list schedule of a launch's tiles (problem 0's
// count0 tiles of cost0 k-blocks, then count1 of cost1) over `units` CTAs:
// tiles in decreasing cost, each to the least loaded unit (ties: lowest unit,
// so equal-cost tiles keep their raster order).  Returns the makespan in
// k-blocks; with `order`, writes slot round * units + unit (kNoTile: none) and
// *nslots, or returns -1 when the slots would exceed kMaxOrder.
int64_t lpt_schedule(int64_t count0, int64_t cost0, int64_t count1, int64_t cost1, int64_t units, uint16_t* order,
                     int* nslots) {
  const int64_t total = count0 + count1;
  if (total <= 0 || units <= 0) return 0;
  units = std::min(units, total);
  std::vector<int64_t> tiles(static_cast<size_t>(total));
  for (int64_t t = 0; t < total; ++t) tiles[static_cast<size_t>(t)] = t;
  auto cost = [&](int64_t t) { return (t < count0 ? cost0 : cost1) + kTileFixedKb; };
  std::stable_sort(tiles.begin(), tiles.end(), [&](int64_t a, int64_t b) { return cost(a) > cost(b); });
  using Load = std::pair<int64_t, int64_t>;  // (load, unit)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int64_t u = 0; u < units; ++u) heap.push({0, u});
  std::vector<std::vector<int64_t>> lists(order ? static_cast<size_t>(units) : 0);
  int64_t makespan = 0;
  for (int64_t t : tiles) {
    Load l = heap.top();
    heap.pop();
    l.first += cost(t);
    makespan = std::max(makespan, l.first);
    if (order) lists[static_cast<size_t>(l.second)].push_back(t);
    heap.push(l);
  }
  if (order) {
    size_t rounds = 0;
    for (const auto& v : lists) rounds = std::max(rounds, v.size());
    if (static_cast<int64_t>(rounds) * units > kMaxOrder) return -1;
    for (size_t r = 0; r < rounds; ++r)
      for (int64_t u = 0; u < units; ++u) {
        const auto& v = lists[static_cast<size_t>(u)];
        order[r * static_cast<size_t>(units) + static_cast<size_t>(u)] =
            r < v.size() ? static_cast<uint16_t>(v[r]) : kNoTile;
      }
    *nslots = static_cast<int>(rounds * static_cast<size_t>(units));
  }
  return makespan;
}

// A launch's tile configuration and schedule.
struct TilePlan {
  int cfg = kGemm128;
  int sk_ctas = 0;         // stream-K: CTAs sharing the cut tiles' k-blocks (0: none)
  int dp_tiles = 0;        // stream-K: tiles run whole first
  int64_t sk_total = 0, sk_u0 = 0;
  double est_us = 0.0;
};

// Tile configuration with the smallest modelled time for a launch of one or
// two problems: the makespan (k-blocks) of the launch's tile schedule -- the
// LPT schedule the single-CTA configurations run for two problems of unequal
// k, round robin otherwise -- times the k-block time measured on a B200 for
// that tile shape, plus a fixed fill/drain cost.  Measured on a B200 (1965
// MHz): 0.31 us per 128x128x128 k-block on one SM; per 128x256x128 of work
// on one SM, 0.35 us for a single-CTA 128x256 tile and 0.37 us for a 256x256
// pair tile while each CTA runs at most 3 tiles, 0.40 and 0.365 us in longer
// launches (the single-CTA tile moves 1.5x the operand bytes per SM through
// L2, which tells once the whole chip streams for long); ~4-5 us fill +
// epilogue + launch.
// With sk_slots > 0 (a stream-K workspace of that many partial slots), the
// single-CTA configurations are also costed with stream-K: whole waves but
// the last one or two run data-parallel, the remaining tiles' k-blocks are
// split evenly over min(SMs, slots) CTAs (at least kSkMinUnits each, and few
// enough that a tile has at most kSkMaxParts partials), plus a fixup for the
// cut tiles: the partials' release and acquire, then the finishing CTA's bulk
// copies of the partials into its idle operand ring (one round per six 4 KB
// (step, partial) blocks of each epilogue warp).  force_sk: only stream-K
// plans of the given configuration.
TilePlan pick_tile(const MmCall* calls, int n, int sms, int64_t sk_slots = 0, int force_cfg = 0,
                   bool force_sk = false) {
  struct Opt { int cfg; int64_t tm, tn, units; double t_kb, t_kb_long, fixed, fixup; };
  const Opt opts[3] = {{kGemm128, 128, 128, sms, 0.31, 0.31, 4.0, 1.5},
                       {kGemm256, 128, 256, sms, 0.35, 0.40, 4.0, 1.5},
                       {kGemmPair256, 256, 256, sms / 2, 0.37, 0.365, 5.0, 0.0}};
  TilePlan best;
  bool have = false;
  bool batched = false;
  for (int i = 0; i < n; ++i) batched = batched || calls[i].batch > 1;
  for (const Opt& o : opts) {
    if (force_cfg && o.cfg != force_cfg) continue;
    int64_t cnt[2] = {0, 0}, kb[2] = {0, 0};
    for (int i = 0; i < n; ++i) {
      cnt[i] = ((calls[i].m + o.tm - 1) / o.tm) * ((calls[i].n + o.tn - 1) / o.tn) * calls[i].batch;
      kb[i] = (calls[i].k + 127) / 128;
    }
    const int64_t tiles = cnt[0] + cnt[1];
    if (!force_sk) {
      int64_t span;
      if (o.cfg != kGemmPair256 && n == 2 && kb[0] != kb[1]) {
        span = lpt_schedule(cnt[0], kb[0], cnt[1], kb[1], o.units, nullptr, nullptr);
      } else {  // round robin: unit u runs tiles u, u + units, ...
        span = 0;
        const int64_t units = std::max<int64_t>(1, std::min(o.units, tiles));
        for (int64_t u = 0; u < std::min(units, tiles); ++u) {
          int64_t load = 0;
          // tiles of problem 0 at u, u + units, ... then problem 1
          for (int64_t t = u; t < tiles; t += units) load += (t < cnt[0] ? kb[0] : kb[1]) + kTileFixedKb;
          span = std::max(span, load);
        }
      }
      const int64_t rounds = (tiles + o.units - 1) / std::max<int64_t>(1, o.units);
      const double t = static_cast<double>(span - kTileFixedKb) * (rounds > 3 ? o.t_kb_long : o.t_kb) + o.fixed;
      if (!have || t < best.est_us) {
        best = TilePlan{};
        best.cfg = o.cfg;
        best.est_us = t;
        have = true;
      }
    }
    // stream-K (unbatched; a pair tile's two CTAs keep one partial slot each)
    if (batched || sk_slots <= 0) continue;
    const bool pair = o.cfg == kGemmPair256;
    const int64_t P = pair ? std::min<int64_t>(sms / 2, kSkMaxCtas / 2) : std::min<int64_t>(sms, kSkMaxCtas);
    const int64_t unit_slots = pair ? sk_slots / 2 : sk_slots;
    const int64_t D = tiles >= 2 * P ? (tiles / P - 1) * P : 0;
    const int64_t u0 = D < cnt[0] ? (cnt[0] - D) * kb[0] : 0;
    const int64_t u1 = (tiles - std::max(D, cnt[0])) * kb[1];
    const int64_t U = u0 + u1;
    // at least kSkMinUnits k-blocks per CTA, and ranges long enough that a
    // tile is cut into at most kSkMaxParts + 1 parts (the finishing CTA stages
    // at most kSkMaxParts partials): ceil((kb - 1) / floor(U / ctas)) <= 6
    const int64_t kbmax = std::max(kb[0], kb[1]);
    const int64_t min_units = std::max<int64_t>(kSkMinUnits, (kbmax - 1 + kSkMaxParts - 1) / kSkMaxParts);
    int64_t ctas = std::min({P, unit_slots, std::max<int64_t>(force_sk ? 1 : 0, U / min_units)});
    while (ctas > 1 && (kbmax - 1 + U / ctas - 1) / (U / ctas) > kSkMaxParts) --ctas;
    if (ctas < (force_sk ? 1 : 2)) continue;
    const int64_t nparts = U / ctas > 0 ? (kbmax - 1 + U / ctas - 1) / (U / ctas) : 0;
    int64_t dp_span = 0;
    for (int64_t u = 0; u < std::min(P, D); ++u) {
      int64_t load = 0;
      for (int64_t t = u; t < D; t += P) load += (t < cnt[0] ? kb[0] : kb[1]) + kTileFixedKb;
      dp_span = std::max(dp_span, load);
    }
    const int64_t sk_span = (U + ctas - 1) / ctas + kTileFixedKb;
    // fixup: flags, then the staged partials in rounds of 6 (step, part) blocks
    const int64_t steps = o.tn / 64;
    const int64_t rounds = nparts > 0 ? (steps + std::max<int64_t>(1, kSkMaxParts / nparts) - 1) /
                                            std::max<int64_t>(1, kSkMaxParts / nparts)
                                      : 0;
    const double fixup = nparts > 0 ? o.fixup + 0.6 * static_cast<double>(rounds) : 0.0;
    const double t = static_cast<double>(dp_span + sk_span - kTileFixedKb) * o.t_kb_long + o.fixed + fixup;
    // stream-K only for a clear gain (5 %) over the data-parallel plans
    if (!have || (force_sk ? t < best.est_us : t < 0.95 * best.est_us)) {
      best = TilePlan{};
      best.cfg = o.cfg;
      best.sk_ctas = static_cast<int>(ctas);
      best.dp_tiles = static_cast<int>(D);
      best.sk_total = U;
      best.sk_u0 = u0;
      best.est_us = t;
      have = true;
    }
  }
  return best;
}

// Problem description and tensor maps of one GEMM for tile configuration cfg.
int build_problem(const MmCall& c, int cfg, GemmProblem* pr, CUtensorMap* maps) {
  const int bn = (cfg == kGemm128 || cfg == kGemmSplit128) ? 128 : 256;
  const int tile_m = cfg == kGemmPair256 ? 256 : 128;
  const int b_box_rows = cfg == kGemm256 ? 256 : 128;   // rows of B one CTA loads
  std::memset(maps, 0, 3 * sizeof(CUtensorMap));
  const bool bcast_a = c.batch > 1 && c.stride_a == 0, bcast_b = c.batch > 1 && c.stride_b == 0;
  const uint64_t ba = bcast_a ? 1 : static_cast<uint64_t>(c.batch), bb = bcast_b ? 1 : static_cast<uint64_t>(c.batch);
  if (c.k > 0) {
    int s = c.a_major == FP8_K_MAJOR ? make_fp8_map(&maps[0], c.a, c.k, c.m, c.lda, 128, ba, c.stride_a)
                                     : make_fp8_map(&maps[0], c.a, c.m, c.k, c.lda, 128, ba, c.stride_a);
    if (s) return s;
    s = c.b_major == FP8_K_MAJOR ? make_fp8_map(&maps[1], c.b, c.k, c.n, c.ldb, b_box_rows, bb, c.stride_b)
                                 : make_fp8_map(&maps[1], c.b, c.n, c.k, c.ldb, 128, bb, c.stride_b);
    if (s) return s;
  }
  // bf16 output through TMA stores when the rows are 16-byte addressable and
  // end on a 16-byte boundary (a B200 run showed the store clipping the row
  // end at 16-byte granularity, writing up to 7 columns past n otherwise):
  // 32 x 32 boxes, 64-byte swizzle (matches the epilogue's staging layout).
  const bool tma_store = aligned(c.d, 16) && ((c.ldd * 2) % 16 == 0) && (c.n % 8 == 0) &&
                         (c.batch <= 1 || (c.stride_d * 2) % 16 == 0);
  if (tma_store) {
    int s = make_map(&maps[2], c.d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.n, c.m, c.ldd * 2, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B, static_cast<uint64_t>(c.batch), static_cast<uint64_t>(c.stride_d) * 2);
    if (s) return s;
  }
  std::memset(pr, 0, sizeof(*pr));
  pr->m = static_cast<int>(c.m);
  pr->n = static_cast<int>(c.n);
  pr->k = static_cast<int>(c.k);
  pr->tiles_m = static_cast<int>((c.m + tile_m - 1) / tile_m);
  pr->tiles_n = static_cast<int>((c.n + bn - 1) / bn);
  pr->num_tiles = pr->tiles_m * pr->tiles_n * static_cast<int>(c.batch);
  pr->batch = static_cast<int>(c.batch);
  pr->bcast_a = bcast_a ? 1 : 0;
  pr->bcast_b = bcast_b ? 1 : 0;
  pr->stride_d = c.stride_d;
  pr->k_blocks = static_cast<int>((c.k + 127) / 128);
  pr->raster_group = 8;
  pr->idesc = idesc_f8(c.fmt_a, c.fmt_b, c.a_major, c.b_major, tile_m, bn);
  pr->a_major = c.a_major;
  pr->b_major = c.b_major;
  pr->scale_a = c.scale_a;
  pr->scale_b = c.scale_b;
  pr->bias = c.bias;
  pr->bias_kind = !c.bias ? 0 : (c.bias_dtype == FP8_DT_BF16 ? 1 : (c.bias_dtype == FP8_DT_E4M3 ? 2 : 3));
  pr->bias_scale = c.bias_scale;
  pr->d = c.d;
  pr->ldd = c.ldd;
  pr->tma_store = tma_store ? 1 : 0;
  return FP8_OK;
}

// Stream-K slots the calls' workspace holds (0: no usable workspace).  A
// two-GEMM launch shares calls[0]'s workspace.
int64_t sk_slots_available(const MmCall* calls, int n) {
  if (!calls[0].ws || calls[0].ws_bytes < kSkFlagBytes + kSkSlotBytes) return 0;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) need = std::max(need, sk_slots_for(calls[i].m, calls[i].n, calls[i].k));
  const int64_t have = static_cast<int64_t>((calls[0].ws_bytes - kSkFlagBytes) / kSkSlotBytes);
  return std::min(need, have);
}

// The plan of a launch: the forced configuration (stream-K when flagged), or
// the cost model's choice over data-parallel, stream-K and split-K schedules.
int plan_launch(const MmCall* calls, int n, int sms, TilePlan* plan, int* split) {
  const int req = calls[0].tile_cfg;
  const bool force_sk = (req & FP8_TILE_STREAMK) != 0;
  const int req_cfg = req & ~FP8_TILE_STREAMK;
  bool batched = false;
  for (int i = 0; i < n; ++i) batched = batched || calls[i].batch > 1;
  const int64_t slots = batched ? 0 : sk_slots_available(calls, n);
  *split = 1;
  // every pair of a stream-K launch on pair tiles must be resident at once
  auto pairs_resident = [&](const TilePlan& pl) {
    if (pl.cfg != kGemmPair256 || pl.sk_ctas == 0) return true;
    int dev = 0;
    const int64_t need = pl.dp_tiles > 0 ? std::min<int64_t>(sms / 2, kSkMaxCtas / 2) : pl.sk_ctas;
    return cudaGetDevice(&dev) == cudaSuccess && gemm_pair_capacity(dev) >= need;
  };
  if (force_sk) {
    if (batched) return FP8_ERR_INVALID_ARG;
    if (slots < (req_cfg == kGemmPair256 ? 2 : 1)) return FP8_ERR_WORKSPACE;
    *plan = pick_tile(calls, n, sms, slots, req_cfg, true);
    if (plan->sk_ctas == 0) return FP8_ERR_WORKSPACE;
    return pairs_resident(*plan) ? FP8_OK : FP8_ERR_UNSUPPORTED;
  }
  if (req_cfg != FP8_TILE_AUTO) {
    *plan = TilePlan{};
    plan->cfg = req_cfg;
  } else {
    // AUTO stays data-parallel: measured on a B200, the stream-K plans the
    // cost model chose were slower inside the benchmark steps (the fixup's
    // flag and copy latency is serialized at the end of the launch)
    *plan = pick_tile(calls, n, sms, 0);
  }
  int& cfg = plan->cfg;
  // Split-K (single-problem launches): few 128 x 128 tiles and a long K leave
  // most SMs idle, so a cluster of S CTAs shares each tile's k-blocks.
  if (cfg == kGemmSplit128 && n != 1) cfg = kGemm128;
  if (cfg == kGemmSplit128 && calls[0].batch > 1) cfg = kGemm128;  // batches already give the tiles
  if (n == 1 && calls[0].batch == 1 && plan->sk_ctas == 0 && (req_cfg == FP8_TILE_AUTO || cfg == kGemmSplit128)) {
    const bool forced = cfg == kGemmSplit128;
    const int64_t tiles = ((calls[0].m + 127) / 128) * ((calls[0].n + 127) / 128);
    const int64_t kb = (calls[0].k + 127) / 128;
    int s = 1;
    if (tiles <= sms && kb >= 2) s = gemm_split_factor(static_cast<int>(tiles), static_cast<int>(kb), sms, forced);
    if (s >= 2) {
      // measured on a B200: moving a 128 x 128 fp32 partial between the SMs of
      // a cluster costs ~1.6 us, parking it ~0.9 us, the cluster launch ~0.5 us
      const double t_split = static_cast<double>(kb / s) * 0.34 + 4.0 + 3.0;
      if (forced || t_split < plan->est_us) {
        cfg = kGemmSplit128;
        *split = s;
      }
    } else if (forced) {
      cfg = kGemm128;
    }
  }
  return FP8_OK;
}

// Enqueue one launch running n (1 or 2) validated GEMMs over one persistent
// tile schedule.  side: writes folded into the launch; fin: rings whose
// quantize deferred its finalize to this launch.
int run_mm_group(const MmCall* calls, int n, const SideWrites* side, cudaStream_t st,
                 const RingFinalize* fin = nullptr, int nfin = 0, const DbiasFinish* dbf = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const int sms = num_sms(dev);
  if (sms <= 0) return cuda_fail(cudaGetLastError());
  TilePlan plan;
  int split = 1;
  int s = plan_launch(calls, n, sms, &plan, &split);
  if (s) return s;
  const int cfg = plan.cfg;
  CUtensorMap maps[6];
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  std::memset(maps, 0, sizeof(maps));
  for (int i = 0; i < n; ++i) {
    if ((s = build_problem(calls[i], cfg, &p.pr[i], &maps[3 * i]))) return s;
    p.any_tma_store |= p.pr[i].tma_store;
  }
  p.nprob = n;
  p.split = cfg == kGemmSplit128 ? split : 1;
  p.tiles0 = p.pr[0].num_tiles;
  p.total_tiles = p.pr[0].num_tiles + (n > 1 ? p.pr[1].num_tiles : 0);
  p.nslots = p.total_tiles;
  p.use_order = 0;
  if (plan.sk_ctas > 0) {
    // stream-K: whole tiles [0, dp_tiles) round robin, the rest by k-block ranges
    p.nslots = plan.dp_tiles;
    p.sk_ctas = plan.sk_ctas;
    p.dp_tiles = plan.dp_tiles;
    p.sk_total = plan.sk_total;
    p.sk_u0 = plan.sk_u0;
    p.sk_flag = static_cast<unsigned*>(calls[0].ws);
    p.sk_part = reinterpret_cast<float*>(static_cast<uint8_t*>(calls[0].ws) + kSkFlagBytes);
  } else if (n == 2 && (cfg == kGemm128 || cfg == kGemm256) && p.pr[0].k_blocks != p.pr[1].k_blocks) {
    // Two problems of unequal k on single-CTA tiles: LPT schedule instead of
    // round robin (the launch's grid is min(tiles, SMs), the schedule's units).
    int nslots = 0;
    if (lpt_schedule(p.pr[0].num_tiles, p.pr[0].k_blocks, p.pr[1].num_tiles, p.pr[1].k_blocks, sms, p.order,
                     &nslots) >= 0) {
      p.nslots = nslots;
      p.use_order = 1;
    }
  }
  p.status = status_ptr(dev);
  if (side) p.side = *side;
  for (int i = 0; i < nfin; ++i) p.fin[i] = fin[i];
  p.nfin = nfin;
  if (dbf) p.dbias = *dbf;
  e = launch_gemm(maps, p, cfg, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return FP8_OK;
}

int run_mm(const MmCall& c, const SideWrites* side, cudaStream_t st, const RingFinalize* fin = nullptr,
           int nfin = 0, const DbiasFinish* dbf = nullptr) {
  return run_mm_group(&c, 1, side, st, fin, nfin, dbf);
}

// D of a GEMM whose contraction is empty (K = 0): every accumulator is 0, so
// D = bias broadcast over the rows (or zero).  Also used for gradients of a
// linear whose contraction dimension is empty.
int run_fill(const MmCall& c, cudaStream_t st) {
  FillParams f;
  std::memset(&f, 0, sizeof(f));
  f.d = c.d;
  f.ldd = c.ldd;
  f.stride_d = c.batch > 1 ? c.stride_d : 0;
  f.m = c.m;
  f.n = c.n;
  f.batch = c.batch;
  f.bias = c.bias;
  f.bias_kind = !c.bias ? 0 : (c.bias_dtype == FP8_DT_BF16 ? 1 : (c.bias_dtype == FP8_DT_E4M3 ? 2 : 3));
  f.bias_scale = c.bias_scale;
  cudaError_t e = launch_fill(f, st);
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

// A bf16 [rows, cols] output (row stride ld) set to zero: the gradient of an
// empty contraction.
int run_zero(void* d, int64_t rows, int64_t cols, int64_t ld, cudaStream_t st) {
  MmCall c{};
  c.m = rows;
  c.n = cols;
  c.d = d;
  c.ldd = ld;
  c.batch = 1;
  return run_fill(c, st);
}

// One validated GEMM call: nothing for an empty output, the fill for an empty
// contraction, else the GEMM kernel.
int run_mm_any(const MmCall& c, cudaStream_t st) {
  if (c.m == 0 || c.n == 0 || c.batch == 0) return FP8_OK;
  if (c.k == 0) return run_fill(c, st);
  return run_mm(c, nullptr, st);
}

RingFinalize ring_fin(void* ring, int H, int fmt, float* amax_out) {
  return RingFinalize{static_cast<float*>(ring), H, fp8_max(fmt), amax_out};
}

QuantizeParams make_qparams(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld_in, int fmt,
                            void* ring, int H, uint8_t* out, int64_t ld_out, float* amax_out, float* scale_out,
                            bool allow_flatten) {
  QuantizeParams p;
  std::memset(&p, 0, sizeof(p));
  p.in = in;
  p.out = out;
  p.ring = static_cast<float*>(ring);
  p.H = H;
  p.fp8_max = fp8_max(fmt);
  p.amax_out = amax_out;
  p.scale_out = scale_out;
  const int es = esize(in_dtype);
  if (allow_flatten && ld_in == cols && ld_out == cols) {  // contiguous: one long row
    p.rows = 1;
    p.cols = rows * cols;
    p.ld_in = p.cols;
    p.ld_out = p.cols;
  } else {
    p.rows = rows;
    p.cols = cols;
    p.ld_in = ld_in;
    p.ld_out = ld_out;
  }
  p.chunks_per_row = (p.cols + 15) / 16;
  p.total_chunks = p.rows * p.chunks_per_row;
  p.vec_ok = aligned(in, 16) && ((p.ld_in * es) % 16 == 0);
  return p;
}

// Current scaling's first pass for the ring-less ones of a and b (either may
// be NULL): zero each one's amax_out, point its dyn_amax there, and reduce
// max |x| into it in one launch.
int amax_pass(int in_dtype, QuantizeParams* a, QuantizeParams* b, cudaStream_t st) {
  const QuantizeParams* d[2] = {nullptr, nullptr};
  SideWrites zero;
  std::memset(&zero, 0, sizeof(zero));
  int n = 0;
  for (QuantizeParams* q : {a, b}) {
    if (!q || q->ring) continue;
    q->dyn_amax = q->amax_out;
    zero.zero_dst[n] = q->amax_out;
    d[n++] = q;
  }
  if (n == 0) return FP8_OK;
  // The amax words start at zero: a one-thread kernel (not a memset, so the
  // amax grid stays a programmatic dependent and prefetches while it runs).
  cudaError_t e = launch_side_writes(zero, st);
  if (e == cudaSuccess) e = launch_amax(in_dtype, d[0], d[1], st);
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

// defer: leave the ring's finalize to the GEMM launch that follows (which
// must then list the ring in its RingFinalize set).
int run_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld_in, int fmt, void* ring,
                 int H, uint8_t* out, int64_t ld_out, float* amax_out, float* scale_out, cudaStream_t st,
                 bool defer = false) {
  QuantizeParams p =
      make_qparams(in, in_dtype, rows, cols, ld_in, fmt, ring, H, out, ld_out, amax_out, scale_out, true);
  p.defer_finalize = defer && ring ? 1 : 0;
  int s = amax_pass(in_dtype, &p, nullptr, st);
  if (s) return s;
  cudaError_t e = launch_quantize(in_dtype, fmt, &p, nullptr, st);
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

// Bytes of a dbias workspace's per-tile counters (16-byte rounded); the
// R x N fp32 partials follow them.
size_t dbias_counter_bytes(int64_t N) {
  const size_t tiles = static_cast<size_t>((N + kDbiasColsPerTile - 1) / kDbiasColsPerTile);
  return (tiles * 4u + 15u) & ~size_t(15);
}

size_t dbias_partial_bytes(int R, int64_t N) {
  return (static_cast<size_t>(R) * static_cast<size_t>(N) * 4u + 15u) & ~size_t(15);
}

// defer: leave both the ring finalize and the column sums to the GEMM
// launch that follows; *dbf then describes the sums it must do.
int run_quantize_dbias(const fp8_quantize_args& g, void* dbias, void* workspace, cudaStream_t st,
                       bool defer = false, DbiasFinish* dbf = nullptr) {
  ColsumParams cp;
  std::memset(&cp, 0, sizeof(cp));
  cp.q = make_qparams(g.in, g.in_dtype, g.rows, g.cols, g.ld_in, g.fmt, g.ring, g.hist_len, g.out, g.ld_out,
                      g.amax_out, g.scale_out, false);
  cp.q.defer_finalize = defer && g.ring ? 1 : 0;
  int s = amax_pass(g.in_dtype, &cp.q, nullptr, st);
  if (s) return s;
  colsum_geometry(g.rows, g.cols, &cp.R, &cp.rows_per_split);
  cp.counters = static_cast<unsigned*>(workspace);
  cp.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + dbias_counter_bytes(g.cols));
  cp.dbias = dbias;
  cp.defer_sum = defer ? 1 : 0;
  if (defer && dbf) *dbf = DbiasFinish{cp.partial, dbias, g.cols, cp.R};
  cudaError_t e = launch_quantize_colsum(g.in_dtype, g.fmt, cp, st);
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

// The backward workspace's bias-gradient part: the tile counters, then the
// partials of the larger of the two column-sum geometries (0 when M or N is 0).
size_t linear_dbias_bytes(int64_t M, int64_t N) {
  if (M <= 0 || N <= 0) return 0;
  int Rd, Rc;
  int64_t rps;
  dbias_geometry(M, N, &Rd, &rps);
  colsum_geometry(M, N, &Rc, &rps);
  return dbias_counter_bytes(N) + dbias_partial_bytes(std::max(Rd, Rc), N);
}

// ring NULL selects current scaling, which reduces the amax into *amax_out
// (required then).
int validate_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld_in, int fmt,
                      void* ring, int H, uint8_t* out, int64_t ld_out, const float* amax_out) {
  if (rows < 0 || cols < 0) return FP8_ERR_INVALID_ARG;
  if (!is_wide(in_dtype) || !is_fmt(fmt)) return FP8_ERR_INVALID_ARG;
  if (ring) {
    if (!ring_len_ok(H) || !aligned(ring, 4)) return FP8_ERR_INVALID_ARG;
  } else if (!amax_out || !aligned(amax_out, 4)) {
    return FP8_ERR_INVALID_ARG;
  }
  if (rows == 0 || cols == 0) return FP8_OK;  // empty: nothing is read or written
  if (!in || !out) return FP8_ERR_INVALID_ARG;
  if (!aligned(in, esize(in_dtype))) return FP8_ERR_INVALID_ARG;
  if (ld_in < cols) return FP8_ERR_INVALID_ARG;
  return check_fp8_matrix(out, ld_out, rows, cols);
}

}  // namespace

int record_cuda_error(cudaError_t e) { return cuda_fail(e); }

int num_sms(int dev) {
  if (dev < 0 || dev >= 64) return 0;
  if (!g_sms[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sms[dev] = v;
  }
  return g_sms[dev];
}

}  // namespace fp8lin

using namespace fp8lin;

extern "C" {

size_t fp8_ring_bytes(int hist_len) {
  return ring_len_ok(hist_len) ? static_cast<size_t>(hist_len + 4) * 4u : 0u;
}

int fp8_ring_init(void* ring, int hist_len, fp8_stream_t stream) {
  if (!ring || !ring_len_ok(hist_len) || !aligned(ring, 4)) return FP8_ERR_INVALID_ARG;
  cudaError_t e = launch_ring_set(static_cast<float*>(ring), hist_len, 1.0f, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

int fp8_ring_seed(void* ring, int hist_len, int fmt, float amax, fp8_stream_t stream) {
  if (!ring || !ring_len_ok(hist_len) || !aligned(ring, 4) || !is_fmt(fmt)) return FP8_ERR_INVALID_ARG;
  float s = 1.0f;
  if (amax > 0.0f && std::isfinite(amax)) {
    volatile float q = fp8_max(fmt) / amax;
    if (std::isfinite(q)) s = q;
  }
  cudaError_t e = launch_ring_set(static_cast<float*>(ring), hist_len, s, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

int fp8_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld_in, int fmt, void* ring,
                 int hist_len, uint8_t* out, int64_t ld_out, float* amax_out, float* scale_out,
                 fp8_stream_t stream) {
  int s = validate_quantize(in, in_dtype, rows, cols, ld_in, fmt, ring, hist_len, out, ld_out, amax_out);
  if (s) return s;
  if (rows == 0 || cols == 0) return FP8_OK;
  return run_quantize(in, in_dtype, rows, cols, ld_in, fmt, ring, hist_len, out, ld_out, amax_out, scale_out,
                      reinterpret_cast<cudaStream_t>(stream));
}

int fp8_quantize_ex(const fp8_quantize_args* q, int flags, fp8_stream_t stream) {
  if (!q || (flags & ~FP8_QUANTIZE_DEFER_RING_STEP)) return FP8_ERR_INVALID_ARG;
  const bool defer = (flags & FP8_QUANTIZE_DEFER_RING_STEP) != 0;
  if (defer && !q->ring) return FP8_ERR_INVALID_ARG;  // a pending step needs a ring
  int s = validate_quantize(q->in, q->in_dtype, q->rows, q->cols, q->ld_in, q->fmt, q->ring, q->hist_len, q->out,
                            q->ld_out, q->amax_out);
  if (s) return s;
  if (q->rows == 0 || q->cols == 0) return FP8_OK;
  return run_quantize(q->in, q->in_dtype, q->rows, q->cols, q->ld_in, q->fmt, q->ring, q->hist_len, q->out,
                      q->ld_out, q->amax_out, q->scale_out, reinterpret_cast<cudaStream_t>(stream), defer);
}

int fp8_ring_finalize(void* ring, int hist_len, int fmt, float* amax_out, fp8_stream_t stream) {
  if (!ring || !aligned(ring, 4) || !ring_len_ok(hist_len) || !is_fmt(fmt)) return FP8_ERR_INVALID_ARG;
  if (amax_out && !aligned(amax_out, 4)) return FP8_ERR_INVALID_ARG;
  cudaError_t e = launch_ring_finalize(ring_fin(ring, hist_len, fmt, amax_out), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

int fp8_quantize_dual(const fp8_quantize_args* a, const fp8_quantize_args* b, fp8_stream_t stream) {
  if (!a || !b) return FP8_ERR_INVALID_ARG;
  int s = validate_quantize(a->in, a->in_dtype, a->rows, a->cols, a->ld_in, a->fmt, a->ring, a->hist_len, a->out,
                            a->ld_out, a->amax_out);
  if (s) return s;
  s = validate_quantize(b->in, b->in_dtype, b->rows, b->cols, b->ld_in, b->fmt, b->ring, b->hist_len, b->out,
                        b->ld_out, b->amax_out);
  if (s) return s;
  if (a->in_dtype != b->in_dtype || a->fmt != b->fmt || (a->ring && a->ring == b->ring)) return FP8_ERR_INVALID_ARG;
  if (!a->ring && !b->ring && a->amax_out == b->amax_out) return FP8_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool ea = a->rows == 0 || a->cols == 0, eb = b->rows == 0 || b->cols == 0;
  if (ea && eb) return FP8_OK;
  if (ea || eb) {
    const fp8_quantize_args* o = ea ? b : a;
    return run_quantize(o->in, o->in_dtype, o->rows, o->cols, o->ld_in, o->fmt, o->ring, o->hist_len, o->out,
                        o->ld_out, o->amax_out, o->scale_out, st);
  }
  QuantizeParams qa = make_qparams(a->in, a->in_dtype, a->rows, a->cols, a->ld_in, a->fmt, a->ring, a->hist_len,
                                   a->out, a->ld_out, a->amax_out, a->scale_out, true);
  QuantizeParams qb = make_qparams(b->in, b->in_dtype, b->rows, b->cols, b->ld_in, b->fmt, b->ring, b->hist_len,
                                   b->out, b->ld_out, b->amax_out, b->scale_out, true);
  if ((s = amax_pass(a->in_dtype, &qa, &qb, st))) return s;
  cudaError_t e = launch_quantize(a->in_dtype, a->fmt, &qa, &qb, st);
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

int fp8_quantize_dbias(const fp8_quantize_args* g, void* dbias, void* workspace, size_t workspace_bytes,
                       fp8_stream_t stream) {
  if (!g) return FP8_ERR_INVALID_ARG;
  int s = validate_quantize(g->in, g->in_dtype, g->rows, g->cols, g->ld_in, g->fmt, g->ring, g->hist_len, g->out,
                            g->ld_out, g->amax_out);
  if (s) return s;
  if (g->rows > kMaxDim || g->cols > kMaxDim) return FP8_ERR_INVALID_ARG;
  if (!dbias || !aligned(dbias, 2)) return FP8_ERR_INVALID_ARG;
  if (g->rows == 0 || g->cols == 0) return FP8_OK;
  const size_t need = fp8_dbias_workspace_bytes(g->rows, g->cols);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return FP8_ERR_WORKSPACE;
  return run_quantize_dbias(*g, dbias, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int fp8_mm_pair(const fp8_mm_args* a, const fp8_mm_args* b, fp8_stream_t stream) {
  if (!a || !b) return FP8_ERR_INVALID_ARG;
  const MmCall c[2] = {mm_call(a, a), mm_call(b, a)};
  int s = validate_mm(c[0]);
  if (s) return s;
  if ((s = validate_mm(c[1]))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool ga = c[0].m > 0 && c[0].n > 0 && c[0].k > 0, gb = c[1].m > 0 && c[1].n > 0 && c[1].k > 0;
  if (ga && gb) return run_mm_group(c, 2, nullptr, st);
  if ((s = run_mm_any(c[0], st))) return s;
  return run_mm_any(c[1], st);
}

int fp8_mm(const fp8_mm_args* a, fp8_stream_t stream) {
  if (!a) return FP8_ERR_INVALID_ARG;
  const MmCall c = mm_call(a, a);
  int s = validate_mm(c);
  if (s) return s;
  return run_mm_any(c, reinterpret_cast<cudaStream_t>(stream));
}

int fp8_mm_batched(const fp8_mm_args* a, int64_t batch, int64_t stride_a, int64_t stride_b, int64_t stride_d,
                   fp8_stream_t stream) {
  if (!a || batch < 0 || stride_a < 0 || stride_b < 0 || stride_d < 0) return FP8_ERR_INVALID_ARG;
  MmCall c = mm_call(a, a);
  c.batch = batch;
  c.stride_a = stride_a;
  c.stride_b = stride_b;
  c.stride_d = stride_d;
  int s = validate_mm(c);
  if (s) return s;
  if (batch == 0 || c.m == 0 || c.n == 0) return FP8_OK;
  if (batch > 1) {
    // batch strides of the fp8 operands are TMA strides: multiples of 16 bytes
    if (stride_a % 16 || stride_b % 16) return FP8_ERR_MISALIGNED;
    // the batches' outputs must not overlap
    if (stride_d < (c.m - 1) * c.ldd + c.n) return FP8_ERR_INVALID_ARG;
    const int64_t tiles = ((c.m + 127) / 128) * ((c.n + 127) / 128) * batch;
    if (tiles > (int64_t(1) << 30)) return FP8_ERR_INVALID_ARG;
  }
  return run_mm_any(c, reinterpret_cast<cudaStream_t>(stream));
}

int fp8_mm_plan(const fp8_mm_args* a, const fp8_mm_args* b, int num_sms, fp8_mm_plan_info* out) {
  if (!a || !out || num_sms <= 0) return FP8_ERR_INVALID_ARG;
  MmCall c[2];
  int n = 0;
  for (const fp8_mm_args* x : {a, b}) {
    if (!x) continue;
    const MmCall m = mm_call(x, a);
    int s = validate_mm(m);
    if (s) return s;
    if (m.m == 0 || m.n == 0 || m.k == 0) continue;  // no GEMM tiles (an empty contraction is a fill)
    c[n++] = m;
  }
  std::memset(out, 0, sizeof(*out));
  if (n == 0) return FP8_OK;
  const int req_cfg = a->tile_cfg & ~FP8_TILE_STREAMK;
  const bool force_sk = (a->tile_cfg & FP8_TILE_STREAMK) != 0;
  const int64_t slots = sk_slots_available(c, n);
  TilePlan plan;
  if (force_sk) {
    if (slots < 1) return FP8_ERR_WORKSPACE;
    plan = pick_tile(c, n, num_sms, slots, req_cfg, true);
  } else if (req_cfg != FP8_TILE_AUTO) {
    plan.cfg = req_cfg;
  } else {
    plan = pick_tile(c, n, num_sms, 0);
  }
  const int cfg = plan.cfg;
  const int64_t tm = cfg == kGemmPair256 ? 256 : 128;
  const int64_t tn = (cfg == kGemm256 || cfg == kGemmPair256) ? 256 : 128;
  int64_t tiles = 0;
  for (int i = 0; i < n; ++i) tiles += ((c[i].m + tm - 1) / tm) * ((c[i].n + tn - 1) / tn);
  const int64_t cap = cfg == kGemmPair256 ? num_sms / 2 : num_sms;
  out->tile_cfg = plan.sk_ctas ? (cfg | FP8_TILE_STREAMK) : cfg;
  out->tiles = tiles;
  const int64_t sk_cap = cfg == kGemmPair256 ? std::min<int64_t>(num_sms / 2, kSkMaxCtas / 2)
                                             : std::min<int64_t>(num_sms, kSkMaxCtas);
  out->units = plan.sk_ctas ? static_cast<int>(plan.dp_tiles > 0 ? sk_cap : plan.sk_ctas)
                            : static_cast<int>(std::max<int64_t>(1, std::min(tiles, cap)));
  out->est_us = req_cfg != FP8_TILE_AUTO && !force_sk ? 0.0 : plan.est_us;
  out->stream_k_ctas = plan.sk_ctas;
  out->dp_tiles = plan.dp_tiles;
  return FP8_OK;
}

size_t fp8_mm_workspace_bytes(int64_t m, int64_t n, int64_t k) { return sk_bytes_for(m, n, k); }

// One size for fp8_dbias and the column-sum quantize (standalone or in the
// linear backward): the larger of the two geometries' partials.
size_t fp8_dbias_workspace_bytes(int64_t M, int64_t N) { return linear_dbias_bytes(M, N); }

int fp8_dbias(const void* g, int g_dtype, int64_t M, int64_t N, int64_t ldg, const float* g_scale, void* dbias,
              void* workspace, size_t workspace_bytes, fp8_stream_t stream) {
  if (M < 0 || N < 0 || M > kMaxDim || N > kMaxDim) return FP8_ERR_INVALID_ARG;
  if (!is_wide(g_dtype) && !is_fp8(g_dtype)) return FP8_ERR_INVALID_ARG;
  if (!g || !dbias || ldg < N || !aligned(g, esize(g_dtype)) || !aligned(dbias, 2)) return FP8_ERR_INVALID_ARG;
  if (is_fp8(g_dtype) && !g_scale) return FP8_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FP8_OK;
  const size_t need = fp8_dbias_workspace_bytes(M, N);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return FP8_ERR_WORKSPACE;
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
  p.counters = static_cast<unsigned*>(workspace);
  p.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + dbias_counter_bytes(N));
  const int es = esize(g_dtype);
  p.vec_ok = is_fp8(g_dtype) ? (aligned(g, 8) && (ldg % 8 == 0)) : (aligned(g, 16) && ((ldg * es) % 16 == 0));
  cudaError_t e = launch_dbias(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

size_t fp8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)K;
  return linear_dbias_bytes(M, N);
}

int fp8_linear_forward(const fp8_linear_fwd_args* a, fp8_stream_t stream) {
  if (!a) return FP8_ERR_INVALID_ARG;
  const int64_t M = a->M, N = a->N, K = a->K;
  if (M < 0 || N < 0 || K < 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8_ERR_INVALID_ARG;
  if (!is_fmt(a->fmt_x) || !is_fmt(a->fmt_w)) return FP8_ERR_INVALID_ARG;
  if (!a->sx_out || !a->sw_out) return FP8_ERR_INVALID_ARG;
  // operands and output with elements need their buffers (validated below)
  if ((M > 0 && K > 0 && !a->x) || (N > 0 && K > 0 && !a->w)) return FP8_ERR_INVALID_ARG;
  const bool xq = is_fp8(a->x_dtype), wq = is_fp8(a->w_dtype);
  if (!xq && !is_wide(a->x_dtype)) return FP8_ERR_INVALID_ARG;
  if (!wq && !is_wide(a->w_dtype)) return FP8_ERR_INVALID_ARG;
  int s;
  if (xq) {
    if (a->x_dtype - FP8_DT_E4M3 != a->fmt_x || !a->x_scale_in) return FP8_ERR_INVALID_ARG;
    if ((s = check_fp8_matrix(a->x, a->ldx, M, K))) return s;
  } else if ((s = validate_quantize(a->x, a->x_dtype, M, K, a->ldx, a->fmt_x, a->ring_x, a->hist_len, a->x8,
                                    a->ldx8, a->amax_x_out))) {
    return s;
  }
  if (wq) {
    if (a->w_dtype - FP8_DT_E4M3 != a->fmt_w || !a->w_scale_in) return FP8_ERR_INVALID_ARG;
    if ((s = check_fp8_matrix(a->w, a->ldw, N, K))) return s;
  } else if ((s = validate_quantize(a->w, a->w_dtype, N, K, a->ldw, a->fmt_w, a->ring_w, a->hist_len, a->w8,
                                    a->ldw8, a->amax_w_out))) {
    return s;
  }
  if (!xq && !wq && a->ring_x && a->ring_x == a->ring_w) return FP8_ERR_INVALID_ARG;
  if (!xq && !wq && !a->ring_x && !a->ring_w && a->amax_x_out == a->amax_w_out) return FP8_ERR_INVALID_ARG;
  const uint8_t* x8 = xq ? static_cast<const uint8_t*>(a->x) : a->x8;
  const uint8_t* w8 = wq ? static_cast<const uint8_t*>(a->w) : a->w8;
  MmCall c{M, N, K, x8, a->fmt_x, FP8_K_MAJOR, xq ? a->ldx : a->ldx8, w8, a->fmt_w, FP8_K_MAJOR,
           wq ? a->ldw : a->ldw8, xq ? a->x_scale_in : a->sx_out, wq ? a->w_scale_in : a->sw_out,
           a->bias, a->bias_dtype, a->bias_scale, a->y, a->ldy, FP8_TILE_AUTO};
  if ((s = validate_mm(c))) return s;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Empty sizes: an operand with no elements is neither quantized nor
  // side-written (its ring does not step); a non-empty one is, whatever the
  // other sizes.  y is written when it has elements: the GEMM, or the bias
  // alone (zero without one) when the contraction K is empty.
  const bool x_live = M > 0 && K > 0, w_live = N > 0 && K > 0;
  const bool gemm = M > 0 && N > 0 && K > 0;
  SideWrites side;
  std::memset(&side, 0, sizeof(side));
  if (xq && x_live) { side.copy_src[0] = a->x_scale_in; side.copy_dst[0] = a->sx_out; side.zero_dst[0] = a->amax_x_out; }
  if (wq && w_live) { side.copy_src[1] = a->w_scale_in; side.copy_dst[1] = a->sw_out; side.zero_dst[1] = a->amax_w_out; }
  if (!gemm) {
    // No GEMM follows: a quantize finishes its ring step in its own last block.
    if (!xq && x_live && (s = run_quantize(a->x, a->x_dtype, M, K, a->ldx, a->fmt_x, a->ring_x, a->hist_len, a->x8,
                                           a->ldx8, a->amax_x_out, a->sx_out, st)))
      return s;
    if (!wq && w_live && (s = run_quantize(a->w, a->w_dtype, N, K, a->ldw, a->fmt_w, a->ring_w, a->hist_len, a->w8,
                                           a->ldw8, a->amax_w_out, a->sw_out, st)))
      return s;
    if (side.copy_dst[0] || side.copy_dst[1]) {
      cudaError_t e = launch_side_writes(side, st);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    return run_mm_any(c, st);  // M, N > 0 here means K == 0: y = bias
  }
  // The quantize launches only max-reduce into their rings; the GEMM, which
  // waits for them to complete anyway, finishes both ring steps.
  RingFinalize fin[2];
  int nfin = 0;
  if (!xq && a->ring_x) fin[nfin++] = ring_fin(a->ring_x, a->hist_len, a->fmt_x, a->amax_x_out);
  if (!wq && a->ring_w) fin[nfin++] = ring_fin(a->ring_w, a->hist_len, a->fmt_w, a->amax_w_out);
  if (!xq && !wq && a->x_dtype == a->w_dtype && a->fmt_x == a->fmt_w) {
    // x and w in one launch
    QuantizeParams qx = make_qparams(a->x, a->x_dtype, M, K, a->ldx, a->fmt_x, a->ring_x, a->hist_len, a->x8,
                                     a->ldx8, a->amax_x_out, a->sx_out, true);
    QuantizeParams qw = make_qparams(a->w, a->w_dtype, N, K, a->ldw, a->fmt_w, a->ring_w, a->hist_len, a->w8,
                                     a->ldw8, a->amax_w_out, a->sw_out, true);
    qx.defer_finalize = a->ring_x ? 1 : 0;
    qw.defer_finalize = a->ring_w ? 1 : 0;
    if ((s = amax_pass(a->x_dtype, &qx, &qw, st))) return s;
    cudaError_t e = launch_quantize(a->x_dtype, a->fmt_x, &qx, &qw, st);
    if (e != cudaSuccess) return cuda_fail(e);
  } else {
    if (!xq && (s = run_quantize(a->x, a->x_dtype, M, K, a->ldx, a->fmt_x, a->ring_x, a->hist_len, a->x8, a->ldx8,
                                 a->amax_x_out, a->sx_out, st, true)))
      return s;
    if (!wq && (s = run_quantize(a->w, a->w_dtype, N, K, a->ldw, a->fmt_w, a->ring_w, a->hist_len, a->w8, a->ldw8,
                                 a->amax_w_out, a->sw_out, st, true)))
      return s;
  }
  return run_mm(c, &side, st, fin, nfin);
}

int fp8_linear_backward(const fp8_linear_bwd_args* a, fp8_stream_t stream) {
  if (!a) return FP8_ERR_INVALID_ARG;
  const int64_t M = a->M, N = a->N, K = a->K;
  if (M < 0 || N < 0 || K < 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8_ERR_INVALID_ARG;
  if (!is_fmt(a->fmt_g) || !is_fmt(a->fmt_x) || !is_fmt(a->fmt_w)) return FP8_ERR_INVALID_ARG;
  if (!a->sg_out || (M > 0 && N > 0 && !a->g)) return FP8_ERR_INVALID_ARG;
  const bool gq = is_fp8(a->g_dtype);
  if (!gq && !is_wide(a->g_dtype)) return FP8_ERR_INVALID_ARG;
  int s;
  if (gq) {
    if (a->g_dtype - FP8_DT_E4M3 != a->fmt_g || !a->g_scale_in) return FP8_ERR_INVALID_ARG;
    if ((s = check_fp8_matrix(a->g, a->ldg, M, N))) return s;
  } else if ((s = validate_quantize(a->g, a->g_dtype, M, N, a->ldg, a->fmt_g, a->ring_g, a->hist_len, a->g8,
                                    a->ldg8, a->amax_g_out))) {
    return s;
  }
  const uint8_t* g8 = gq ? static_cast<const uint8_t*>(a->g) : a->g8;
  const int64_t ldg8 = gq ? a->ldg : a->ldg8;
  const float* sg = gq ? a->g_scale_in : a->sg_out;
  // dX[M,K] = G8[M,N] . W8[N,K]: A = G8 K-major, B(j=k, n) = W8[n, k] MN-major.
  MmCall cdx{M, K, N, g8, a->fmt_g, FP8_K_MAJOR, ldg8, a->w8, a->fmt_w, FP8_MN_MAJOR, a->ldw8,
             sg, a->sw, nullptr, 0, nullptr, a->dx, a->lddx, FP8_TILE_AUTO};
  // dW[N,K] = G8^T . X8: A(i=n, m) = G8[m, n] MN-major, B(j=k, m) = X8[m, k] MN-major.
  MmCall cdw{N, K, M, g8, a->fmt_g, FP8_MN_MAJOR, ldg8, a->x8, a->fmt_x, FP8_MN_MAJOR, a->ldx8,
             sg, a->sx, nullptr, 0, nullptr, a->dw, a->lddw, FP8_TILE_AUTO};
  if (a->need_dx && (s = validate_mm(cdx))) return s;
  if (a->need_dw && (s = validate_mm(cdw))) return s;
  const size_t ws_need = a->need_dbias ? linear_dbias_bytes(M, N) : 0;
  if (a->need_dbias && N > 0) {
    if (!a->dbias || !aligned(a->dbias, 2)) return FP8_ERR_INVALID_ARG;
    if (ws_need && (!a->workspace || a->workspace_bytes < ws_need || !aligned(a->workspace, 16)))
      return FP8_ERR_WORKSPACE;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Empty sizes: g is quantized (or side-written) only when it has elements;
  // each requested gradient with elements is written -- by its GEMM, or as
  // zero when its contraction is empty (dX: N = 0; dW: M = 0; dbias: M = 0).
  const bool g_live = M > 0 && N > 0;
  const bool dx_live = a->need_dx && M > 0 && K > 0, dw_live = a->need_dw && N > 0 && K > 0;
  const bool db_live = a->need_dbias && N > 0;
  const bool dx_gemm = dx_live && N > 0, dw_gemm = dw_live && M > 0;
  SideWrites side;
  std::memset(&side, 0, sizeof(side));
  bool side_pending = false;
  bool dbias_done = false;
  // With a GEMM to follow, the quantize of g leaves its ring step to it.
  const bool gemm_follows = dx_gemm || dw_gemm;
  RingFinalize fin[1];
  int nfin = 0;
  DbiasFinish dbf{};
  if (g_live) {
    if (!gq && gemm_follows && a->ring_g) fin[nfin++] = ring_fin(a->ring_g, a->hist_len, a->fmt_g, a->amax_g_out);
    if (gq) {
      side.copy_src[0] = a->g_scale_in; side.copy_dst[0] = a->sg_out; side.zero_dst[0] = a->amax_g_out;
      side_pending = true;
    } else if (db_live) {
      // quantize g and sum its columns in the same pass over g
      const fp8_quantize_args qg = {a->g, a->g_dtype, M, N, a->ldg, a->fmt_g, a->ring_g, a->hist_len,
                                    a->g8, a->ldg8, a->amax_g_out, a->sg_out};
      if ((s = run_quantize_dbias(qg, a->dbias, a->workspace, st, gemm_follows, &dbf))) return s;
      dbias_done = true;
    } else if ((s = run_quantize(a->g, a->g_dtype, M, N, a->ldg, a->fmt_g, a->ring_g, a->hist_len, a->g8, a->ldg8,
                                 a->amax_g_out, a->sg_out, st, gemm_follows))) {
      return s;
    }
  }
  if (dx_gemm && dw_gemm) {  // one launch for both (they share the G8 operand)
    const MmCall both[2] = {cdx, cdw};
    if ((s = run_mm_group(both, 2, side_pending ? &side : nullptr, st, fin, nfin, dbf.partial ? &dbf : nullptr)))
      return s;
    side_pending = false;
  } else if (dx_gemm || dw_gemm) {
    if ((s = run_mm(dx_gemm ? cdx : cdw, side_pending ? &side : nullptr, st, fin, nfin,
                    dbf.partial ? &dbf : nullptr)))
      return s;
    side_pending = false;
  }
  if (side_pending) {
    cudaError_t e = launch_side_writes(side, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (dx_live && !dx_gemm && (s = run_zero(a->dx, M, K, a->lddx, st))) return s;
  if (dw_live && !dw_gemm && (s = run_zero(a->dw, N, K, a->lddw, st))) return s;
  if (db_live && !dbias_done) {
    if (M == 0) {
      if ((s = run_zero(a->dbias, 1, N, N, st))) return s;
    } else if ((s = fp8_dbias(a->g, a->g_dtype, M, N, a->ldg, a->g_scale_in, a->dbias, a->workspace,
                              a->workspace_bytes, stream))) {
      return s;
    }
  }
  return FP8_OK;
}

int fp8_wait_selftest(const void* flag, uint64_t limit_ns, int* results, fp8_stream_t stream) {
  if (!flag || !results || !aligned(flag, 4) || !aligned(results, 4)) return FP8_ERR_INVALID_ARG;
  if (limit_ns == 0 || limit_ns > 2000000000ull) return FP8_ERR_INVALID_ARG;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  int* status = status_ptr(dev);
  if (!status) return cuda_fail(cudaGetLastError());
  e = launch_wait_selftest(static_cast<const uint32_t*>(flag), status, results, limit_ns,
                           reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP8_OK : cuda_fail(e);
}

int fp8_get_device_status(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8_ERR_CUDA;
  int* p = status_ptr(dev);
  if (!p) return cuda_fail(cudaGetLastError());
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  return v;
}

const char* fp8_status_string(int status) {
  switch (status) {
    case FP8_OK: return "ok";
    case FP8_ERR_INVALID_ARG: return "invalid argument";
    case FP8_ERR_UNSUPPORTED: return "unsupported";
    case FP8_ERR_MISALIGNED: return "fp8 matrix misaligned (ld % 16 != 0 or base not 16-byte aligned)";
    case FP8_ERR_CUDA: return g_err[0] ? g_err : "CUDA error";
    case FP8_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    case FP8_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FP8_ERR_TOO_LARGE: return "request exceeds the fixed scratch of a no-allocation entry point";
    default: return "unknown status";
  }
}

const char* fp8_version(void) { return "fp8lin 0.1 sm_100a"; }

}  // extern "C"
