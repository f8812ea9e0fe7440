// partials.cuh -- fixed-order sum of R column partials (stride ld floats),
// shared by the bias-gradient reductions.  Split r goes to accumulator r % 16
// and the 16 accumulators are combined pairwise in a fixed tree, so the result
// depends only on R and the partials; sixteen loads are in flight at a time.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fp8lin {

__device__ __forceinline__ float sum_partials(const float* col, int64_t ld, int R) {
  float acc[16];
  #pragma unroll
  for (int u = 0; u < 16; ++u) acc[u] = 0.0f;
  int r = 0;
  for (; r + 16 <= R; r += 16) {
    float t[16];
    #pragma unroll
    for (int u = 0; u < 16; ++u) t[u] = __ldcg(col + static_cast<int64_t>(r + u) * ld);
    #pragma unroll
    for (int u = 0; u < 16; ++u) acc[u] += t[u];
  }
  if (r < R) {
    float t[16];
    #pragma unroll
    for (int u = 0; u < 16; ++u) t[u] = (r + u < R) ? __ldcg(col + static_cast<int64_t>(r + u) * ld) : 0.0f;
    #pragma unroll
    for (int u = 0; u < 16; ++u) acc[u] += t[u];
  }
  #pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
    #pragma unroll
    for (int u = 0; u < w; ++u) acc[u] = acc[u] + acc[u + w];
  }
  return acc[0];
}

}  // namespace fp8lin
