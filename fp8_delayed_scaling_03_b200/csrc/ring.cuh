// ring.cuh -- the delayed-scaling ring step done by one warp, for rings whose
// quantize left the step pending (its blocks only max-reduced into the
// scratch word): the GEMM of a fused linear, and fp8_ring_finalize after a
// data-parallel all-reduce of the scratch word.
#pragma once

#include "device.cuh"
#include "internal.h"

namespace fp8lin {

// Completes a delayed-scaling step for a ring whose quantize deferred it (its
// blocks only max-reduced into the scratch word).  Runs after
// griddepcontrol.wait, so every block's reduction is visible and nothing else
// touches the ring until this grid completes.  Same rule as the quantize's
// own last-block finalize: hist[step % H] = amax, window max over the history
// with the new amax in place of the overwritten slot, next scale, step + 1.
__device__ __forceinline__ void ring_finalize_warp(const RingFinalize& f, int lane) {
  uint32_t* words = reinterpret_cast<uint32_t*>(f.ring);
  const int H = f.H;
  const uint32_t step = words[ring_step(H)];
  const float a = __uint_as_float(words[ring_scratch(H)]);
  const float s = f.ring[H];
  const uint32_t slot = step % static_cast<uint32_t>(H);
  float m = a;
  for (int i = lane; i < H; i += 32)
    if (static_cast<uint32_t>(i) != slot) m = fmaxf(m, f.ring[i]);
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) {
    f.ring[slot] = a;
    f.ring[H] = next_scale(s, m, f.fp8_max);
    words[ring_step(H)] = step + 1;
    words[ring_scratch(H)] = 0u;
    if (f.amax_out) *f.amax_out = a;
  }
}

}  // namespace fp8lin
