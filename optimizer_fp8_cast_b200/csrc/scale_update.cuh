// scale_update.cuh — amax-history roll and next-scale computation, one CTA per tensor.
//
// Method: "LLM FP8 微调上线生产实战", 核心原理 — scale = (FP8_MAX / amax) / 2^margin, with the
// representative amax taken from a history window (its max, or its most recent entry) and the
// scale used by the next iteration. History row t is [H] floats, entry 0 newest; the roll moves
// entries i-1 -> i from the top down in chunks of the block size (read, barrier, write,
// barrier), so no entry is overwritten before it is read. The window max is a u32 max of the
// magnitude bits, which orders non-negative floats and puts NaN above infinity. Each consumed
// amax slot is reset to 0 so that the next step's casts can max-accumulate into it.
// Latency-bound: n * (8H + 16) bytes.
#pragma once

#include "ptx.cuh"

namespace fp8t {
namespace scale {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    k_scale_update(float* __restrict__ amax, float* __restrict__ hist, int H,
                   const float* __restrict__ fp8_max, int algo_max, int margin,
                   float* __restrict__ scale, float* __restrict__ scale_inv) {
  __shared__ uint32_t red[kThreads / 32];
  const int t = blockIdx.x;
  float* h = hist + static_cast<int64_t>(t) * H;
  const float a = amax[t];
  uint32_t m = __float_as_uint(a) & 0x7FFFFFFFu;

  for (int top = H - 1; top >= 1; top -= kThreads) {
    const int i = top - static_cast<int>(threadIdx.x);
    float v = 0.0f;
    if (i >= 1) v = h[i - 1];
    __syncthreads();
    if (i >= 1) {
      h[i] = v;
      if (algo_max) m = max(m, __float_as_uint(v) & 0x7FFFFFFFu);
    }
    __syncthreads();
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t rep = 0;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) rep = max(rep, red[i]);
    if (!algo_max) rep = __float_as_uint(a) & 0x7FFFFFFFu;
    h[0] = a;
    float s;
    if (rep >= 0x7F800000u) {
      s = scale[t];                                           // NaN or inf: keep
    } else if (rep == 0u) {
      s = 1.0f;
    } else {
      const float pow2 = __uint_as_float(static_cast<uint32_t>(127 - margin) << 23);
      s = __fdiv_rn(fp8_max[t], __uint_as_float(rep));
      s = __fmul_rn(s, pow2);
      if (isinf(s)) s = 3.40282346638528859812e+38f;          // FLT_MAX
    }
    scale[t] = s;
    scale_inv[t] = __fdiv_rn(1.0f, s);
    amax[t] = 0.0f;                                           // consumed: ready to accumulate
  }
}

}  // namespace scale
}  // namespace fp8t
