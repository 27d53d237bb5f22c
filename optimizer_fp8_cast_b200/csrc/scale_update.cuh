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

// Next scale from the representative amax (its magnitude bits): FP8_MAX / rep, times 2^-margin;
// rep 0 gives 1; NaN or infinity keeps the previous scale; an overflow to infinity gives FLT_MAX.
__device__ __forceinline__ float next_scale(uint32_t rep, float fmax, int margin, float prev) {
  if (rep >= 0x7F800000u) return prev;
  if (rep == 0u) return 1.0f;
  const float pow2 = __uint_as_float(static_cast<uint32_t>(127 - margin) << 23);
  float s = __fmul_rn(__fdiv_rn(fmax, __uint_as_float(rep)), pow2);
  if (isinf(s)) s = 3.40282346638528859812e+38f;                // FLT_MAX
  return s;
}

// Pull a tensor's history and scale into this SM's L1 (non-binding prefetches, one 128-byte
// line per lane and step). Kernels that finish with an update issue it ahead of their ticket, so
// the CTA that turns out to be last reads its state from L1; nothing but that update writes these
// words during the launch, and L1 holds no older copy of them (it starts each launch empty).
__device__ __forceinline__ void warp_prefetch_state(const float* h, int H, const float* scale) {
  const int lane = threadIdx.x & 31;
  for (int i = 32 * lane; i < H; i += 32 * 32)
    asm volatile("prefetch.global.L1 [%0];" ::"l"(h + i));
  if (lane == 0) asm volatile("prefetch.global.L1 [%0];" ::"l"(scale));
}

// The same update for one tensor, done by one warp (used inside other kernels once their amax
// is complete). The roll goes from the top down in chunks of 32 x kPer entries: every lane
// reads its kPer entries (all loads in flight at once), the warp synchronises, then writes them
// one place higher; a history of up to 1025 entries takes a single round trip to memory.
// amax is read with a volatile load: other CTAs of the calling kernel accumulated it.
template <int kPer = 32>
__device__ __forceinline__ void warp_update(float* amax, float* h, int H, float fmax, bool algo_max,
                                            int margin, float* scale, float* scale_inv) {
  const int lane = threadIdx.x & 31;
  const float a = *reinterpret_cast<volatile float*>(amax);
  uint32_t m = __float_as_uint(a) & 0x7FFFFFFFu;
  for (int top = H - 1; top >= 1; top -= 32 * kPer) {
    float v[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = top - lane - 32 * j;
      v[j] = i >= 1 ? h[i - 1] : 0.0f;
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = top - lane - 32 * j;
      if (i >= 1) {
        h[i] = v[j];
        if (algo_max) m = max(m, __float_as_uint(v[j]) & 0x7FFFFFFFu);
      }
    }
    __syncwarp();
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if (lane == 0) {
    const uint32_t rep = algo_max ? m : (__float_as_uint(a) & 0x7FFFFFFFu);
    h[0] = a;
    const float s = next_scale(rep, fmax, margin, *scale);
    *scale = s;
    *scale_inv = __fdiv_rn(1.0f, s);
    *amax = 0.0f;
  }
}

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
    const float s = next_scale(rep, fp8_max[t], margin, scale[t]);
    scale[t] = s;
    scale_inv[t] = __fdiv_rn(1.0f, s);
    amax[t] = 0.0f;                                           // consumed: ready to accumulate
  }
}

}  // namespace scale
}  // namespace fp8t
