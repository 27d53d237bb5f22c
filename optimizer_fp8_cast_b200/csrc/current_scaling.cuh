// current_scaling.cuh — amax pass of current (just-in-time) scaling: the scale of a cast is
// derived from the amax of the very tensor being cast, instead of from the amax history of
// earlier steps.
//
// Method: the FP8Tensor quantize step of "FP8 混合精度训练工程实践" §四 measures amax = max|x|
// of the tensor it is about to quantise; applied at once (no delay) with the scale rule of
// "LLM FP8 微调上线生产实战" 核心原理 — scale = (FP8_MAX / amax) / 2^margin, 0 -> 1, a
// non-finite amax keeps the previous scale — this is the current-scaling recipe.
// One persistent launch per group of up to 8 tensors: each CTA walks its share of every
// tensor with 16-byte loads (8 BF16), keeps a 16-bit SIMD max of the magnitude bits, and each
// warp max-accumulates into a per-tensor word of a small workspace; the CTA that finishes last
// (ticket counter in the same workspace) turns every amax into its scale and zeroes the words
// again. The cast itself then runs as usual with that scale (and records the amax in the
// caller's slot). Traffic: 2 B read per element, and the cast reads the tensors again. This pass
// takes them last to first with loads of normal L2 priority, so the cast, going first to last,
// starts on what the pass read most recently: on the 4096 step (X, W, dY: 168 MB) that part is
// still in L2 and the cast launch pair takes 80.6 instead of 85.4 µs.
#pragma once

#include "ptx.cuh"
#include "scale_update.cuh"

namespace fp8t {
namespace current {

constexpr int kThreads = 256;
constexpr int kMaxTensors = 8;

struct Group {
  const uint4* x[kMaxTensors];        // BF16 data, 8 elements per uint4
  int64_t nvec[kMaxTensors];          // numel / 8
  float* scale[kMaxTensors];
  float fp8_max[kMaxTensors];
  int32_t n, margin;
  unsigned int* ws;                   // [kMaxTensors] amax bits, then the ticket: zero on entry,
                                      // left zero
};

__global__ void __launch_bounds__(kThreads) k_current_amax(const __grid_constant__ Group g) {
  const int tid = threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  // last tensor first: the cast launch that follows reads the tensors first to last, so it starts
  // on the ones this pass read most recently, still in L2
  for (int t = g.n - 1; t >= 0; --t) {
    const uint4* __restrict__ x = g.x[t];
    uint32_t m2 = 0;
    int64_t v = static_cast<int64_t>(blockIdx.x) * kThreads + tid;
    for (; v + 3 * stride < g.nvec[t]; v += 4 * stride) {      // four 16-byte loads in flight
      uint4 a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = __ldg(x + v + u * stride);   // kept in L2 for the cast
#pragma unroll
      for (int u = 0; u < 4; ++u)
        m2 = __vmaxu2(__vmaxu2(m2, __vmaxu2(a[u].x & 0x7FFF7FFFu, a[u].y & 0x7FFF7FFFu)),
                      __vmaxu2(a[u].z & 0x7FFF7FFFu, a[u].w & 0x7FFF7FFFu));
    }
    for (; v < g.nvec[t]; v += stride) {
      const uint4 a = __ldg(x + v);
      m2 = __vmaxu2(__vmaxu2(m2, __vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu)),
                    __vmaxu2(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu));
    }
    uint32_t m = __reduce_max_sync(0xffffffffu, max(m2 & 0xFFFFu, m2 >> 16));
    if ((tid & 31) == 0 && m) {
      if (m > 0x7F80u) m = 0x7FC0u;                              // canonical NaN
      atomicMax(g.ws + t, m << 16);
    }
  }
  __shared__ int s_last;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(g.ws + kMaxTensors, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int warp = tid >> 5;
  if (warp < g.n && (tid & 31) == 0) {
    const uint32_t rep = *reinterpret_cast<volatile unsigned int*>(g.ws + warp) & 0x7FFFFFFFu;
    const float prev = *reinterpret_cast<volatile float*>(g.scale[warp]);
    *g.scale[warp] = scale::next_scale(rep, g.fp8_max[warp], g.margin, prev);
    g.ws[warp] = 0u;
  }
  if (tid == 0) atomicExch(g.ws + kMaxTensors, 0u);
}

}  // namespace current
}  // namespace fp8t
