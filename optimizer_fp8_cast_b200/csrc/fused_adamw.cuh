// fused_adamw.cuh — multi-tensor global-norm pass and fused AdamW update.
//
// Method: "算子与编译器：FP8 训练与优化器 Kernel", Fused Optimizer 的意义 (read the gradient,
// update the moments, bias correction, weight decay and the parameter update in one kernel) and
// 优化器 kernel 的带宽账 (every split kernel re-reads grad, m, v, param); the unscale and clip in
// front of it come from FP8 训练主路径图 and "FP8 混合精度训练工程实践" §四.
//
// Two kernels per batch of up to kMaxTensors tensors, whose table travels in the kernel
// parameters (no host->device copy, so a step captures cleanly into a CUDA graph):
//   k_adamw_sumsq   fixed grid of kSumsqBlocks CTAs striding over 8192-element chunks; each CTA
//                   writes the FP64 sum of f32(g)^2 over its chunks to one workspace slot.
//   k_adamw_update  persistent CTAs; each first reduces all workspace slots in a fixed order
//                   (so every CTA derives the identical norm and clip factor), then streams its
//                   chunks: 16-byte loads of g (8 BF16) and 2 x 16-byte loads of m, v, p.
// Traffic: 2 B/param for the norm pass, 28 B/param for the update (g 2 + m, v, p 4 each read,
// m, v, p 4 each + BF16 weight 2 written).
// Every f32 operation is an explicit round-to-nearest intrinsic, so no multiply-add is fused.
#pragma once

#include "ptx.cuh"

namespace fp8t {
namespace adamw {

constexpr int kMaxTensors = 256;
constexpr int kThreads = 256;
constexpr int kVec = 8;                                  // elements per 16-byte BF16 vector
constexpr int64_t kChunk = 4 * kThreads * kVec;          // 8192 elements per chunk
constexpr int kSumsqBlocks = 592;

struct Batch {
  int32_t n;
  int32_t first;                                          // 1 for the batch that reports
  int64_t chunk_start[kMaxTensors + 1];                   // prefix sums of chunks per tensor
  int64_t numel[kMaxTensors];
  float* master[kMaxTensors];
  float* m[kMaxTensors];
  float* v[kMaxTensors];
  const uint16_t* g[kMaxTensors];
  uint16_t* w[kMaxTensors];
};

struct Scalars {            // host-computed, rounded once to f32 (double where noted)
  float beta1, beta2, omb1, omb2, decay, step_size, bc2_sqrt, eps, inv_s, max_norm;
  double inv_s_d;
  // device step counter (may be null): the step is read from step_slot (counter + 1, written by
  // the norm pass), step_size and bc2_sqrt are formed on the device, and the counter is advanced
  // by the first CTA of the first update launch unless the step is skipped
  int64_t* d_step;
  const int64_t* step_slot;
  double lr_d, beta1_d, beta2_d;
};

__device__ __forceinline__ int find_tensor(const Batch& b, int64_t chunk) {
  int lo = 0, hi = b.n - 1;                               // largest t with chunk_start[t] <= chunk
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.chunk_start[mid] <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float bf16_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_rne(float f) {
  const uint32_t b = __float_as_uint(f);
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0x7FC0u;
  return (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
}

template <typename T>
__device__ __forceinline__ T block_sum_fixed(T v, T* sh) {  // deterministic tree over the block
  sh[threadIdx.x] = v;
  __syncthreads();
#pragma unroll
  for (int s = kThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] = sh[threadIdx.x] + sh[threadIdx.x + s];
    __syncthreads();
  }
  const T r = sh[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads)
    k_adamw_sumsq(const __grid_constant__ Batch b, double* __restrict__ partials,
                  const int64_t* __restrict__ step_counter, int64_t* __restrict__ step_slot) {
  __shared__ double sh[kThreads];
  // the step this call performs, for the update kernels that run after this one
  if (step_counter && blockIdx.x == 0 && threadIdx.x == 0) *step_slot = *step_counter + 1;
  double acc = 0.0;
  const int64_t nchunks = b.chunk_start[b.n];
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const int t = find_tensor(b, c);
    const int64_t base = (c - b.chunk_start[t]) * kChunk;
    const uint16_t* __restrict__ g = b.g[t];
    const int64_t n = b.numel[t];
    uint4 gv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = base + static_cast<int64_t>(u * kThreads + threadIdx.x) * kVec;
      if (e + kVec <= n) gv[u] = ld_stream_u4(g + e);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = base + static_cast<int64_t>(u * kThreads + threadIdx.x) * kVec;
      if (e + kVec <= n) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&gv[u]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const double lo = bf16_to_f32(w[j] & 0xFFFFu), hi = bf16_to_f32(w[j] >> 16);
          acc = __dadd_rn(acc, __dmul_rn(lo, lo));
          acc = __dadd_rn(acc, __dmul_rn(hi, hi));
        }
      } else {
        for (int64_t i = e; i < n && i < e + kVec; ++i) {
          const double x = bf16_to_f32(g[i]);
          acc = __dadd_rn(acc, __dmul_rn(x, x));
        }
      }
    }
  }
  const double total = block_sum_fixed(acc, sh);
  if (threadIdx.x == 0) partials[blockIdx.x] = total;
}

__device__ __forceinline__ void adam_one(float& p, float& m, float& v, float g, const Scalars& k,
                                         float f) {
  const float gg = __fmul_rn(g, f);
  const float mm = __fadd_rn(__fmul_rn(k.beta1, m), __fmul_rn(k.omb1, gg));
  const float vv = __fadd_rn(__fmul_rn(k.beta2, v), __fmul_rn(k.omb2, __fmul_rn(gg, gg)));
  float pp = __fmul_rn(p, k.decay);
  const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(vv), k.bc2_sqrt), k.eps);
  pp = __fsub_rn(pp, __fmul_rn(k.step_size, __fdiv_rn(mm, denom)));
  p = pp;
  m = mm;
  v = vv;
}

__global__ void __launch_bounds__(kThreads)
    k_adamw_update(const __grid_constant__ Batch b, const Scalars k,
                   const double* __restrict__ partials, int nparts, float* __restrict__ norm_out,
                   int32_t* __restrict__ skipped_out) {
  __shared__ double sh[kThreads];
  __shared__ float s_f, s_step_size, s_bc2_sqrt;
  __shared__ int s_skip;
  {
    double acc = 0.0;
    for (int i = threadIdx.x; i < nparts; i += kThreads) acc = __dadd_rn(acc, partials[i]);
    const double G = block_sum_fixed(acc, sh);
    if (threadIdx.x == 0) {
      const float norm = static_cast<float>(__dmul_rn(__dsqrt_rn(G), k.inv_s_d));
      const int skip = !isfinite(norm);
      const float coef =
          (k.max_norm > 0.0f && norm > k.max_norm) ? __fdiv_rn(k.max_norm, norm) : 1.0f;
      s_f = __fmul_rn(coef, k.inv_s);
      s_skip = skip;
      if (k.d_step) {
        const int64_t step = *k.step_slot;
        const double t = static_cast<double>(step);
        s_step_size = static_cast<float>(__ddiv_rn(k.lr_d, 1.0 - pow(k.beta1_d, t)));
        s_bc2_sqrt = static_cast<float>(__dsqrt_rn(1.0 - pow(k.beta2_d, t)));
        if (b.first && blockIdx.x == 0 && !skip) *k.d_step = step;   // no CTA reads the counter
      } else {
        s_step_size = k.step_size;
        s_bc2_sqrt = k.bc2_sqrt;
      }
      if (b.first && blockIdx.x == 0) {
        if (norm_out) *norm_out = norm;
        if (skipped_out) *skipped_out = skip;
      }
    }
    __syncthreads();
  }
  if (s_skip) return;
  const float f = s_f;
  Scalars kk = k;
  kk.step_size = s_step_size;
  kk.bc2_sqrt = s_bc2_sqrt;
  const int64_t nchunks = b.chunk_start[b.n];
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const int t = find_tensor(b, c);
    const int64_t base = (c - b.chunk_start[t]) * kChunk;
    const int64_t n = b.numel[t];
    float* __restrict__ P = b.master[t];
    float* __restrict__ M = b.m[t];
    float* __restrict__ V = b.v[t];
    const uint16_t* __restrict__ G = b.g[t];
    uint16_t* __restrict__ W = b.w[t];
#pragma unroll 1
    for (int u0 = 0; u0 < 4; u0 += 2) {
      uint4 gv[2];
      float4 pv[2][2], mv[2][2], vv[2][2];
      bool full[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int64_t e = base + static_cast<int64_t>((u0 + u) * kThreads + threadIdx.x) * kVec;
        full[u] = e + kVec <= n;
        if (full[u]) {
          gv[u] = ld_stream_u4(G + e);
          mv[u][0] = __ldcs(reinterpret_cast<const float4*>(M + e));
          mv[u][1] = __ldcs(reinterpret_cast<const float4*>(M + e + 4));
          vv[u][0] = __ldcs(reinterpret_cast<const float4*>(V + e));
          vv[u][1] = __ldcs(reinterpret_cast<const float4*>(V + e + 4));
          pv[u][0] = __ldcs(reinterpret_cast<const float4*>(P + e));
          pv[u][1] = __ldcs(reinterpret_cast<const float4*>(P + e + 4));
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int64_t e = base + static_cast<int64_t>((u0 + u) * kThreads + threadIdx.x) * kVec;
        if (full[u]) {
          const uint32_t* gw = reinterpret_cast<const uint32_t*>(&gv[u]);
          float* pp = reinterpret_cast<float*>(&pv[u][0]);
          float* mm = reinterpret_cast<float*>(&mv[u][0]);
          float* vq = reinterpret_cast<float*>(&vv[u][0]);
          uint32_t wout[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            adam_one(pp[2 * j], mm[2 * j], vq[2 * j], bf16_to_f32(gw[j] & 0xFFFFu), kk, f);
            adam_one(pp[2 * j + 1], mm[2 * j + 1], vq[2 * j + 1], bf16_to_f32(gw[j] >> 16), kk, f);
            wout[j] = f32_to_bf16_rne(pp[2 * j]) | (f32_to_bf16_rne(pp[2 * j + 1]) << 16);
          }
          __stcs(reinterpret_cast<float4*>(M + e), mv[u][0]);
          __stcs(reinterpret_cast<float4*>(M + e + 4), mv[u][1]);
          __stcs(reinterpret_cast<float4*>(V + e), vv[u][0]);
          __stcs(reinterpret_cast<float4*>(V + e + 4), vv[u][1]);
          __stcs(reinterpret_cast<float4*>(P + e), pv[u][0]);
          __stcs(reinterpret_cast<float4*>(P + e + 4), pv[u][1]);
          *reinterpret_cast<uint4*>(W + e) = make_uint4(wout[0], wout[1], wout[2], wout[3]);
        } else {
          for (int64_t i = e; i < n && i < e + kVec; ++i) {
            float p = P[i], mq = M[i], vq1 = V[i];
            adam_one(p, mq, vq1, bf16_to_f32(G[i]), kk, f);
            P[i] = p;
            M[i] = mq;
            V[i] = vq1;
            W[i] = static_cast<uint16_t>(f32_to_bf16_rne(p));
          }
        }
      }
    }
  }
}

}  // namespace adamw
}  // namespace fp8t
