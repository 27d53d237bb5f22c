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
// When the sum of squares was formed elsewhere (the wgrad GEMM's epilogue), k_adamw_update runs
// alone on that one value; a device step counter is then read by every CTA at its start and
// advanced by the CTA of the last batch that finishes last (a ticket counter).
// A tensor may also carry the FP8 cast of its new BF16 weight for the next step (delayed
// scaling: that step's scale is already known): each 8-element vector of new BF16 weights is
// quantised where it is produced (f32 multiply by the scale, cvt.rn.satfinite, the cast kernel's
// codes) and stored row-major as 8 bytes; each warp keeps the amax of the weights it cast and
// max-accumulates it into the tensor's slot when it moves on. The GEMMs read these codes
// MN-major where they need the transpose, so none is written.
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
constexpr int kMaxCasts = 32;                            // weight casts per launch

struct CastInfo {
  const float* scale;
  unsigned int* amax_bits;
  float* scale_inv;                                       // may be null
  uint8_t* q;                                             // row-major codes, may be null
  int32_t fmt;
};

struct Batch {
  int32_t n;
  int32_t first;                                          // 1 for the batch that reports
  int32_t last;                                           // 1 for the last batch of the call
  int64_t chunk_start[kMaxTensors + 1];                   // prefix sums of chunks per tensor
  int64_t numel[kMaxTensors];
  float* master[kMaxTensors];
  float* m[kMaxTensors];
  float* v[kMaxTensors];
  const uint16_t* g[kMaxTensors];
  uint16_t* w[kMaxTensors];
  int8_t cast_of[kMaxTensors];                            // index into cast, or -1
  CastInfo cast[kMaxCasts];
};

struct Scalars {            // host-computed, rounded once to f32 (double where noted)
  float beta1, beta2, omb1, omb2, decay, step_size, bc2_sqrt, eps, inv_s, max_norm;
  double inv_s_d;
  // device step counter (may be null): the step is read from step_slot (counter + 1, written by
  // the norm pass), step_size and bc2_sqrt are formed on the device, and the counter is advanced
  // by the first CTA of the first update launch unless the step is skipped
  int64_t* d_step;
  const int64_t* step_slot;      // null: read the counter itself and advance it by ticket
  unsigned int* step_ticket;
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

// 8 BF16 weights (4 words) -> 8 FP8 codes; `mag` receives their largest magnitude bit pattern.
// NaN products (a NaN weight or a non-finite scale) give the byte 0x7F, as in the cast kernel.
template <int FMT>
__device__ __forceinline__ uint2 quant8(const uint32_t (&w)[4], float s, uint32_t& mag) {
  uint32_t out[2] = {0u, 0u}, m2 = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    m2 = __vmaxu2(m2, w[j] & 0x7FFF7FFFu);
    const float p0 = __fmul_rn(__uint_as_float(w[j] << 16), s);
    const float p1 = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), s);
    out[j >> 1] |= cvt_fp8x2<FMT>(p0, p1) << (16 * (j & 1));
  }
  mag = max(m2 & 0xFFFFu, m2 >> 16);
  if (mag > 0x7F80u || !isfinite(s)) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p0 = __fmul_rn(__uint_as_float(w[j] << 16), s);
      const float p1 = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), s);
      const int sh = 16 * (j & 1);
      if (p0 != p0) out[j >> 1] = (out[j >> 1] & ~(0xFFu << sh)) | (0x7Fu << sh);
      if (p1 != p1) out[j >> 1] = (out[j >> 1] & ~(0xFF00u << sh)) | (0x7F00u << sh);
    }
  }
  return make_uint2(out[0], out[1]);
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

// amax of the new weights a warp cast, max-accumulated into the tensor's slot (all lanes).
__device__ __forceinline__ void flush_amax(unsigned int* amax_bits, uint32_t vmax) {
  uint32_t m = __reduce_max_sync(0xffffffffu, vmax);
  if ((threadIdx.x & 31) == 0) {
    if (m > 0x7F80u) m = 0x7FC0u;                  // canonical NaN
    atomicMax(amax_bits, m << 16);
  }
}

template <bool CAST>
__global__ void __launch_bounds__(kThreads, 2)
    k_adamw_update(const __grid_constant__ Batch b, const Scalars k,
                   const double* __restrict__ partials, int nparts, float* __restrict__ norm_out,
                   int32_t* __restrict__ skipped_out) {
  __shared__ double sh[kThreads];
  __shared__ float s_f, s_step_size, s_bc2_sqrt;
  __shared__ int s_skip;
  __shared__ int64_t s_step;
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
        const int64_t step = k.step_slot ? *k.step_slot
                                         : *reinterpret_cast<volatile int64_t*>(k.d_step) + 1;
        s_step = step;
        const double t = static_cast<double>(step);
        s_step_size = static_cast<float>(__ddiv_rn(k.lr_d, 1.0 - pow(k.beta1_d, t)));
        s_bc2_sqrt = static_cast<float>(__dsqrt_rn(1.0 - pow(k.beta2_d, t)));
        if (k.step_slot && b.first && blockIdx.x == 0 && !skip)
          *k.d_step = step;                                   // no CTA reads the counter
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
  if (s_skip && !CAST) return;          // a skipped step only re-casts weights that carry a cast
  const bool skip = s_skip != 0;
  const float f = s_f;
  Scalars kk = k;
  kk.step_size = s_step_size;
  kk.bc2_sqrt = s_bc2_sqrt;
  int cur = -1;                          // cast this CTA's warps are accumulating an amax for
  uint32_t vmax = 0;
  const int64_t nchunks = b.chunk_start[b.n];
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const int t = find_tensor(b, c);
    const int cj = CAST ? b.cast_of[t] : -1;
    if (CAST && cj != cur) {
      if (cur >= 0) flush_amax(b.cast[cur].amax_bits, vmax);
      cur = cj;
      vmax = 0;
    }
    if (CAST && skip && cj < 0) continue;
    const float s = CAST && cj >= 0 ? __ldg(b.cast[cj].scale) : 0.0f;
    if (CAST && cj >= 0 && c == b.chunk_start[t] && threadIdx.x == 0 && b.cast[cj].scale_inv)
      *b.cast[cj].scale_inv = __fdiv_rn(1.0f, s);
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
        if (CAST && skip) {                  // skipped step: the unchanged weight, cast again
          if (full[u]) gv[u] = *reinterpret_cast<const uint4*>(W + e);
        } else if (full[u]) {
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
        if (CAST && skip) {
          if (full[u]) {
            const uint32_t wout[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
            uint32_t mag;
            const uint2 q8 = b.cast[cj].fmt == 0 ? quant8<0>(wout, s, mag) : quant8<1>(wout, s, mag);
            vmax = max(vmax, mag);
            if (b.cast[cj].q) *reinterpret_cast<uint2*>(b.cast[cj].q + e) = q8;
          }
        } else if (full[u]) {
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
          if (CAST && cj >= 0) {
            uint32_t mag;
            const uint2 q8 = b.cast[cj].fmt == 0 ? quant8<0>(wout, s, mag) : quant8<1>(wout, s, mag);
            vmax = max(vmax, mag);
            if (b.cast[cj].q) *reinterpret_cast<uint2*>(b.cast[cj].q + e) = q8;
          }
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
  if (CAST && cur >= 0) flush_amax(b.cast[cur].amax_bits, vmax);
  // counter read by every CTA above: the last CTA of the last batch advances it
  if (k.d_step && !k.step_slot && b.last && !skip) {
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      s_last = atomicAdd(k.step_ticket, 1u) == gridDim.x - 1;
      if (s_last) {
        *k.d_step = s_step;
        atomicExch(k.step_ticket, 0u);
      }
    }
  }
}

}  // namespace adamw
}  // namespace fp8t
