// gemm_tcgen05.cuh — per-tensor scaled FP8 GEMM on the 5th-generation tensor cores.
//
// Method: the FP8 GEMM of "FP8 混合精度训练工程实践" §三 (FP8 inputs, FP32 accumulation,
// 16-bit output) with per-tensor dequantisation (§四 dequantize; §五 per-tensor mode:
// FP8 x FP8, FP32 accumulate, BF16 out). The pages' kernel design is Hopper WGMMA (m64nNk32
// warpgroup MMA reading shared memory); on sm_100a the same contraction runs as
// tcgen05.mma.kind::f8f6f4 issued by one thread, with the accumulator in tensor memory.
//
// D[M x N] = bf16((A[M x K] . B[N x K]^T) * sa * sb), A and B K-major ("TN").
// One CTA of 128 threads computes a 128 x 256 tile:
//   warp 0, lane 0  TMA producer: 128-byte-swizzled 128 x 128 (A) and 256 x 128 (B) byte tiles
//                   into a 4-stage ring (48 KB per stage), one mbarrier per stage;
//   warp 1, lane 0  MMA issuer: 4 x tcgen05.mma (M=128, N=256, K=32) per stage into a
//                   128 x 256 f32 accumulator in TMEM (256 columns), tcgen05.commit frees the
//                   stage; a final commit signals the epilogue;
//   warps 0-3       epilogue: tcgen05.ld 32 lanes x 32 columns per warp-chunk, scale by sa*sb,
//                   round to BF16, 16-byte stores (rows >= M and columns >= N masked).
// Every mbarrier wait is bounded (globaltimer). On expiry the CTA records kErrTimeout, stops
// issuing, waits (with a separate fixed bound) for the TMA loads and MMAs it already issued,
// frees its TMEM and returns without writing D.
#pragma once

#include "ptx.cuh"

namespace fp8t {
namespace gemm {

constexpr int kBM = 128, kBN = 256, kBK = 128, kStages = 4, kUmmaK = 32;
constexpr int kThreads = 128;
constexpr int kABytes = kBM * kBK, kBBytes = kBN * kBK, kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 256;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*alignment slack*/ + 256 /*barriers*/;

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t make_sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);        // start address
  d |= static_cast<uint64_t>(1) << 16;                       // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
  return d;
}

// Instruction descriptor: FP32 accumulator, FP8 A/B formats (0 = E4M3, 1 = E5M2), both K-major.
__host__ __device__ constexpr uint32_t make_idesc(int a_fmt, int b_fmt) {
  return (1u << 4) | (static_cast<uint32_t>(a_fmt) << 7) | (static_cast<uint32_t>(b_fmt) << 10) |
         (static_cast<uint32_t>(kBN >> 3) << 17) | (static_cast<uint32_t>(kBM >> 4) << 24);
}

// Two f32 -> two BF16 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_fp8_gemm(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
               uint16_t* __restrict__ D, int M, int N, int K, const float* __restrict__ d_sa,
               const float* __restrict__ d_sb, uint32_t idesc, int n_tiles_n) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accum = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x / n_tiles_n, nt = blockIdx.x % n_tiles_n;
  const int m0 = mt * kBM, n0 = nt * kBN;
  const int num_kb = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(accum), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tma_a);
    tma_prefetch_desc(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t limit = wait_limit_ns();

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int issued = 0;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (kb / kStages) & 1;
      if (*abort_flag) break;
      if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, limit)) {
        *abort_flag = 1;
        record_error(kErrTimeout);
        break;
      }
      mbar_arrive_expect_tx(smem_u32(&full[s]), kStageBytes);
      tma_load_2d(smem_u32(sA + s * kABytes), &tma_a, kb * kBK, m0, smem_u32(&full[s]));
      tma_load_2d(smem_u32(sB + s * kBBytes), &tma_b, kb * kBK, n0, smem_u32(&full[s]));
      ++issued;
    }
    // every issued load must land before the CTA may exit (only the last kStages can be open)
    for (int kb = issued > kStages ? issued - kStages : 0; kb < issued; ++kb)
      mbar_wait(smem_u32(&full[kb % kStages]), (kb / kStages) & 1, kDrainLimitNs);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (kb / kStages) & 1;
      if (*abort_flag) break;
      if (!mbar_wait(smem_u32(&full[s]), ph, limit)) {
        *abort_flag = 1;
        record_error(kErrTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t a_base = smem_u32(sA + s * kABytes);
      const uint32_t b_base = smem_u32(sB + s * kBBytes);
#pragma unroll
      for (int k = 0; k < kBK / kUmmaK; ++k)
        tc_mma_f8(tmem, make_sw128_desc(a_base + k * kUmmaK), make_sw128_desc(b_base + k * kUmmaK),
                  idesc, (kb | k) != 0 ? 1u : 0u);
      tc_commit(smem_u32(&empty[s]));
    }
    tc_commit(smem_u32(accum));  // arrives when every MMA issued above has completed
  }
  __syncwarp();

  // ---------------- epilogue (all four warps)
  if (!mbar_wait(smem_u32(accum), 0, limit)) {
    record_error(kErrTimeout);
    *abort_flag = 1;
    mbar_wait(smem_u32(accum), 0, kDrainLimitNs);  // MMAs must finish before TMEM is freed
  }
  tc_fence_after();
  __syncthreads();
  const bool aborted = *abort_flag != 0;

  const float alpha = __fmul_rn(__ldg(d_sa), __ldg(d_sb));
  const int row = m0 + warp * 32 + lane;
#pragma unroll 1
  for (int c = 0; c < kBN / 32; ++c) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c * 32, r);
    tmem_ld_wait();
    const int col = n0 + c * 32;
    if (!aborted && row < M && col < N) {
      uint32_t packed[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        packed[j] = pack_bf16x2(__fmul_rn(__uint_as_float(r[2 * j]), alpha),
                                __fmul_rn(__uint_as_float(r[2 * j + 1]), alpha));
      uint16_t* dst = D + static_cast<int64_t>(row) * N + col;
#pragma unroll
      for (int qd = 0; qd < 4; ++qd)
        if (col + 8 * qd < N)
          *reinterpret_cast<uint4*>(dst + 8 * qd) =
              make_uint4(packed[4 * qd], packed[4 * qd + 1], packed[4 * qd + 2], packed[4 * qd + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace gemm
}  // namespace fp8t
