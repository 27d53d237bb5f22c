// gemm_mx_wide.cuh — the block-scaled (MXFP8) grouped GEMM on 256 x 384 tiles.
//
// Why a second MXFP8 kernel: on 256 x 256 tiles each SM must take in 32 KB of operands per
// 128-deep k-block, close to the rate its TMA loads reach, and the scale atoms on top of that
// leave the tensor pipe waiting for data. A wider tile reuses each A box for more columns. The
// per-tensor kernel's 256 x 512 tile does not fit here: its accumulator takes all 512 TMEM
// columns and the scales need 16 more. So a tile is 384 columns wide, as two MMAs per k-step
// whose B rows start on 128-row scale-atom boundaries:
//   MMA 0: N = 256, tile columns 0..255, each CTA holding 128 of the B rows (as in the 256 x 256
//          kernel), accumulator columns 0..255;
//   MMA 1: N = 128, tile columns 256..383, each CTA holding 64 B rows, accumulator 256..383.
// TMEM per CTA: accumulator 0..383, A scales 384..387, the scales of MMA 0's 256 B rows 388..395,
// of MMA 1's 128 rows 396..399. Per stage each CTA loads the A box (128 rows), a 128-row and a
// 64-row B box (MN-major: the 64-column box uses the 64-byte swizzle) and four 512-byte scale
// atoms: 42 KB, four stages; the MMA thread copies the atoms to TMEM (tcgen05.cp 32x128b,
// replicated to the four lane quarters) before the k-block's MMAs, which select each 32-deep
// sub-block's scale byte through the descriptor. A column tile that starts within 256 of N's end
// runs MMA 0 only (N is a multiple of 128, so such a tile has no rows for MMA 1).
// As in the per-tensor 256 x 512 kernel there is one accumulator: eight epilogue warps (a TMEM
// lane quarter and a 192-column half each) read it into registers as packed BF16, release it,
// then store. Summed problems (the wgrad outputs of a step) also leave f32(bf16(D))^2 per warp and
// tile in a partial slot, added up in index order by the last CTA, as in the per-tensor kernels.
// Waits are bounded as in the other kernels.
#pragma once

#include "gemm_tcgen05.cuh"

namespace fp8t {
namespace gemm {

constexpr int kBNx = 384;
constexpr int kStagesX = 4;
constexpr int kB0BytesX = kHalf * kBK;                     // 128 B rows x 128 bytes
constexpr int kB1BytesX = (kHalf / 2) * kBK;               // 64 B rows x 128 bytes
constexpr int kSfBytesX = 4 * 512;                         // A atom, three B atoms
constexpr int kStageBytesX = kABytes + kB0BytesX + kB1BytesX + kSfBytesX;
constexpr int kAccColsX = kBNx / 2;                        // columns per epilogue half
constexpr uint32_t kSfaColX = 384, kSfb0ColX = 388, kSfb1ColX = 396;
constexpr int kEpiWarpsX = 8;
constexpr int kThreadsX = 64 + 32 * kEpiWarpsX;
constexpr int kEpiBytesX = kEpiWarpsX * 2 * kEpiChunkBytes;
constexpr int kSmemBytesX = kStagesX * kStageBytesX + kEpiBytesX + 1024 + 256;
static_assert(kStageBytesX % 1024 == 0, "stages stay 1024-byte aligned");
static_assert(kSfb1ColX + 4 <= static_cast<uint32_t>(kTmemCols), "TMEM columns");

// Shared-memory descriptor, MN-major operand, 64-byte swizzle: 64 MN-elements per swizzle row,
// 8 K-rows (512 B) per swizzle atom; a CTA's 64 rows of B are one atom wide.
__device__ __forceinline__ uint64_t make_sw64_desc_mn(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);        // start address
  d |= static_cast<uint64_t>(8192 >> 4) << 16;               // leading byte offset (unused)
  d |= static_cast<uint64_t>(512 >> 4) << 32;                // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
  d |= static_cast<uint64_t>(4) << 61;                       // 64-byte swizzle
  return d;
}

// Block-scaled instruction descriptor with N given (M = 256, pair).
__device__ __forceinline__ uint32_t make_idesc_mx_n(int a_fmt, int b_fmt, int a_mn, int b_mn,
                                                    int sf_id, int n) {
  return (static_cast<uint32_t>(sf_id) << 4) | (static_cast<uint32_t>(a_fmt) << 7) |
         (static_cast<uint32_t>(b_fmt) << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(kBM >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

struct SmemX {
  uint64_t full[kStagesX];
  uint64_t empty[kStagesX];
  uint64_t acc_full;          // both CTAs: the accumulator holds a finished tile
  uint64_t acc_empty;         // even CTA: every epilogue warp of both CTAs has read it
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// Tile geometry shared by the roles: first B row of the tile and whether MMA 1 has rows.
__device__ __forceinline__ void mxw_tile(const Problem& P, int local, int& mt, int& nt, bool& has1) {
  mt = local / P.tiles_n;
  nt = local % P.tiles_n;
  has1 = nt * kBNx + 256 < P.N;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsX, 1)
    k_fp8_gemm_mx_wide(const __grid_constant__ Group g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  // stage s: [A 128 x 128 B][B0 128 x 128 B][B1 64 x 128 B][scale atoms 4 x 512 B]
  uint8_t* sStage = smem;
  uint8_t* sEpi = smem + kStagesX * kStageBytesX;
  SmemX* S = reinterpret_cast<SmemX*>(sEpi + kEpiBytesX);
  volatile int* abort_flag = &S->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int my_tiles = tiles_of(g, cluster, n_clusters);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesX; ++s) {
      mbar_init(smem_u32(&S->full[s]), 1);
      mbar_init(smem_u32(&S->empty[s]), 1);
    }
    mbar_init(smem_u32(&S->acc_full), 1);
    mbar_init(smem_u32(&S->acc_empty), 2 * kEpiWarpsX);
    mbar_init(smem_u32(&S->mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int p = 0; p < g.n && p < 8; ++p) {
      tma_prefetch_desc(&g.p[p].a);
      tma_prefetch_desc(&g.p[p].b);
      tma_prefetch_desc(&g.p[p].b64);
      tma_prefetch_desc(&g.p[p].d);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&S->tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;
  const uint64_t limit = wait_limit_ns();
  const int expire = expire_mode();
  const bool expire_main = expire == kExpireAll;
  const bool expire_epi = expire == kExpireAll || expire == kExpireGemmEpilogue;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      uint32_t it = 0, issued = 0;
      for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
        const int tile = tile_at(g, cluster, n_clusters, i);
        const Problem& P = g.p[find_problem(g, tile)];
        int mt, nt;
        bool has1;
        mxw_tile(P, tile - P.tile_start, mt, nt, has1);
        const int m0 = mt * kBM + static_cast<int>(rank) * kHalf;
        const int nb0 = nt * kBNx + static_cast<int>(rank) * kHalf;           // MMA 0 rows
        const int nb1 = nt * kBNx + 256 + static_cast<int>(rank) * (kHalf / 2); // MMA 1 rows
        const int ra = 2 * mt + static_cast<int>(rank), rb = 3 * nt;          // atom rows
        const int num_kb = (P.K + kBK - 1) / kBK;
        const uint32_t tx = 2u * (kABytes + kB0BytesX + 3 * 512 + (has1 ? kB1BytesX + 512 : 0));
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % kStagesX, ph = (it / kStagesX) & 1;
          if (*abort_flag) break;
          if (!mbar_wait(smem_u32(&S->empty[s]), ph ^ 1, limit, expire_main)) {
            *abort_flag = 1;
            record_error(kErrTimeout);
            break;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&S->full[s]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&S->full[s]), tx);
          const uint32_t base = smem_u32(sStage + s * kStageBytesX);
          const uint32_t a_dst = base, b0_dst = base + kABytes, b1_dst = b0_dst + kB0BytesX;
          const uint32_t sf_dst = b1_dst + kB1BytesX;
          if (P.a_mn) tma_load_2d_pair(a_dst, &P.a, m0, kb * kBK, full_leader);
          else        tma_load_2d_pair(a_dst, &P.a, kb * kBK, m0, full_leader);
          if (P.b_mn) tma_load_2d_pair(b0_dst, &P.b, nb0, kb * kBK, full_leader);
          else        tma_load_2d_pair(b0_dst, &P.b, kb * kBK, nb0, full_leader);
          tma_load_2d_pair(sf_dst, &P.sfa, 0, ra * P.kb128 + kb, full_leader);
          tma_load_2d_pair(sf_dst + 512, &P.sfb, 0, rb * P.kb128 + kb, full_leader);
          tma_load_2d_pair(sf_dst + 1024, &P.sfb, 0, (rb + 1) * P.kb128 + kb, full_leader);
          if (has1) {
            if (P.b_mn) tma_load_2d_pair(b1_dst, &P.b64, nb1, kb * kBK, full_leader);
            else        tma_load_2d_pair(b1_dst, &P.b64, kb * kBK, nb1, full_leader);
            tma_load_2d_pair(sf_dst + 1536, &P.sfb, 0, (rb + 2) * P.kb128 + kb, full_leader);
          }
          ++issued;
        }
      }
      if (leader) {
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t i = issued > kStagesX ? issued - kStagesX : 0; i < issued; ++i) {
          const uint64_t spent = globaltimer_ns() - t0;
          if (spent >= kPairDrainNs) break;
          mbar_wait(smem_u32(&S->full[i % kStagesX]), (i / kStagesX) & 1, kPairDrainNs - spent);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA): per k-step an N = 256 and an N = 128 MMA
      uint32_t it = 0, local = 0;
      for (int i = 0; i < my_tiles && !*abort_flag; ++i, ++local) {
        const int tile = tile_at(g, cluster, n_clusters, i);
        const Problem& P = g.p[find_problem(g, tile)];
        int mt, nt;
        bool has1;
        mxw_tile(P, tile - P.tile_start, mt, nt, has1);
        const int num_kb = (P.K + kBK - 1) / kBK;
        const bool a_mn = P.a_mn != 0, b_mn = P.b_mn != 0;
        if (!mbar_wait(smem_u32(&S->acc_empty), (local & 1) ^ 1, limit, expire_main)) {
          *abort_flag = 1;
          record_error(kErrTimeout);
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % kStagesX, ph = (it / kStagesX) & 1;
          if (*abort_flag || !mbar_wait(smem_u32(&S->full[s]), ph, limit, expire_main)) {
            if (!*abort_flag) record_error(kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(sStage + s * kStageBytesX);
          const uint32_t a_base = base, b0_base = base + kABytes, b1_base = b0_base + kB0BytesX;
          const uint32_t sf = b1_base + kB1BytesX;
          tc_cp_32x128b_warpx4_pair(tmem + kSfaColX, make_sf_desc(sf));
          tc_cp_32x128b_warpx4_pair(tmem + kSfb0ColX, make_sf_desc(sf + 512));
          tc_cp_32x128b_warpx4_pair(tmem + kSfb0ColX + 4, make_sf_desc(sf + 1024));
          if (has1) tc_cp_32x128b_warpx4_pair(tmem + kSfb1ColX, make_sf_desc(sf + 1536));
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            const uint64_t adesc = a_mn ? make_sw128_desc_mn(a_base + k * kUmmaK * 128)
                                        : make_sw128_desc(a_base + k * kUmmaK);
            const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
            const uint32_t sfa = (tmem + kSfaColX) | (static_cast<uint32_t>(k) << 30);
            tc_mma_mxf8_pair(tmem, adesc,
                             b_mn ? make_sw128_desc_mn(b0_base + k * kUmmaK * 128)
                                  : make_sw128_desc(b0_base + k * kUmmaK),
                             make_idesc_mx_n(P.a_fmt, P.b_fmt, P.a_mn, P.b_mn, k, 256), sfa,
                             (tmem + kSfb0ColX) | (static_cast<uint32_t>(k) << 30), acc);
            if (has1)
              tc_mma_mxf8_pair(tmem + 256, adesc,
                               b_mn ? make_sw64_desc_mn(b1_base + k * kUmmaK * 64)
                                    : make_sw128_desc(b1_base + k * kUmmaK),
                               make_idesc_mx_n(P.a_fmt, P.b_fmt, P.a_mn, P.b_mn, k, 128), sfa,
                               (tmem + kSfb1ColX) | (static_cast<uint32_t>(k) << 30), acc);
          }
          tc_commit_pair_mc(smem_u32(&S->empty[s]), 0x3);
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&S->acc_full), 0x3);
      }
      tc_commit_pair(smem_u32(&S->mma_done));
      mbar_wait(smem_u32(&S->mma_done), 0, kDrainLimitNs);
    }
  } else {
    // ---------------- epilogue warps 2..9 (both CTAs): TMEM lane quarter warp % 4, column half
    const int quad = warp & 3, half = (warp - 2) >> 2;
    uint8_t* my_buf = sEpi + (warp - 2) * 2 * kEpiChunkBytes;
    uint32_t local = 0, chunk_count = 0;
    for (int i = 0; i < my_tiles; ++i, ++local) {
      const int tile = tile_at(g, cluster, n_clusters, i);
      if (*abort_flag) break;
      if (!mbar_wait(smem_u32(&S->acc_full), local & 1, limit, expire_epi)) {
        *abort_flag = 1;
        record_error(kErrTimeout);
        break;
      }
      tc_fence_after();
      const Problem& P = g.p[find_problem(g, tile)];
      const int M = P.M, N = P.N, local_tile = tile - P.tile_start;
      const int row0 = (local_tile / P.tiles_n) * kBM + static_cast<int>(rank) * kHalf + quad * 32;
      const int n0 = (local_tile % P.tiles_n) * kBNx + half * kAccColsX;
      const uint32_t t_base = tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * kAccColsX;
      uint32_t w[kAccColsX / 32][16];
#pragma unroll
      for (int c = 0; c < kAccColsX / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_base + c * 32, r);
        tmem_ld_wait();
        tmem_reg_fence(r);
#pragma unroll
        for (int j = 0; j < 16; ++j) w[c][j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&S->acc_empty), 0));
      const bool sumsq = P.sumsq_slot >= 0;
      double ss = 0.0;
#pragma unroll
      for (int c = 0; c < kAccColsX / 32; ++c) {
        if (n0 + c * 32 >= N || row0 >= M) continue;       // chunk entirely outside the matrix
        uint8_t* buf = my_buf + (chunk_count & 1) * kEpiChunkBytes;
        ++chunk_count;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          if (sumsq) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t v = w[c][4 * p + q];
              const double lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
              ss = __fma_rn(lo, lo, ss);
              ss = __fma_rn(hi, hi, ss);
            }
          }
          const int pp = p ^ ((lane >> 1) & 3);
          *reinterpret_cast<uint4*>(buf + lane * 64 + pp * 16) =
              make_uint4(w[c][4 * p], w[c][4 * p + 1], w[c][4 * p + 2], w[c][4 * p + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&P.d, smem_u32(buf), n0 + c * 32, row0);
          bulk_commit_group();
        }
      }
      if (sumsq) {                       // this warp's rows of the tile: one partial slot
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        if (lane == 0) {
          g.partials[P.sumsq_slot + local_tile * kSumsqPerTileW + static_cast<int>(rank) * kEpiWarpsX +
                     half * 4 + quad] = ss;
          __threadfence();
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();
  }
  __syncwarp();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < kSettleNs) {
    }
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);

  // ---------------- sum of squares: the last CTA of the last launch adds the slots in order
  if (!g.sumsq_out) return;
  if (threadIdx.x == 0 && *abort_flag) atomicOr(g.abort_word, 1u);
  if (!g.last_launch) return;
  __shared__ int s_last;
  double* s_part = reinterpret_cast<double*>(sStage);   // the stage buffers are idle by now
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(g.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = threadIdx.x; i < g.n_partials; i += kThreadsX) acc = __dadd_rn(acc, __ldcg(g.partials + i));
  s_part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double total = 0.0;
    for (int i = 0; i < kThreadsX; ++i) total = __dadd_rn(total, s_part[i]);
    if (*reinterpret_cast<volatile unsigned int*>(g.abort_word) != 0u)
      total = __longlong_as_double(0x7FF8000000000000LL);
    *g.sumsq_out = total;
    atomicExch(g.abort_word, 0u);
    atomicExch(g.ticket, 0u);
  }
}

}  // namespace gemm
}  // namespace fp8t
