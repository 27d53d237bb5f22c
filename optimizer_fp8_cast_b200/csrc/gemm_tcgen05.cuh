// gemm_tcgen05.cuh — per-tensor scaled FP8 GEMM on the 5th-generation tensor cores.
//
// Method: the FP8 GEMM of "FP8 混合精度训练工程实践" §三 (FP8 inputs, FP32 accumulation,
// 16-bit output) with per-tensor dequantisation (§四 dequantize; §五 per-tensor mode:
// FP8 x FP8, FP32 accumulate, BF16 out). The pages' kernel design is Hopper WGMMA (m64nNk32
// warpgroup MMA reading shared memory, one SM per tile); on sm_100a the same contraction runs
// as tcgen05.mma.kind::f8f6f4 issued by one thread for a PAIR of SMs, with the accumulator in
// tensor memory.
//
// D[M x N] = bf16((A[M x K] . B[N x K]^T) * sa * sb). Each operand is either K-major (stored
// [M or N rows][K], "TN") or MN-major (stored [K rows][M or N]): tcgen05 reads 8-bit operands in
// both orders, so the transposed FP8 copies that a K-major-only tensor core needs (the pages'
// Hopper design) are optional here. An MN-major operand is loaded as 128 K-rows x 128 bytes
// boxes with the same 128-byte swizzle; its descriptor steps 32 K-rows (4 KB) per MMA.
// A cluster of two CTAs (one per SM) computes a 256 x 256 tile: CTA r loads A rows
// [128r, 128r+128) and B rows (N columns) [128r, 128r+128) of the tile, 128-byte swizzled
// 128 x 128-byte boxes, into its own 6-stage ring (32 KB per stage). Both CTAs' loads count on
// the even CTA's "full" barrier; the even CTA's MMA thread issues tcgen05.mma.cta_group::2
// (M=256, N=256, K=32), which reads A and B halves from both CTAs' shared memory, and releases
// each stage in both CTAs with one multicast tcgen05.commit. Per SM that is 32 KB of operands per
// 512 tensor-core cycles, two thirds of what a single-SM 128 x 256 tile needs.
// Persistent: cluster c walks the tiles c, c + clusters, ... or, for launches of up to
// kMaxSchedTiles tiles, the list the host built for it: tiles cost K / 128 k-blocks each, and a
// longest-first greedy assignment balances the clusters (a grouped step mixes K = T wgrad tiles
// with K = features fprop/dgrad tiles, which round-robin leaves several percent apart). Two TMEM
// accumulators (2 x 256 columns) let the epilogue of one tile overlap the main loop of the next.
// Launches whose every problem has N >= 512 use the wide form (k_fp8_gemm_wide, below): 256 x 512
// tiles, a quarter fewer operand bytes per FLOP; its host schedule may run a tile as its two
// 256-column halves on different clusters to even out the clusters' loads.
// Warp roles (192 threads per CTA):
//   warp 0, lane 0  TMA producer (both CTAs)
//   warp 1, lane 0  MMA issuer (even CTA only); warp 1 also owns the TMEM allocation
//   warps 2-5       epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 of its own CTA (rows of
//                   its half), 32 columns at a time, scales by sa*sb, rounds to BF16 and writes
//                   the 32 x 32 chunk into a 64-byte-swizzled shared-memory buffer (double
//                   buffered per warp), which one lane stores with a TMA bulk tensor store
//                   (clipped at the M and N edges). Per-lane 16-byte stores to 32 different rows
//                   cost ~15% of the GEMM's throughput. Once its TMEM reads are done the warp
//                   tells the even CTA that the accumulator is free (4 warps x 2 CTAs arrive).
// Optional sum of squares (the AdamW global norm's input, fused here so that the gradient is not
// read again): for flagged problems each epilogue warp adds up f32(bf16(D))^2 of its rows of the
// tile in FP64 (a fixed butterfly over the lanes) and stores one partial per (tile, CTA, warp)
// into a workspace slot; the CTA that finishes the last launch last (a ticket counter) sums all
// slots in index order, so the result does not depend on scheduling. Out-of-range rows and
// columns hold exact zeros (TMA zero-fills the operands there) and add nothing.
// MXFP8 variant (template MX): block-scaled MMAs (tcgen05.mma.kind::mxf8f6f4.block_scale) with
// one E8M0 scale per 32 K values of every row of A and B. Per stage each CTA also loads, by TMA,
// the 512-byte scale atom of its 128 A rows and the two atoms of the tile's 256 B rows (the 4
// K-blocks of the stage); the MMA thread copies them into tensor memory (tcgen05.cp 32x128b,
// replicated into the four lane quarters: A scales in 4 columns, B scales in 8) right before
// the stage's four MMAs, which pick the byte of their K-block through the descriptor's
// scale-factor ids. The copies and MMAs run in issue order, so one set of scale columns serves
// every stage. Two full accumulators and the 12 scale columns do not fit the 512 TMEM columns,
// so the MX kernel overlaps its accumulators by one 32-column chunk: accumulator 0 at columns
// 0..255, accumulator 1 at 224..479, scales at 480..491. The epilogue reads the shared chunk
// first (accumulator 0 backwards from its last chunk, accumulator 1 forwards) and releases it
// through its own barrier, so the next tile's MMAs, which overwrite that chunk, can start while
// the rest of the accumulator is being stored.
// Every mbarrier wait is bounded (globaltimer). On expiry a CTA records kErrTimeout and stops
// issuing; issued MMAs are awaited with a fixed bound, loads in flight are given time to land,
// and both CTAs meet at a cluster barrier before TMEM is freed; D is then incomplete.
#pragma once

#include "ptx.cuh"

namespace fp8t {
namespace gemm {

constexpr int kBM = 256, kBN = 256, kBK = 128, kStages = 6, kUmmaK = 32;
constexpr int kHalf = 128;                               // rows of A and of B per CTA
constexpr int kThreads = 192;
constexpr int kABytes = kHalf * kBK, kBBytes = kHalf * kBK, kStageBytes = kABytes + kBBytes;
constexpr uint32_t kPairTxBytes = 2 * kStageBytes;       // both CTAs' boxes of one stage
constexpr int kAccCols = 256, kTmemCols = 2 * kAccCols;
constexpr int kEpiWarps = 4;
constexpr int kEpiChunkBytes = 32 * 32 * 2;              // 32 rows x 32 BF16 columns
constexpr int kEpiBytes = kEpiWarps * 2 * kEpiChunkBytes; // double-buffered per epilogue warp
constexpr int kSmemBytes =
    kStages * kStageBytes + kEpiBytes + 1024 /*alignment slack*/ + 256 /*barriers*/;
constexpr int kSfaBytes = 512, kSfbBytes = 1024;         // MX scale atoms per stage and CTA
constexpr int kSfStageBytes = kSfaBytes + kSfbBytes;
constexpr int kSmemBytesMX = kSmemBytes + kStages * kSfStageBytes;
constexpr uint32_t kMxAcc1Col = kAccCols - 32;           // MX: second accumulator, overlapping
constexpr uint32_t kSfaCol = kMxAcc1Col + kAccCols, kSfbCol = kSfaCol + 4;   // MX: scale columns
constexpr uint64_t kSettleNs = 200000;                   // let loads in flight land on abort
constexpr uint64_t kPairDrainNs = 1000000;               // producer drain budget (1 ms)

// Shared-memory matrix descriptor, MN-major operand, 128-byte swizzle: 128 MN-elements per
// swizzle row, 8 K-rows (1024 B) per swizzle atom, atoms along K 1024 B apart (stride byte
// offset); the 128 rows (M or N) a CTA holds are a single atom wide, so the leading byte offset
// (distance between atoms along MN) is never stepped over.
__device__ __forceinline__ uint64_t make_sw128_desc_mn(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);        // start address
  d |= static_cast<uint64_t>(16384 >> 4) << 16;              // leading byte offset
  d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
  return d;
}

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

// Instruction descriptor: FP32 accumulator, FP8 A/B formats (0 = E4M3, 1 = E5M2), A and B
// major-ness (0 = K-major, 1 = MN-major), M = 256 (pair), N = 256.
__host__ __device__ constexpr uint32_t make_idesc(int a_fmt, int b_fmt, int a_mn = 0, int b_mn = 0) {
  return (1u << 4) | (static_cast<uint32_t>(a_fmt) << 7) | (static_cast<uint32_t>(b_fmt) << 10) |
         (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(kBN >> 3) << 17) | (static_cast<uint32_t>(kBM >> 4) << 24);
}

// Block-scaled instruction descriptor (MXFP8): A/B formats and major-ness as above, E8M0 scales
// (bit 23), scale-factor byte `sf_id` for A (bits 29-30) and B (bits 4-5), M = 256, N = 256.
__host__ __device__ constexpr uint32_t make_idesc_mx(int a_fmt, int b_fmt, int a_mn, int b_mn, int sf_id) {
  return (static_cast<uint32_t>(sf_id) << 4) | (static_cast<uint32_t>(a_fmt) << 7) |
         (static_cast<uint32_t>(b_fmt) << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(kBN >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(kBM >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

// Shared-memory descriptor of a 32-row x 16-byte scale atom (no swizzle, K-major): rows 16 B
// apart, 8-row groups 128 B apart.
__device__ __forceinline__ uint64_t make_sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);        // start address
  d |= static_cast<uint64_t>(1) << 16;                       // leading byte offset (unused)
  d |= static_cast<uint64_t>(128 >> 4) << 32;                // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
  return d;                                                  // layout type 0: no swizzle
}

// Two f32 -> two BF16 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// One GEMM of a grouped launch. Tiles are numbered problem by problem.
constexpr int kMaxProblems = 24;
struct alignas(64) Problem {
  CUtensorMap b64;               // MX 256 x 384 tiles: B boxes of 64 rows (K-major) or columns
  CUtensorMap a, b, d;           // A [M][K] or [K][M], B [N][K] or [K][N] (128 x 128-byte boxes),
                                 // D [M][N] (32 x 32)
  CUtensorMap sfa, sfb;          // MX: scale atoms as [atoms][128] 32-bit words, one-atom boxes
  const float* sa;
  const float* sb;
  int32_t M, N, K;
  uint32_t idesc;
  int32_t tiles_n, tile_start;
  int32_t sumsq_slot;            // first partial slot of this problem, or -1 (not summed)
  int32_t a_mn, b_mn;            // 1: operand stored MN-major ([K][M], [K][N])
  int32_t kb128;                 // MX: K / 128, atoms per 128 rows
  int32_t a_fmt, b_fmt;          // MX: element formats (the descriptor is formed per K-block)
};
constexpr int kMaxSchedTiles = 4096, kMaxClusters = 128;
struct alignas(64) Group {
  Problem p[kMaxProblems];
  int32_t n, total_tiles;
  int32_t scheduled;             // 1: cluster c runs order[start[c] .. start[c+1])
  uint16_t start[kMaxClusters + 1];
  uint16_t order[kMaxSchedTiles];  // 3 * tile + part; part 0: whole tile, 1 / 2: the first / second
                                   // 256-column half of a wide tile
  // sum of squares (sumsq_out null: off)
  double* partials;              // every launch's slots (8 per summed tile)
  double* sumsq_out;
  unsigned int* ticket;          // zero on entry, left zero
  unsigned int* abort_word;      // set by any CTA of the call whose waits expired; zero on entry,
                                 // left zero
  int32_t n_partials;            // slots of all launches of the call
  int32_t last_launch;           // this launch reduces the slots
};
constexpr int kSumsqPerTile = 8; // 2 CTAs x 4 epilogue warps

// Number of work items cluster c runs, and the tile and part of its i-th.
__device__ __forceinline__ int tiles_of(const Group& g, int c, int n_clusters) {
  return g.scheduled ? g.start[c + 1] - g.start[c]
                     : (g.total_tiles > c ? (g.total_tiles - c + n_clusters - 1) / n_clusters : 0);
}
__device__ __forceinline__ int tile_at(const Group& g, int c, int n_clusters, int i) {
  return g.scheduled ? g.order[g.start[c] + i] / 3 : c + i * n_clusters;
}
__device__ __forceinline__ int part_at(const Group& g, int c, int i) {
  return g.scheduled ? g.order[g.start[c] + i] % 3 : 0;
}

__device__ __forceinline__ int find_problem(const Group& g, int tile) {
  int p = 0;
  while (p + 1 < g.n && g.p[p + 1].tile_start <= tile) ++p;
  return p;
}

struct Smem {
  uint64_t full[kStages];     // even CTA: both CTAs' loads of a stage have landed
  uint64_t empty[kStages];    // both CTAs: the pair MMA has consumed a stage
  uint64_t acc_full[2];       // both CTAs: an accumulator holds a finished tile
  uint64_t acc_empty[2];      // even CTA: both epilogues have drained an accumulator
  uint64_t acc_shared_free;   // even CTA (MX): both epilogues have read the overlapping chunk
  uint64_t mma_done;          // even CTA: every issued MMA has completed
  uint32_t tmem_base;
  int abort;
};

template <bool MX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_fp8_gemm(const __grid_constant__ Group g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint8_t* sEpi = smem + kStages * kStageBytes;              // 1024-byte aligned
  uint8_t* sSF = sEpi + kEpiBytes;                           // MX: [stage][SFA 512 | SFB 1024]
  Smem* S = reinterpret_cast<Smem*>(sSF + (MX ? kStages * kSfStageBytes : 0));
  constexpr uint32_t kTx = kPairTxBytes + (MX ? 2 * kSfStageBytes : 0);
  volatile int* abort_flag = &S->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int my_tiles = tiles_of(g, cluster, n_clusters);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&S->full[s]), 1);
      mbar_init(smem_u32(&S->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&S->acc_full[a]), 1);
      mbar_init(smem_u32(&S->acc_empty[a]), 8);      // 4 epilogue warps x 2 CTAs
    }
    mbar_init(smem_u32(&S->acc_shared_free), 8);
    mbar_init(smem_u32(&S->mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int p = 0; p < g.n && p < 8; ++p) {
      tma_prefetch_desc(&g.p[p].a);
      tma_prefetch_desc(&g.p[p].b);
      tma_prefetch_desc(&g.p[p].d);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&S->tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                 // barriers initialised and TMEM allocated in both CTAs
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
        const int local = tile - P.tile_start;
        const int m0 = (local / P.tiles_n) * kBM + static_cast<int>(rank) * kHalf;
        const int n0 = (local % P.tiles_n) * kBN + static_cast<int>(rank) * kHalf;
        const int num_kb = (P.K + kBK - 1) / kBK;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (*abort_flag) break;
          if (!mbar_wait(smem_u32(&S->empty[s]), ph ^ 1, limit, expire_main)) {
            *abort_flag = 1;
            record_error(kErrTimeout);
            break;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&S->full[s]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&S->full[s]), kTx);
          if (MX) {                    // scale atoms: this CTA's 128 A rows, the tile's 256 B rows
            const int mt = (local / P.tiles_n), nt = (local % P.tiles_n);
            uint8_t* sf = sSF + s * kSfStageBytes;
            tma_load_2d_pair(smem_u32(sf), &P.sfa, 0,
                             (2 * mt + static_cast<int>(rank)) * P.kb128 + kb, full_leader);
            tma_load_2d_pair(smem_u32(sf + kSfaBytes), &P.sfb, 0, (2 * nt) * P.kb128 + kb,
                             full_leader);
            tma_load_2d_pair(smem_u32(sf + kSfaBytes + 512), &P.sfb, 0,
                             (2 * nt + 1) * P.kb128 + kb, full_leader);
          }
          if (P.a_mn) tma_load_2d_pair(smem_u32(sA + s * kABytes), &P.a, m0, kb * kBK, full_leader);
          else        tma_load_2d_pair(smem_u32(sA + s * kABytes), &P.a, kb * kBK, m0, full_leader);
          if (P.b_mn) tma_load_2d_pair(smem_u32(sB + s * kBBytes), &P.b, n0, kb * kBK, full_leader);
          else        tma_load_2d_pair(smem_u32(sB + s * kBBytes), &P.b, kb * kBK, n0, full_leader);
          ++issued;
        }
      }
      // the even CTA can see its own stages land: wait for the last ones it armed (one shared
      // budget; after an abort a stage may miss the peer's bytes, and the settle delay below
      // covers loads still in flight)
      if (leader) {
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t i = issued > kStages ? issued - kStages : 0; i < issued; ++i) {
          const uint64_t spent = globaltimer_ns() - t0;
          if (spent >= kPairDrainNs) break;
          mbar_wait(smem_u32(&S->full[i % kStages]), (i / kStages) & 1, kPairDrainNs - spent);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA)
      uint32_t it = 0, local = 0;
      for (int i = 0; i < my_tiles && !*abort_flag; ++i, ++local) {
        const int tile = tile_at(g, cluster, n_clusters, i);
        const Problem& P = g.p[find_problem(g, tile)];
        const int num_kb = (P.K + kBK - 1) / kBK;
        const uint32_t idesc = P.idesc;
        const bool a_mn = P.a_mn != 0, b_mn = P.b_mn != 0;
        const uint32_t acc = local & 1, aph = (local >> 1) & 1;
        if (!mbar_wait(smem_u32(&S->acc_empty[acc]), aph ^ 1, limit, expire_main)) {
          *abort_flag = 1;
          record_error(kErrTimeout);
          break;
        }
        // MX: the previous tile (other accumulator) must have handed back the shared chunk
        if (MX && local > 0 &&
            !mbar_wait(smem_u32(&S->acc_shared_free), (local - 1) & 1, limit, expire_main)) {
          *abort_flag = 1;
          record_error(kErrTimeout);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * (MX ? kMxAcc1Col : kAccCols);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (*abort_flag || !mbar_wait(smem_u32(&S->full[s]), ph, limit, expire_main)) {
            if (!*abort_flag) record_error(kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * kABytes);
          const uint32_t b_base = smem_u32(sB + s * kBBytes);
          if (MX) {                    // this stage's scales into tensor memory, then 4 MMAs
            const uint32_t sf = smem_u32(sSF + s * kSfStageBytes);
            tc_cp_32x128b_warpx4_pair(tmem + kSfaCol, make_sf_desc(sf));
            tc_cp_32x128b_warpx4_pair(tmem + kSfbCol, make_sf_desc(sf + kSfaBytes));
            tc_cp_32x128b_warpx4_pair(tmem + kSfbCol + 4, make_sf_desc(sf + kSfaBytes + 512));
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k)
              tc_mma_mxf8_pair(d_tmem,
                               a_mn ? make_sw128_desc_mn(a_base + k * kUmmaK * 128)
                                    : make_sw128_desc(a_base + k * kUmmaK),
                               b_mn ? make_sw128_desc_mn(b_base + k * kUmmaK * 128)
                                    : make_sw128_desc(b_base + k * kUmmaK),
                               make_idesc_mx(P.a_fmt, P.b_fmt, P.a_mn, P.b_mn, k),
                               (tmem + kSfaCol) | (static_cast<uint32_t>(k) << 30),
                               (tmem + kSfbCol) | (static_cast<uint32_t>(k) << 30),
                               (kb | k) != 0 ? 1u : 0u);
          } else {
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)
            tc_mma_f8_pair(d_tmem,
                           a_mn ? make_sw128_desc_mn(a_base + k * kUmmaK * 128)
                                : make_sw128_desc(a_base + k * kUmmaK),
                           b_mn ? make_sw128_desc_mn(b_base + k * kUmmaK * 128)
                                : make_sw128_desc(b_base + k * kUmmaK),
                           idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair_mc(smem_u32(&S->empty[s]), 0x3);
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&S->acc_full[acc]), 0x3);
      }
      // every MMA issued here must complete before either CTA frees TMEM or shared memory
      tc_commit_pair(smem_u32(&S->mma_done));
      mbar_wait(smem_u32(&S->mma_done), 0, kDrainLimitNs);
    }
  } else {
    // ---------------- epilogue warps 2..5 (both CTAs)
    const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
    uint8_t* my_buf = sEpi + (warp - 2) * 2 * kEpiChunkBytes;
    uint32_t local = 0, chunk_count = 0;
    for (int i = 0; i < my_tiles; ++i, ++local) {
      const int tile = tile_at(g, cluster, n_clusters, i);
      const uint32_t acc = local & 1, aph = (local >> 1) & 1;
      if (*abort_flag) break;
      if (!mbar_wait(smem_u32(&S->acc_full[acc]), aph, limit, expire_epi)) {
        *abort_flag = 1;
        record_error(kErrTimeout);
        break;
      }
      tc_fence_after();
      const Problem& P = g.p[find_problem(g, tile)];
      const int M = P.M, N = P.N, local_tile = tile - P.tile_start;
      const float alpha = P.sa ? __fmul_rn(__ldg(P.sa), __ldg(P.sb)) : 1.0f;
      const int row0 = (local_tile / P.tiles_n) * kBM + static_cast<int>(rank) * kHalf + quad * 32;
      const int n0 = (local_tile % P.tiles_n) * kBN;
      const uint32_t t_base =
          tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * (MX ? kMxAcc1Col : kAccCols);
      const bool sumsq = P.sumsq_slot >= 0;
      double ss = 0.0;
      // one 32 x 32 chunk of packed BF16 (16 words per lane) into the swizzled staging buffer
      // and out with a TMA store; the sum of squares of the stored values when asked
      auto store_chunk = [&](int c, const uint32_t (&w16)[16]) {
        uint8_t* buf = my_buf + (chunk_count & 1) * kEpiChunkBytes;
        ++chunk_count;
        if (lane == 0) bulk_wait_group_read<1>();    // the store that last used buf has read it
        __syncwarp();
        // row `lane` of the chunk: 64 bytes = four 16-byte pieces, 64-byte swizzle
        // (piece p of row i lives at piece p ^ ((i >> 1) & 3)), matching the store's map
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          if (sumsq) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t w = w16[4 * p + q];
              const double lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
              ss = __fma_rn(lo, lo, ss);                // squares of BF16 values are exact
              ss = __fma_rn(hi, hi, ss);
            }
          }
          const int pp = p ^ ((lane >> 1) & 3);
          *reinterpret_cast<uint4*>(buf + lane * 64 + pp * 16) =
              make_uint4(w16[4 * p], w16[4 * p + 1], w16[4 * p + 2], w16[4 * p + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&P.d, smem_u32(buf), n0 + c * 32, row0);
          bulk_commit_group();
        }
      };
      if (MX) {
        // the chunk the two accumulators share comes first (accumulator 0: chunk 7, walking
        // down; accumulator 1: chunk 0, walking up); once it is in registers it is released
#pragma unroll 1
        for (int step = 0; step < kBN / 32; ++step) {
          const int c = acc == 0 ? kBN / 32 - 1 - step : step;
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_base + c * 32, r);
          tmem_ld_wait();
          tmem_reg_fence(r);
          if (step == 0) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&S->acc_shared_free), 0));
          }
          if (n0 + c * 32 >= N || row0 >= M) continue;  // chunk entirely outside the matrix
          uint32_t w16[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w16[j] = pack_bf16x2(__fmul_rn(__uint_as_float(r[2 * j]), alpha),
                                 __fmul_rn(__uint_as_float(r[2 * j + 1]), alpha));
          store_chunk(c, w16);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&S->acc_empty[acc]), 0));
      } else {
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_base + c * 32, r);
          tmem_ld_wait();
          tmem_reg_fence(r);
          if (n0 + c * 32 >= N || row0 >= M) continue;  // chunk entirely outside the matrix
          uint32_t w16[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w16[j] = pack_bf16x2(__fmul_rn(__uint_as_float(r[2 * j]), alpha),
                                 __fmul_rn(__uint_as_float(r[2 * j + 1]), alpha));
          store_chunk(c, w16);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&S->acc_empty[acc]), 0));
      }
      if (sumsq) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        if (lane == 0) {
          g.partials[P.sumsq_slot + local_tile * kSumsqPerTile + static_cast<int>(rank) * 4 + quad] = ss;
          __threadfence();                           // before this CTA's ticket
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();             // every store complete before exit
  }
  __syncwarp();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {           // loads of either CTA may still be in flight
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < kSettleNs) {
    }
  }
  tc_fence_before();
  cluster_sync();                 // neither CTA leaves while the pair MMA may still read it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);

  // ---------------- sum of squares: the last CTA of the last launch adds the slots in order
  if (!g.sumsq_out) return;
  // a CTA whose waits expired left slots unwritten: it marks the call (any of its launches)
  if (threadIdx.x == 0 && *abort_flag) atomicOr(g.abort_word, 1u);
  if (!g.last_launch) return;
  __shared__ int s_last;
  __shared__ double s_part[kThreads];
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(g.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = threadIdx.x; i < g.n_partials; i += kThreads) acc = __dadd_rn(acc, __ldcg(g.partials + i));
  s_part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double total = 0.0;
    for (int i = 0; i < kThreads; ++i) total = __dadd_rn(total, s_part[i]);
    // a launch of this call whose waits expired has slots that were never written (expired waits
    // of other calls do not matter here)
    if (*reinterpret_cast<volatile unsigned int*>(g.abort_word) != 0u)
      total = __longlong_as_double(0x7FF8000000000000LL);
    *g.sumsq_out = total;
    atomicExch(g.abort_word, 0u);
    atomicExch(g.ticket, 0u);
  }
}

// ---------------------------------------------------------------- wide tiles (N = 512 per pair)
// For launches whose every problem has N >= 512: a pair computes a 256 x 512 tile, each k-step
// two N = 256 MMAs into one 512-column accumulator (the whole of tensor memory). Per SM and
// k-block that is 48 KB of operands (A 16 KB, two B boxes 32 KB) for 1024 tensor-core cycles,
// three quarters of the bytes per FLOP of the 256 x 256 tile: the narrow tile needs about 64 B
// per SM-cycle from L2, at the limit of what an SM's TMA loads bring in, and its MMAs waited for
// operands about a sixth of the time. With a single accumulator the next tile's MMAs wait until
// the epilogue has read this one, so eight epilogue warps (two per TMEM lane quarter, one per
// 256-column half) pull the accumulator into registers as packed BF16 (128 registers a thread),
// release it, and only then store it. A work item may also be one 256-column half of a tile
// (part 1 or 2): only that half's B box is loaded, one MMA per k-step runs, and only that half's
// epilogue warps store; the host uses such halves to balance the clusters' loads.
constexpr int kBNw = 512;
constexpr int kStagesW = 4;
constexpr int kBBytesW = 2 * kHalf * kBK;                  // two 128-row B boxes per CTA
constexpr int kStageBytesW = kABytes + kBBytesW;
constexpr uint32_t kPairTxBytesW = 2 * kStageBytesW;
constexpr int kEpiWarpsW = 8;
constexpr int kThreadsW = 64 + 32 * kEpiWarpsW;            // producer, MMA issuer, 8 epilogue warps
constexpr int kEpiBytesW = kEpiWarpsW * 2 * kEpiChunkBytes;
constexpr int kSmemBytesW = kStagesW * kStageBytesW + kEpiBytesW + 1024 + 256;
constexpr int kSumsqPerTileW = 16;                         // 2 CTAs x 8 epilogue warps

struct SmemW {
  uint64_t full[kStagesW];
  uint64_t empty[kStagesW];
  uint64_t acc_full;          // both CTAs: the accumulator holds a finished tile
  uint64_t acc_empty;         // even CTA: every epilogue warp of both CTAs has read it
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsW, 1)
    k_fp8_gemm_wide(const __grid_constant__ Group g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;                                        // [stage][128 rows][128 B]
  uint8_t* sB = smem + kStagesW * kABytes;                   // [stage][2 boxes][128 rows][128 B]
  uint8_t* sEpi = smem + kStagesW * kStageBytesW;
  SmemW* S = reinterpret_cast<SmemW*>(sEpi + kEpiBytesW);
  volatile int* abort_flag = &S->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int my_tiles = tiles_of(g, cluster, n_clusters);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesW; ++s) {
      mbar_init(smem_u32(&S->full[s]), 1);
      mbar_init(smem_u32(&S->empty[s]), 1);
    }
    mbar_init(smem_u32(&S->acc_full), 1);
    mbar_init(smem_u32(&S->acc_empty), 2 * kEpiWarpsW);
    mbar_init(smem_u32(&S->mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int p = 0; p < g.n && p < 8; ++p) {
      tma_prefetch_desc(&g.p[p].a);
      tma_prefetch_desc(&g.p[p].b);
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
      // ---------------- TMA producer (both CTAs): A box and two B boxes per stage
      uint32_t it = 0, issued = 0;
      for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
        const int tile = tile_at(g, cluster, n_clusters, i), part = part_at(g, cluster, i);
        const Problem& P = g.p[find_problem(g, tile)];
        const int local = tile - P.tile_start;
        const int m0 = (local / P.tiles_n) * kBM + static_cast<int>(rank) * kHalf;
        const int n0 = (local % P.tiles_n) * kBNw + static_cast<int>(rank) * kHalf;
        const int num_kb = (P.K + kBK - 1) / kBK;
        const int h0 = part == 2 ? 1 : 0, h1 = part == 1 ? 1 : 2;   // B halves [h0, h1)
        const uint32_t tx = 2u * (kABytes + (h1 - h0) * kBBytes);    // both CTAs' boxes
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % kStagesW, ph = (it / kStagesW) & 1;
          if (*abort_flag) break;
          if (!mbar_wait(smem_u32(&S->empty[s]), ph ^ 1, limit, expire_main)) {
            *abort_flag = 1;
            record_error(kErrTimeout);
            break;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&S->full[s]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&S->full[s]), tx);
          const uint32_t a_dst = smem_u32(sA + s * kABytes), b_dst = smem_u32(sB + s * kBBytesW);
          if (P.a_mn) tma_load_2d_pair(a_dst, &P.a, m0, kb * kBK, full_leader);
          else        tma_load_2d_pair(a_dst, &P.a, kb * kBK, m0, full_leader);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h < h0 || h >= h1) continue;     // the other half of a split tile
            const uint32_t dst = b_dst + h * kBBytes;
            if (P.b_mn) tma_load_2d_pair(dst, &P.b, n0 + h * kBN, kb * kBK, full_leader);
            else        tma_load_2d_pair(dst, &P.b, kb * kBK, n0 + h * kBN, full_leader);
          }
          ++issued;
        }
      }
      if (leader) {
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t i = issued > kStagesW ? issued - kStagesW : 0; i < issued; ++i) {
          const uint64_t spent = globaltimer_ns() - t0;
          if (spent >= kPairDrainNs) break;
          mbar_wait(smem_u32(&S->full[i % kStagesW]), (i / kStagesW) & 1, kPairDrainNs - spent);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA): two N = 256 MMAs per k-step
      uint32_t it = 0, local = 0;
      for (int i = 0; i < my_tiles && !*abort_flag; ++i, ++local) {
        const int tile = tile_at(g, cluster, n_clusters, i), part = part_at(g, cluster, i);
        const Problem& P = g.p[find_problem(g, tile)];
        const int num_kb = (P.K + kBK - 1) / kBK;
        const uint32_t idesc = P.idesc;
        const bool a_mn = P.a_mn != 0, b_mn = P.b_mn != 0;
        const int h0 = part == 2 ? 1 : 0, h1 = part == 1 ? 1 : 2;
        if (!mbar_wait(smem_u32(&S->acc_empty), (local & 1) ^ 1, limit, expire_main)) {
          *abort_flag = 1;
          record_error(kErrTimeout);
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % kStagesW, ph = (it / kStagesW) & 1;
          if (*abort_flag || !mbar_wait(smem_u32(&S->full[s]), ph, limit, expire_main)) {
            if (!*abort_flag) record_error(kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * kABytes);
          const uint32_t b_base = smem_u32(sB + s * kBBytesW);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            const uint64_t adesc = a_mn ? make_sw128_desc_mn(a_base + k * kUmmaK * 128)
                                        : make_sw128_desc(a_base + k * kUmmaK);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (h < h0 || h >= h1) continue;   // the other half of a split tile
              const uint32_t bb = b_base + h * kBBytes;
              tc_mma_f8_pair(tmem + h * kAccCols, adesc,
                             b_mn ? make_sw128_desc_mn(bb + k * kUmmaK * 128)
                                  : make_sw128_desc(bb + k * kUmmaK),
                             idesc, (kb | k) != 0 ? 1u : 0u);
            }
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
      const int tile = tile_at(g, cluster, n_clusters, i), part = part_at(g, cluster, i);
      if (*abort_flag) break;
      if (!mbar_wait(smem_u32(&S->acc_full), local & 1, limit, expire_epi)) {
        *abort_flag = 1;
        record_error(kErrTimeout);
        break;
      }
      tc_fence_after();
      if (part != 0 && part != half + 1) {        // the other half of a split tile: nothing here
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&S->acc_empty), 0));
        continue;
      }
      const Problem& P = g.p[find_problem(g, tile)];
      const int M = P.M, N = P.N, local_tile = tile - P.tile_start;
      const float alpha = P.sa ? __fmul_rn(__ldg(P.sa), __ldg(P.sb)) : 1.0f;
      const int row0 = (local_tile / P.tiles_n) * kBM + static_cast<int>(rank) * kHalf + quad * 32;
      const int n0 = (local_tile % P.tiles_n) * kBNw + half * kAccCols;
      const uint32_t t_base = tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * kAccCols;
      // the whole half-row of this lane into registers as packed BF16, then release the
      // accumulator so the next tile's MMAs can start while these values are stored
      uint32_t w[kAccCols / 32][16];
#pragma unroll
      for (int c = 0; c < kAccCols / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_base + c * 32, r);
        tmem_ld_wait();
        tmem_reg_fence(r);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          w[c][j] = pack_bf16x2(__fmul_rn(__uint_as_float(r[2 * j]), alpha),
                                __fmul_rn(__uint_as_float(r[2 * j + 1]), alpha));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&S->acc_empty), 0));
      const bool sumsq = P.sumsq_slot >= 0;
      double ss = 0.0;
#pragma unroll
      for (int c = 0; c < kAccCols / 32; ++c) {
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
      if (sumsq) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        if (lane == 0) {
          g.partials[P.sumsq_slot + local_tile * kSumsqPerTileW + static_cast<int>(rank) * kEpiWarpsW +
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

  if (!g.sumsq_out) return;
  if (threadIdx.x == 0 && *abort_flag) atomicOr(g.abort_word, 1u);
  if (!g.last_launch) return;
  __shared__ int s_last;
  double* s_part = reinterpret_cast<double*>(sA);  // the stage buffers are idle by now
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(g.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = threadIdx.x; i < g.n_partials; i += kThreadsW) acc = __dadd_rn(acc, __ldcg(g.partials + i));
  s_part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double total = 0.0;
    for (int i = 0; i < kThreadsW; ++i) total = __dadd_rn(total, s_part[i]);
    if (*reinterpret_cast<volatile unsigned int*>(g.abort_word) != 0u)
      total = __longlong_as_double(0x7FF8000000000000LL);
    *g.sumsq_out = total;
    atomicExch(g.abort_word, 0u);
    atomicExch(g.ticket, 0u);
  }
}

}  // namespace gemm
}  // namespace fp8t
