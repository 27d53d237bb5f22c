// cast_transpose_amax.cuh — BF16 -> FP8 quantise with a per-tensor scale, row-major and
// transposed outputs, amax and quality counters, in one pass over HBM, for one or several
// tensors per launch.
//
// Method: the FP8Tensor quantize step of "FP8 混合精度训练工程实践" §四 (amax = max|x|;
// q = clamp(x * scale) stored as FP8) with the HYBRID format choice of "LLM FP8 微调上线生产实战"
// (核心原理: E4M3 forward, E5M2 gradients) and its saturation / zero-fraction metrics (第四步).
//
// Persistent CTAs (two per SM) walk the 128 x 128 tiles of all tensors of the launch. Per CTA:
//   * thread 0 keeps two input tiles in flight: 128 x 128 BF16 boxes (32 KB) loaded by TMA into a
//     double buffer in shared memory, completion on one mbarrier per buffer;
//   * each of 256 threads converts four 16-element row segments (f32 multiply,
//     cvt.rn.satfinite), stores its 16 FP8 bytes row-major straight to global memory (a warp
//     writes four full 128-byte row pieces) and stages them in a 16-byte-chunk XOR-swizzled tile;
//   * the transposing pass gathers 16 x 4-byte blocks from the staged tile (conflict-free),
//     transposes 4 x 4 byte blocks with byte permutes and writes the 128 x 128 q^T tile to shared
//     memory, which thread 0 stores with one TMA bulk tensor store (clipped at the tensor edge);
//   * amax and counters are reduced per tile (warp reductions, one atomic per tile);
//   * optionally the CTA that finishes last (a ticket counter) performs the delayed-scaling
//     update of every tensor of the launch, one warp per tensor: history roll, next scale and
//     its inverse, amax slot reset (the same arithmetic as the scale-update kernel). Every read
//     of a tensor's scale and every amax atomic happened before the ticket was taken.
// Algorithmic traffic: 2 B read + 2 B written per element.
#pragma once

#include "ptx.cuh"
#include "scale_update.cuh"

namespace fp8t {
namespace cast {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kMaxTensors = 8;                       // tensors per launch
constexpr int kInBytes = kTile * kTile * 2;          // one BF16 input box
constexpr int kQBytes = kTile * kTile;               // one FP8 tile
constexpr int kSmemBytes = 2 * kInBytes + 2 * kQBytes + 1024 /*alignment*/ + 64 /*barriers*/;

struct alignas(64) Tensor {
  CUtensorMap x_map;               // BF16 [rows][cols], 128 x 128 boxes
  CUtensorMap qt_map;              // FP8 [cols][rows] (q^T), 128 x 128 boxes
  const uint4* x;                  // the same BF16 data (row-major kernel), null: update only
  float* scale;                    // read by the cast; replaced by the next scale when updating
  unsigned int* amax_bits;
  float* scale_inv;
  float* hist;                     // update only: [H] history, entry 0 newest
  float* scale_inv_next;           // update only: 1 / next scale
  unsigned long long* counters;    // may be null
  uint8_t* q;                      // row-major FP8 output, may be null
  int64_t rows, cols, tiles_c, tile_start;
  int32_t fmt, has_qt;
};

struct alignas(64) Group {
  Tensor t[kMaxTensors];
  int32_t n;
  int64_t total_tiles;
  unsigned int* ticket;            // update only: zero on entry, left zero
  int32_t update, H, algo_max, margin;
};

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) { return __reduce_max_sync(0xffffffffu, v); }
__device__ __forceinline__ uint32_t warp_add_u32(uint32_t v) { return __reduce_add_sync(0xffffffffu, v); }

__device__ __forceinline__ int find_tensor(const Group& g, int64_t tile) {
  int t = 0;
  while (t + 1 < g.n && g.t[t + 1].tile_start <= tile) ++t;
  return t;
}

__device__ __forceinline__ void issue_tile_load(const Group& g, int64_t tile, uint32_t dst,
                                                uint32_t bar) {
  const Tensor& T = g.t[find_tensor(g, tile)];
  const int64_t local = tile - T.tile_start;
  const int32_t r0 = static_cast<int32_t>((local / T.tiles_c) * kTile);
  const int32_t c0 = static_cast<int32_t>((local % T.tiles_c) * kTile);
  mbar_arrive_expect_tx(bar, kInBytes);              // out-of-range parts are zero-filled
  tma_load_2d(dst, &T.x_map, c0, r0, bar);
}

// 16 BF16 (two 16-byte words) -> 16 FP8 codes. Returns the segment's largest magnitude pair
// (two 16-bit halves); counters are updated only in the COUNT variant.
template <int FMT, bool COUNT>
__device__ __forceinline__ uint32_t quantise16(const uint4 (&in)[2], float s, uint32_t (&packed)[4],
                                               uint32_t& nsat, uint32_t& nzero,
                                               uint32_t& nnonfinite) {
  constexpr float kMax = FMT == 0 ? 448.0f : 57344.0f;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&in[0]);
  uint32_t mag2 = 0;                                // per-half max of |x| bit patterns
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    mag2 = __vmaxu2(mag2, w[j] & 0x7FFF7FFFu);
    const float p0 = __fmul_rn(__uint_as_float(w[j] << 16), s);
    const float p1 = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), s);
    const uint32_t pair = cvt_fp8x2<FMT>(p0, p1);
    packed[j >> 1] |= pair << (16 * (j & 1));
    if (COUNT) {
      nsat += (fabsf(p0) > kMax) + (fabsf(p1) > kMax);
      nzero += ((pair & 0x7Fu) == 0) + ((pair & 0x7F00u) == 0);
      const uint32_t m0 = w[j] & 0x7FFFu, m1 = (w[j] >> 16) & 0x7FFFu;
      nnonfinite += (m0 >= 0x7F80u) + (m1 >= 0x7F80u);
    }
  }
  return mag2;
}

// Rare path: a segment with a NaN input, or a non-finite scale, may hold NaN products; those are
// stored as the byte 0x7F whatever their sign.
__device__ __forceinline__ void canonicalise_nan16(const uint4 (&in)[2], float s,
                                                   uint32_t (&packed)[4]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&in[0]);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float p0 = __fmul_rn(__uint_as_float(w[j] << 16), s);
    const float p1 = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), s);
    const int sh = 16 * (j & 1);
    if (p0 != p0) packed[j >> 1] = (packed[j >> 1] & ~(0xFFu << sh)) | (0x7Fu << sh);
    if (p1 != p1) packed[j >> 1] = (packed[j >> 1] & ~(0xFF00u << sh)) | (0x7F00u << sh);
  }
}

template <bool COUNT>
__device__ __forceinline__ uint32_t quantise_segment(const Tensor& T, const uint4 (&in)[2], float s,
                                                     uint32_t (&packed)[4], uint32_t& nsat,
                                                     uint32_t& nzero, uint32_t& nnonfinite) {
  const uint32_t mag2 = T.fmt == 0 ? quantise16<0, COUNT>(in, s, packed, nsat, nzero, nnonfinite)
                                   : quantise16<1, COUNT>(in, s, packed, nsat, nzero, nnonfinite);
  const uint32_t m = max(mag2 & 0xFFFFu, mag2 >> 16);
  if (m > 0x7F80u || !isfinite(s)) canonicalise_nan16(in, s, packed);   // no zero code changes
  return m;
}

// Ticket word of a fused cast launch: each CTA adds 1 when it is done, plus kTicketAbort if one
// of its waits expired (grids stay far below 2^16 CTAs), so the last CTA learns from the value it
// draws whether this launch, and only this launch, is complete.
constexpr unsigned kTicketAbort = 1u << 16;

// The last CTA of a launch to finish (ticket counter) updates the scale state of every tensor of
// the launch, one warp per tensor. Called by every thread of every CTA once its own work, amax
// atomics included, is issued; `aborted` is the same for every thread of the CTA.
__device__ __forceinline__ void last_cta_update(const Group& g, bool aborted) {
  __shared__ int s_last, s_complete;
  const int warp = threadIdx.x >> 5;
  // every CTA pulls its warps' scale state (a few KB) into its SM's L1 ahead of its ticket, so
  // the CTA that turns out to be last does not wait for HBM or L2 there
  if (warp < g.n) scale::warp_prefetch_state(g.t[warp].hist, g.H, g.t[warp].scale);
  __threadfence();                                 // this CTA's amax atomics before its ticket
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned old = atomicAdd(g.ticket, aborted ? 1u + kTicketAbort : 1u);
    s_last = (old & (kTicketAbort - 1u)) == gridDim.x - 1;
    s_complete = !aborted && old < kTicketAbort;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // a launch whose own waits expired leaves the scale state alone (its amax may be incomplete);
  // an expired wait of any other launch does not matter here
  const bool ok = s_complete != 0;
  if (ok && warp < g.n) {
    const Tensor& T = g.t[warp];
    scale::warp_update(reinterpret_cast<float*>(T.amax_bits), T.hist, g.H,
                       T.fmt == 0 ? 448.0f : 57344.0f, g.algo_max != 0, g.margin, T.scale,
                       T.scale_inv_next);
  }
  if (threadIdx.x == 0) atomicExch(g.ticket, 0u);
}

template <bool COUNT>
__global__ void __launch_bounds__(kThreads, 2) k_cast_transpose_amax(const __grid_constant__ Group g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* in_buf = smem;                                           // [2][128][256 B]
  uint32_t* stage = reinterpret_cast<uint32_t*>(smem + 2 * kInBytes);   // swizzled q tile
  uint8_t* qt_tile = smem + 2 * kInBytes + kQBytes;                 // [128][128 B] q^T tile
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * kInBytes + 2 * kQBytes);
  __shared__ uint32_t red[4][kThreads / 32];
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t stride = gridDim.x;
  uint32_t pending = 0;      // thread 0: bit b = a load into buffer b not yet consumed
  uint32_t pending_ph = 0;   // bit b = the mbarrier phase that load completes

  if (tid == 0) {
    mbar_init(smem_u32(&full[0]), 1);
    mbar_init(smem_u32(&full[1]), 1);
    fence_mbar_init();
    s_abort = 0;
    for (int b = 0; b < 2; ++b) {
      const int64_t tile = blockIdx.x + b * stride;
      if (tile < g.total_tiles) {
        issue_tile_load(g, tile, smem_u32(in_buf + b * kInBytes), smem_u32(&full[b]));
        pending |= 1u << b;                // iteration b uses phase (b >> 1) & 1 == 0
      }
    }
  }
  __syncthreads();
  const uint64_t limit = wait_limit_ns();
  const bool expire = expire_mode() != kExpireNone;

  for (int64_t i = 0;; ++i) {
    const int64_t tile = blockIdx.x + i * stride;
    if (tile >= g.total_tiles) break;
    const int buf = static_cast<int>(i & 1);
    if (tid == 0) {
      if (!mbar_wait(smem_u32(&full[buf]), static_cast<uint32_t>((i >> 1) & 1), limit, expire)) {
        record_error(kErrTimeout);
        s_abort = 1;
      } else {
        pending &= ~(1u << buf);
      }
    }
    __syncthreads();
    if (s_abort) break;

    const Tensor& T = g.t[find_tensor(g, tile)];
    const int64_t local = tile - T.tile_start;
    const int64_t r0 = (local / T.tiles_c) * kTile, c0 = (local % T.tiles_c) * kTile;
    const float s = __ldg(T.scale);
    const uint8_t* src = in_buf + buf * kInBytes;
    uint32_t vmax = 0, nsat = 0, nzero = 0, nnonfinite = 0;

    // ---- phase 1: four 16-element row segments per thread
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int seg = tid + kThreads * k;
      const int row = seg >> 3, c16 = seg & 7;
      uint32_t packed[4] = {0u, 0u, 0u, 0u};
      const int64_t gr = r0 + row, gc = c0 + 16 * c16;
      if (gr < T.rows && gc < T.cols) {
        uint4 in[2];
        in[0] = *reinterpret_cast<const uint4*>(src + row * 256 + c16 * 32);
        in[1] = *reinterpret_cast<const uint4*>(src + row * 256 + c16 * 32 + 16);
        vmax = max(vmax, quantise_segment<COUNT>(T, in, s, packed, nsat, nzero, nnonfinite));
        if (T.q)
          *reinterpret_cast<uint4*>(T.q + gr * T.cols + gc) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      if (T.has_qt) {
        const int pchunk = c16 ^ ((row >> 4) & 7);
        *reinterpret_cast<uint4*>(&stage[row * 32 + pchunk * 4]) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
    }
    vmax = warp_max_u32(vmax);
    nsat = warp_add_u32(nsat);
    nzero = warp_add_u32(nzero);
    nnonfinite = warp_add_u32(nnonfinite);
    if (lane == 0) {
      red[0][warp] = vmax;
      red[1][warp] = nsat;
      red[2][warp] = nzero;
      red[3][warp] = nnonfinite;
    }
    if (tid == 0) bulk_wait_group_read<0>();       // the previous q^T store has read its tile
    __syncthreads();                               // input buffer consumed, staged tile complete

    if (tid == 0) {
      uint32_t m = 0, a = 0, b = 0, c = 0;
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) {
        m = max(m, red[0][w]);
        a += red[1][w];
        b += red[2][w];
        c += red[3][w];
      }
      if (m > 0x7F80u) m = 0x7FC0u;                // canonical NaN
      atomicMax(T.amax_bits, m << 16);             // max-accumulated into the caller's slot
      if (T.counters) {
        if (a) atomicAdd(T.counters + 0, static_cast<unsigned long long>(a));
        if (b) atomicAdd(T.counters + 1, static_cast<unsigned long long>(b));
        if (c) atomicAdd(T.counters + 2, static_cast<unsigned long long>(c));
      }
      if (T.scale_inv && local == 0) *T.scale_inv = __fdiv_rn(1.0f, s);
      const int64_t next = tile + 2 * stride;      // refill the buffer just consumed
      if (next < g.total_tiles) {
        issue_tile_load(g, next, smem_u32(in_buf + buf * kInBytes), smem_u32(&full[buf]));
        pending |= 1u << buf;
        pending_ph = (pending_ph & ~(1u << buf)) | (static_cast<uint32_t>(((i + 2) >> 1) & 1) << buf);
      }
    }

    // ---- phase 2: q^T tile, 16 q-rows x 4 q-columns per thread
    if (T.has_qt) {
      const int ig = lane & 7;                     // q rows 16*ig .. 16*ig+15
      const int jg = 4 * warp + (lane >> 3);       // q columns 4*jg .. 4*jg+3
      uint32_t v[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int row = 16 * ig + r;
        const int chunk = (jg >> 2) ^ ig;          // (row >> 4) & 7 == ig
        v[r] = stage[row * 32 + chunk * 4 + (jg & 3)];
      }
      uint32_t o[4][4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a = v[4 * kk], b = v[4 * kk + 1], c = v[4 * kk + 2], d = v[4 * kk + 3];
        const uint32_t t0 = __byte_perm(a, b, 0x5140), t1 = __byte_perm(a, b, 0x7362);
        const uint32_t u0 = __byte_perm(c, d, 0x5140), u1 = __byte_perm(c, d, 0x7362);
        o[0][kk] = __byte_perm(t0, u0, 0x5410);
        o[1][kk] = __byte_perm(t0, u0, 0x7632);
        o[2][kk] = __byte_perm(t1, u1, 0x5410);
        o[3][kk] = __byte_perm(t1, u1, 0x7632);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(qt_tile + (4 * jg + c) * kTile + 16 * ig) =
            make_uint4(o[c][0], o[c][1], o[c][2], o[c][3]);
      fence_proxy_async_smem();                    // visible to the TMA store
      __syncthreads();                             // q^T tile complete; staged tile free again
      if (tid == 0) {
        tma_store_2d(&T.qt_map, smem_u32(qt_tile), static_cast<int32_t>(r0), static_cast<int32_t>(c0));
        bulk_commit_group();
      }
    }
  }

  if (tid == 0) {
    // loads still in flight after an abort must land before shared memory is released
    for (int b = 0; b < 2; ++b)
      if (pending & (1u << b)) mbar_wait(smem_u32(&full[b]), (pending_ph >> b) & 1u, kDrainLimitNs);
    bulk_wait_group<0>();                          // stores complete before the CTA exits
  }
  if (g.update) last_cta_update(g, s_abort != 0);
}

// Row-major-only casts (no tensor of the launch wants q^T): a plain streaming kernel. Each
// thread converts 16-element segments (two 16-byte loads, one 16-byte store), four segments
// (128 bytes) in flight, grid-striding over one tensor after another; amax and counters are
// reduced per warp (one atomic per warp and tensor).
template <bool COUNT>
__global__ void __launch_bounds__(kThreads, 3) k_cast_rowmajor(const __grid_constant__ Group g) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int t = 0; t < g.n; ++t) {
    const Tensor& T = g.t[t];
    if (!T.x) continue;                            // scale update only
    const uint4* __restrict__ x = T.x;
    uint4* __restrict__ q = reinterpret_cast<uint4*>(T.q);
    const int64_t nseg = T.rows * T.cols / 16;
    const float s = __ldg(T.scale);
    uint32_t vmax = 0, nsat = 0, nzero = 0, nnonfinite = 0;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + tid;
    for (; i + 3 * stride < nseg; i += 4 * stride) {
      uint4 in[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        in[u][0] = ld_stream_u4(x + 2 * (i + u * stride));
        in[u][1] = ld_stream_u4(x + 2 * (i + u * stride) + 1);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t p[4] = {0u, 0u, 0u, 0u};
        vmax = max(vmax, quantise_segment<COUNT>(T, in[u], s, p, nsat, nzero, nnonfinite));
        if (q) q[i + u * stride] = make_uint4(p[0], p[1], p[2], p[3]);
      }
    }
    for (; i < nseg; i += stride) {
      uint4 in[2];
      in[0] = ld_stream_u4(x + 2 * i);
      in[1] = ld_stream_u4(x + 2 * i + 1);
      uint32_t p[4] = {0u, 0u, 0u, 0u};
      vmax = max(vmax, quantise_segment<COUNT>(T, in, s, p, nsat, nzero, nnonfinite));
      if (q) q[i] = make_uint4(p[0], p[1], p[2], p[3]);
    }
    vmax = warp_max_u32(vmax);
    if (COUNT) {
      nsat = warp_add_u32(nsat);
      nzero = warp_add_u32(nzero);
      nnonfinite = warp_add_u32(nnonfinite);
    }
    if (lane == 0) {
      if (vmax > 0x7F80u) vmax = 0x7FC0u;          // canonical NaN
      if (vmax) atomicMax(T.amax_bits, vmax << 16);
      if (COUNT && T.counters) {
        if (nsat) atomicAdd(T.counters + 0, static_cast<unsigned long long>(nsat));
        if (nzero) atomicAdd(T.counters + 1, static_cast<unsigned long long>(nzero));
        if (nnonfinite) atomicAdd(T.counters + 2, static_cast<unsigned long long>(nnonfinite));
      }
    }
    if (T.scale_inv && blockIdx.x == 0 && tid == 0) *T.scale_inv = __fdiv_rn(1.0f, s);
  }
  if (g.update) last_cta_update(g, false);        // this kernel has no waits that can expire
}

}  // namespace cast
}  // namespace fp8t
