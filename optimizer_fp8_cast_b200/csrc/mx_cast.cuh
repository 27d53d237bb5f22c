// mx_cast.cuh — MXFP8 quantisation: FP8 codes with one E8M0 scale per 32 values.
//
// Method: "FP8 混合精度训练工程实践" §九 (Blackwell microscaling: 32 values share an 8-bit E8M0
// scale, each value stored as FP8) and §三 (micro scaling with E4M3 elements). The shared
// exponent of a block is X = floor(log2(amax)) - emax (emax 8 for E4M3, 15 for E5M2, the
// exponents of 448 and 57344), clamped to [-127, 127]; amax 0 gives -127, an infinite amax
// 127, a NaN in the block the scale code 0xFF (elements then encoded at unit scale). Elements
// are cvt.rn.satfinite(f32(x) * 2^-X), NaN products stored as 0x7F.
//
// Each 128 x 128 tile of x yields, for the row-wise copy (blocks along a row, the K-major GEMM
// operand) and for the column-wise copy (blocks down a column, the MN-major operand), 128 x 128
// codes in x's own row-major layout and one 512-byte atom of scales. A scale atom covers 128
// rows (M or N) x 4 blocks (128 K values): byte (i % 32) * 16 + (i / 32) * 4 + kb holds row i,
// block kb, which is the order the tensor-core scale copy (tcgen05.cp 32x128b, replicated to
// the four lane quarters) expects; atoms are stored [MN / 128][K / 128].
// Persistent CTAs (three per SM); thread 0 keeps two tiles in flight: each tile arrives as two
// TMA boxes of 128 rows x 64 columns (128-byte swizzle: 16-byte chunk c of a row's 128 bytes at
// c ^ (row % 8)) into a double buffer, completion on one mbarrier per buffer. Then, in parallel,
//   warps 0-3 quantise the column-wise blocks: a thread takes 4 adjacent columns of one block of
//     32 rows, reads them once (eight-byte shared loads) for the four scales and again to
//     quantise (a loop compiled per format and per NaN case, so neither choice is made per
//     element), and stores each row's four codes as one 4-byte word straight to global memory
//     (the warp's 32 lanes cover the row's 128 columns, so each store instruction writes one
//     whole 128-byte line);
//   warps 4-7 quantise the row-wise blocks straight to global memory: a quarter-warp takes the
//     same block of 8 consecutive rows, so its shared loads hit 8 different bank groups;
// and after a barrier the two 512-byte scale atoms, gathered in shared memory, go out. Every wait
// on an mbarrier is bounded: on expiry the CTA records the timeout in the device error word,
// stops, and waits (bounded) for its loads.
#pragma once

#include "ptx.cuh"

namespace fp8t {
namespace mx {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kMaxTensors = 8;
constexpr int kHalfBytes = kTile * 64 * 2;                 // one 128-row x 64-column BF16 box
constexpr int kXBytes = 2 * kHalfBytes;                    // one 128 x 128 BF16 tile
constexpr int kSmemBytes = 2 * kXBytes + 2 * 512 + 64 + 1024 /*alignment*/;

struct alignas(64) Tensor {
  CUtensorMap x_map;               // BF16 [rows][cols], 64 x 128 boxes, 128-byte swizzle
  uint8_t* q_row;                  // codes, blocks along rows (may be null)
  uint8_t* sf_row;                 // atoms [rows/128][cols/128]
  uint8_t* q_col;                  // codes, blocks down columns (may be null)
  uint8_t* sf_col;                 // atoms [cols/128][rows/128]
  int64_t rows, cols, tiles_c, tile_start;
  int32_t fmt;
};

struct alignas(64) Group {
  Tensor t[kMaxTensors];
  int32_t n;
  int64_t total_tiles;
};

// Shared exponent of a block from its largest BF16 magnitude pattern m (m > 0x7F80: NaN).
__device__ __forceinline__ int block_exponent(uint32_t m, int emax) {
  if (m == 0) return -127;
  if (m >= 0x7F80u) return 127;                               // infinity (NaN handled apart)
  const int e = static_cast<int>(m >> 7);
  const int fl = e ? e - 127 : (31 - __clz(m)) - 133;         // floor(log2) of normal/subnormal
  return max(-127, min(127, fl - emax));
}

// 2^-X as an f32 (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2_neg(int X) {
  return X == 127 ? __uint_as_float(0x00400000u) : __uint_as_float(static_cast<uint32_t>(127 - X) << 23);
}

// Four BF16 values (two words) -> four codes; with NAN_CHECK, NaN products become 0x7F. Only a
// block whose amax is NaN can hold a NaN product (2^-X is finite and an infinite input
// saturates), so the check runs for those blocks only.
template <int FMT, bool NAN_CHECK>
__device__ __forceinline__ uint32_t q4(uint32_t w0, uint32_t w1, float inv) {
  const float p0 = __fmul_rn(__uint_as_float(w0 << 16), inv), p1 = __fmul_rn(__uint_as_float(w0 & 0xFFFF0000u), inv);
  const float p2 = __fmul_rn(__uint_as_float(w1 << 16), inv), p3 = __fmul_rn(__uint_as_float(w1 & 0xFFFF0000u), inv);
  uint32_t r = cvt_fp8x2<FMT>(p0, p1) | (cvt_fp8x2<FMT>(p2, p3) << 16);
  if (!NAN_CHECK) return r;
  if (p0 != p0) r = (r & 0xFFFFFF00u) | 0x7Fu;
  if (p1 != p1) r = (r & 0xFFFF00FFu) | 0x7F00u;
  if (p2 != p2) r = (r & 0xFF00FFFFu) | 0x7F0000u;
  if (p3 != p3) r = (r & 0x00FFFFFFu) | 0x7F000000u;
  return r;
}

// Byte offset of BF16 element (row, col) in a tile as the two swizzled TMA boxes lay it out.
__device__ __forceinline__ uint32_t xoff(int row, int col) {
  return (col >> 6) * kHalfBytes + row * 128 + ((((col >> 3) & 7) ^ (row & 7)) << 4) + (col & 7) * 2;
}

__device__ __forceinline__ int tensor_of(const Group& g, int64_t tile) {
  int ti = 0;
  while (ti + 1 < g.n && g.t[ti + 1].tile_start <= tile) ++ti;
  return ti;
}

__device__ __forceinline__ void issue_tile(const Group& g, int64_t tile, uint32_t dst, uint32_t bar) {
  const Tensor& T = g.t[tensor_of(g, tile)];
  const int64_t local = tile - T.tile_start;
  const int32_t r0 = static_cast<int32_t>((local / T.tiles_c) * kTile);
  const int32_t c0 = static_cast<int32_t>((local % T.tiles_c) * kTile);
  mbar_arrive_expect_tx(bar, kXBytes);
  tma_load_2d(dst, &T.x_map, c0, r0, bar);
  tma_load_2d(dst + kHalfBytes, &T.x_map, c0 + 64, r0, bar);
}

__device__ __forceinline__ uint8_t scale_code(uint32_t m, int X) {
  return m > 0x7F80u ? 0xFF : static_cast<uint8_t>(X + 127);
}

// Column-wise codes of 4 adjacent columns x 32 rows of a tile (one format per instantiation),
// each row's four codes stored as one 4-byte word.
template <int FMT, bool NAN_CHECK>
__device__ __forceinline__ void col_codes(const uint8_t* xs, int rb, int col, const float (&inv)[4],
                                          uint8_t* dst, int64_t cols) {
#pragma unroll 8
  for (int r = 0; r < 32; ++r) {
    const uint2 v = *reinterpret_cast<const uint2*>(xs + xoff(32 * rb + r, col));
    const float p0 = __fmul_rn(__uint_as_float(v.x << 16), inv[0]);
    const float p1 = __fmul_rn(__uint_as_float(v.x & 0xFFFF0000u), inv[1]);
    const float p2 = __fmul_rn(__uint_as_float(v.y << 16), inv[2]);
    const float p3 = __fmul_rn(__uint_as_float(v.y & 0xFFFF0000u), inv[3]);
    uint32_t c = cvt_fp8x2<FMT>(p0, p1) | (cvt_fp8x2<FMT>(p2, p3) << 16);
    if (NAN_CHECK) {                       // only a NaN input gives a NaN product
      if (p0 != p0) c = (c & 0xFFFFFF00u) | 0x7Fu;
      if (p1 != p1) c = (c & 0xFFFF00FFu) | 0x7F00u;
      if (p2 != p2) c = (c & 0xFF00FFFFu) | 0x7F0000u;
      if (p3 != p3) c = (c & 0x00FFFFFFu) | 0x7F000000u;
    }
    *reinterpret_cast<uint32_t*>(dst + r * cols) = c;
  }
}

__global__ void __launch_bounds__(kThreads, 3) k_mx_cast(const __grid_constant__ Group g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* xbuf = smem;                                             // [2][2 boxes][128][128 B]
  uint8_t* atom_r = smem + 2 * kXBytes;                             // 512 B
  uint8_t* atom_c = atom_r + 512;                                   // 512 B
  uint64_t* full = reinterpret_cast<uint64_t*>(atom_c + 512);       // 2 mbarriers
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t stride = gridDim.x;
  uint32_t pending = 0, pending_ph = 0;      // thread 0: loads not yet consumed, their phases

  if (tid == 0) {
    mbar_init(smem_u32(&full[0]), 1);
    mbar_init(smem_u32(&full[1]), 1);
    fence_mbar_init();
    s_abort = 0;
    for (int b = 0; b < 2; ++b) {
      const int64_t tile = blockIdx.x + b * stride;
      if (tile < g.total_tiles) {
        issue_tile(g, tile, smem_u32(xbuf + b * kXBytes), smem_u32(&full[b]));
        pending |= 1u << b;
      }
    }
  }
  __syncthreads();
  const uint64_t limit = wait_limit_ns();
  const bool expire = expire_mode() == kExpireAll;

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
    __syncthreads();                          // tile landed; the previous tile's atoms written
    if (s_abort) break;
    const Tensor& T = g.t[tensor_of(g, tile)];
    const int64_t local = tile - T.tile_start;
    const int64_t r0 = (local / T.tiles_c) * kTile, c0 = (local % T.tiles_c) * kTile;
    const int emax = T.fmt == 0 ? 8 : 15;
    const uint8_t* xs = xbuf + buf * kXBytes;

    if (warp < 4) {
      // ---- column-wise blocks: columns 4cq .. 4cq+3, rows 32rb .. 32rb+31
      if (T.q_col) {
        const int cq = lane, rb = warp, col = 4 * cq;
        uint32_t ma = 0, mb = 0;
#pragma unroll 8
        for (int r = 0; r < 32; ++r) {
          const uint2 v = *reinterpret_cast<const uint2*>(xs + xoff(32 * rb + r, col));
          ma = __vmaxu2(ma, v.x & 0x7FFF7FFFu);
          mb = __vmaxu2(mb, v.y & 0x7FFF7FFFu);
        }
        const uint32_t m[4] = {ma & 0xFFFFu, ma >> 16, mb & 0xFFFFu, mb >> 16};
        int X[4];
        float inv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          X[c] = m[c] > 0x7F80u ? 0 : block_exponent(m[c], emax);
          inv[c] = pow2_neg(X[c]);
        }
        const bool nan_block = max(max(m[0], m[1]), max(m[2], m[3])) > 0x7F80u;
        uint8_t* dst = T.q_col + (r0 + 32 * rb) * T.cols + c0 + col;
        if (nan_block)
          T.fmt == 0 ? col_codes<0, true>(xs, rb, col, inv, dst, T.cols)
                     : col_codes<1, true>(xs, rb, col, inv, dst, T.cols);
        else if (T.fmt == 0) col_codes<0, false>(xs, rb, col, inv, dst, T.cols);
        else                 col_codes<1, false>(xs, rb, col, inv, dst, T.cols);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          atom_c[((col + c) & 31) * 16 + ((col + c) >> 5) * 4 + rb] = scale_code(m[c], X[c]);
      }
    } else if (T.q_row) {
      // ---- row-wise blocks: a quarter-warp takes block b of 8 consecutive rows
      const int wr = warp - 4, b = lane >> 3;
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {
        const int row = 32 * u + 8 * wr + (lane & 7);
        uint4 w[4];
        uint32_t m2 = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          w[k] = *reinterpret_cast<const uint4*>(xs + xoff(row, 32 * b + 8 * k));
          m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(w[k].x & 0x7FFF7FFFu, w[k].y & 0x7FFF7FFFu),
                                     __vmaxu2(w[k].z & 0x7FFF7FFFu, w[k].w & 0x7FFF7FFFu)));
        }
        const uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
        const int X = m > 0x7F80u ? 0 : block_exponent(m, emax);
        const float inv = pow2_neg(X);
        uint32_t out[8];
        if (m > 0x7F80u) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            out[2 * k] = T.fmt == 0 ? q4<0, true>(w[k].x, w[k].y, inv) : q4<1, true>(w[k].x, w[k].y, inv);
            out[2 * k + 1] = T.fmt == 0 ? q4<0, true>(w[k].z, w[k].w, inv) : q4<1, true>(w[k].z, w[k].w, inv);
          }
        } else if (T.fmt == 0) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            out[2 * k] = q4<0, false>(w[k].x, w[k].y, inv);
            out[2 * k + 1] = q4<0, false>(w[k].z, w[k].w, inv);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            out[2 * k] = q4<1, false>(w[k].x, w[k].y, inv);
            out[2 * k + 1] = q4<1, false>(w[k].z, w[k].w, inv);
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(T.q_row + (r0 + row) * T.cols + c0 + 32 * b);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
        atom_r[(row & 31) * 16 + (row >> 5) * 4 + b] = scale_code(m, X);
      }
    }
    __syncthreads();                          // input tile consumed; both atoms complete
    if (tid == 0) {                           // refill the buffer just consumed
      const int64_t next = tile + 2 * stride;
      if (next < g.total_tiles) {
        issue_tile(g, next, smem_u32(xbuf + buf * kXBytes), smem_u32(&full[buf]));
        pending |= 1u << buf;
        pending_ph = (pending_ph & ~(1u << buf)) | (static_cast<uint32_t>(((i + 2) >> 1) & 1) << buf);
      }
    }
    if (tid < 32 && T.q_row)
      reinterpret_cast<uint4*>(T.sf_row + ((r0 / kTile) * T.tiles_c + c0 / kTile) * 512)[tid] =
          reinterpret_cast<const uint4*>(atom_r)[tid];
    if (tid >= 32 && tid < 64 && T.q_col)
      reinterpret_cast<uint4*>(T.sf_col + ((c0 / kTile) * (T.rows / kTile) + r0 / kTile) * 512)[tid - 32] =
          reinterpret_cast<const uint4*>(atom_c)[tid - 32];
  }
  if (tid == 0) {
    // loads still in flight after an abort must land before shared memory is released
    for (int b = 0; b < 2; ++b)
      if (pending & (1u << b)) mbar_wait(smem_u32(&full[b]), (pending_ph >> b) & 1u, kDrainLimitNs);
  }
}

}  // namespace mx
}  // namespace fp8t
