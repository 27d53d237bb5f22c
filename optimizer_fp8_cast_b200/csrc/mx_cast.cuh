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
// A CTA reads its tiles into a double-buffered shared tile with 16-byte asynchronous copies (the
// next tile's copies are in flight while the current one is quantised; 16-byte chunk c of row r
// is stored at c ^ (r % 8), so that the row-wise and the column-wise reads are free of bank
// conflicts),
// quantises the row-wise blocks
// straight to global memory, the column-wise blocks into a staged tile that it then writes out
// row by row, and writes each atom with 16-byte stores.
#pragma once

#include "ptx.cuh"

namespace fp8t {
namespace mx {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kMaxTensors = 8;
constexpr int kSmemBytes = 2 * kTile * kTile * 2 + kTile * kTile + 2 * 512 + 128;

struct Tensor {
  const uint4* x;                  // BF16 [rows][cols]
  uint8_t* q_row;                  // codes, blocks along rows (may be null)
  uint8_t* sf_row;                 // atoms [rows/128][cols/128]
  uint8_t* q_col;                  // codes, blocks down columns (may be null)
  uint8_t* sf_col;                 // atoms [cols/128][rows/128]
  int64_t rows, cols, tiles_c, tile_start;
  int32_t fmt;
};

struct Group {
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

// position of 16-byte chunk c16 of tile row `row` in the swizzled BF16 tile (uint4 units)
__device__ __forceinline__ int xchunk(int row, int c16) { return row * 16 + (c16 ^ (row & 7)); }
// position of BF16 element (row, col) of the tile (uint16 units)
__device__ __forceinline__ int xelem(int row, int col) { return xchunk(row, col >> 3) * 8 + (col & 7); }

__device__ __forceinline__ int tensor_of(const Group& g, int64_t tile) {
  int ti = 0;
  while (ti + 1 < g.n && g.t[ti + 1].tile_start <= tile) ++ti;
  return ti;
}

// Issue the 16-byte copies of one 128 x 128 BF16 tile (128 rows x 256 bytes) into xs.
__device__ __forceinline__ void prefetch_tile(const Group& g, int64_t tile, uint16_t* xs) {
  const Tensor& T = g.t[tensor_of(g, tile)];
  const int64_t local = tile - T.tile_start;
  const int64_t r0 = (local / T.tiles_c) * kTile, c0 = (local % T.tiles_c) * kTile;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int v = u * kThreads + threadIdx.x, row = v >> 4, c16 = v & 15;
    cp_async_16(smem_u32(reinterpret_cast<uint4*>(xs) + xchunk(row, c16)),
                T.x + ((r0 + row) * T.cols + c0) / 8 + c16);
  }
}

__global__ void __launch_bounds__(kThreads) k_mx_cast(const __grid_constant__ Group g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  // [2][128][128] BF16 tiles at smem and smem + kXBytes
  constexpr int kXBytes = kTile * kTile * 2;
  auto xbuf = [&](int b) { return reinterpret_cast<uint16_t*>(smem + b * kXBytes); };
  uint8_t* qs = smem + 2 * kTile * kTile * 2;                       // [128][128] column-wise codes
  uint8_t* atom_r = qs + kTile * kTile;                             // 512 B
  uint8_t* atom_c = atom_r + 512;                                   // 512 B
  const int tid = threadIdx.x;

  if (static_cast<int64_t>(blockIdx.x) < g.total_tiles) prefetch_tile(g, blockIdx.x, xbuf(0));
  cp_async_commit();
  int k = 0;
  for (int64_t tile = blockIdx.x; tile < g.total_tiles; tile += gridDim.x, ++k) {
    const Tensor& T = g.t[tensor_of(g, tile)];
    const int64_t local = tile - T.tile_start;
    const int64_t r0 = (local / T.tiles_c) * kTile, c0 = (local % T.tiles_c) * kTile;
    const int emax = T.fmt == 0 ? 8 : 15;
    uint16_t* xs = xbuf(k & 1);

    // ---- the next tile's copies go out; this tile's have landed
    if (tile + gridDim.x < g.total_tiles) prefetch_tile(g, tile + gridDim.x, xbuf((k + 1) & 1));
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    // ---- row-wise blocks: 128 rows x 4 blocks, two per thread
    if (T.q_row) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int j = u * kThreads + tid, row = j >> 2, b = j & 3;
        const uint4* src = reinterpret_cast<const uint4*>(xs);
        uint4 w[4];
        uint32_t m2 = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          w[k] = src[xchunk(row, 4 * b + k)];
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
        atom_r[(row & 31) * 16 + (row >> 5) * 4 + b] = m > 0x7F80u ? 0xFF : static_cast<uint8_t>(X + 127);
      }
    }
    // ---- column-wise blocks: 128 columns x 4 blocks of 32 rows; each thread takes a column
    //      pair of one block: 32 four-byte reads (two BF16 each) and 32 two-byte code stores
    if (T.q_col) {
      const int cp = tid & 63, rb = tid >> 6, col = 2 * cp;
      uint32_t v[32];
      uint32_t m2 = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        v[i] = *reinterpret_cast<const uint32_t*>(xs + xelem(32 * rb + i, col));
        m2 = __vmaxu2(m2, v[i] & 0x7FFF7FFFu);
      }
      const uint32_t m0 = m2 & 0xFFFFu, m1 = m2 >> 16;   // column col, column col + 1
      const int X0 = m0 > 0x7F80u ? 0 : block_exponent(m0, emax);
      const int X1 = m1 > 0x7F80u ? 0 : block_exponent(m1, emax);
      const float inv0 = pow2_neg(X0), inv1 = pow2_neg(X1);
      const bool nan_block = max(m0, m1) > 0x7F80u;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = __fmul_rn(__uint_as_float(v[i] << 16), inv0);
        const float p1 = __fmul_rn(__uint_as_float(v[i] & 0xFFFF0000u), inv1);
        uint32_t c = T.fmt == 0 ? cvt_fp8x2<0>(p0, p1) : cvt_fp8x2<1>(p0, p1);
        if (nan_block) {                       // only a NaN input gives a NaN product
          if (p0 != p0) c = (c & 0xFF00u) | 0x7Fu;
          if (p1 != p1) c = (c & 0x00FFu) | 0x7F00u;
        }
        *reinterpret_cast<uint16_t*>(qs + (32 * rb + i) * kTile + col) = static_cast<uint16_t>(c);
      }
      atom_c[(col & 31) * 16 + (col >> 5) * 4 + rb] = m0 > 0x7F80u ? 0xFF : static_cast<uint8_t>(X0 + 127);
      atom_c[((col + 1) & 31) * 16 + ((col + 1) >> 5) * 4 + rb] =
          m1 > 0x7F80u ? 0xFF : static_cast<uint8_t>(X1 + 127);
    }
    __syncthreads();                                   // staged codes and both atoms complete
    if (T.q_col) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = u * kThreads + tid, row = v >> 3, c16 = v & 7;
        *reinterpret_cast<uint4*>(T.q_col + (r0 + row) * T.cols + c0 + 16 * c16) =
            reinterpret_cast<const uint4*>(qs)[v];
      }
    }
    if (tid < 32 && T.q_row)
      reinterpret_cast<uint4*>(T.sf_row + ((r0 / kTile) * T.tiles_c + c0 / kTile) * 512)[tid] =
          reinterpret_cast<const uint4*>(atom_r)[tid];
    if (tid >= 32 && tid < 64 && T.q_col)
      reinterpret_cast<uint4*>(T.sf_col + ((c0 / kTile) * (T.rows / kTile) + r0 / kTile) * 512)[tid - 32] =
          reinterpret_cast<const uint4*>(atom_c)[tid - 32];
    __syncthreads();                                   // shared buffers free for the next tile
  }
}

}  // namespace mx
}  // namespace fp8t
