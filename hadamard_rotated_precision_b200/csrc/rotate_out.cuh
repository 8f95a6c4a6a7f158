// De-rotation of a GEMM output that is still rotated on both sides: out = bf16(H Z H), H =
// blockdiag(H_k / sqrt(k)), Z fp32 [rows][cols] (the dequantized accumulators).  The rotation
// along the columns runs in the GEMM's epilogue (an epilogue thread owns an output row); this
// kernel does the one along the rows.
//
// Method: "HALO: Hadamard-Assisted Lower-Precision Optimization for LLMs", Approach (the
// quantized rotated tensors of the forward pass are reused in the backward pass, which puts a
// left-hand Hadamard on the output gradient): the input gradient then comes out of its GEMM
// rotated along the tokens (rows) and along K (columns), and both rotations are undone here.
//
// Numerics, as the library's rotation: Sylvester butterflies h = 1, 2, ..., k/2 (index bit 0
// first), every add / sub fp32 round-to-nearest-even, then one multiply by fp32(1/sqrt(k));
// the columns' rotation (each row's k-blocks) runs first, in fp32, then the rows', which
// rounds to bf16 once at the end.
//
// Streams 4 bytes read and 2 written per element.  Requires cols % k == 0 and rows % k == 0
// (so both are even and whole blocks).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace hq {
namespace rot {

constexpr int kThreads = 256;

// Along the rows, fp32 in, bf16 out.  A CTA takes a tile of 256 rows x 64 columns (whole
// k-blocks of rows, since rows % k == 0 and k divides 256); a thread holds two adjacent
// columns (8-byte loads, bf16x2 stores):
//   phase 1: thread (warp w, lane l) holds columns 2l, 2l+1 of rows 32w .. 32w+31 (bits 0-4 of
//            the row in registers) and runs the stages h = 1 .. 16;
//   phase 2 (k >= 64): through shared memory, the thread holds rows r + 32j (j = 0..7) for
//            r = 4w .. 4w+3 (bits 5-7 in registers) and runs the stages h = 32 .. k/2.
// Both phases read and write shared memory along a row (lanes = column pairs): conflict-free.
constexpr int kRowTile = 256, kColTile = 64;
constexpr size_t kRowsSmemBytes = size_t(kRowTile) * kColTile * 4;  // 64 KB (k >= 64)

template <int K>
__global__ void __launch_bounds__(kThreads) rot_rows_f32_bf16_kernel(const float* __restrict__ z, int64_t rows,
                                                                     int64_t cols, float c,
                                                                     __nv_bfloat16* __restrict__ out) {
  static_assert(K >= 16 && K <= 256 && (K & (K - 1)) == 0, "k must be a power of two in [16,256]");
  extern __shared__ float2 tile2[];  // [kRowTile][kColTile / 2], used when K >= 64
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t col_tiles = (cols + kColTile - 1) / kColTile;
  const int64_t row0 = (int64_t(blockIdx.x) / col_tiles) * kRowTile;
  const int64_t col = (int64_t(blockIdx.x) % col_tiles) * kColTile + 2 * lane;
  const bool col_ok = col < cols;  // cols is even: both columns or neither

  float2 v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int64_t r = row0 + 32 * warp + i;
    v[i] = (col_ok && r < rows) ? *reinterpret_cast<const float2*>(z + r * cols + col) : make_float2(0.0f, 0.0f);
  }
  constexpr int H1 = K < 32 ? K : 32;  // phase 1 covers h < H1
#pragma unroll
  for (int h = 1; h < H1; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i & h) continue;
      const float2 u = v[i], w = v[i + h];
      v[i] = make_float2(__fadd_rn(u.x, w.x), __fadd_rn(u.y, w.y));
      v[i + h] = make_float2(__fsub_rn(u.x, w.x), __fsub_rn(u.y, w.y));
    }
  }
  auto store = [&](int64_t r, float2 t) {
    if (col_ok && r < rows)
      *reinterpret_cast<__nv_bfloat162*>(out + r * cols + col) =
          __floats2bfloat162_rn(__fmul_rn(t.x, c), __fmul_rn(t.y, c));
  };
  if constexpr (K <= 32) {
#pragma unroll
    for (int i = 0; i < 32; ++i) store(row0 + 32 * warp + i, v[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) tile2[(32 * warp + i) * (kColTile / 2) + lane] = v[i];
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 u8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) u8[j] = tile2[(4 * warp + q + 32 * j) * (kColTile / 2) + lane];
#pragma unroll
      for (int h = 1; h < K / 32; h <<= 1) {  // register bit s of j is row bit 5 + s
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j & h) continue;
          const float2 a = u8[j], b = u8[j + h];
          u8[j] = make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
          u8[j + h] = make_float2(__fsub_rn(a.x, b.x), __fsub_rn(a.y, b.y));
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) store(row0 + 4 * warp + q + 32 * j, u8[j]);
    }
  }
}

}  // namespace rot
}  // namespace hq
