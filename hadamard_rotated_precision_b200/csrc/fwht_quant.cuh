// Fused block-Hadamard rotation + tensor-wise absmax + INT8 / FP8-e4m3 quantization.
//
// Method: "Training Transformers with 4-bit Integers", section 3.3 (Hadamard quantization:
// a block-diagonal transform of k x k Hadamard blocks applied to an operand before it is
// quantized) and "HALO: Hadamard-Assisted Lower-Precision Optimization for LLMs" (Approach:
// tensor-wise quantization after the rotation; Limitations: round-to-nearest).
//
// Numerics, identical to the reference definition of the library:
//   t = Sylvester FWHT of each k-block, stages h = 1, 2, 4, ..., k/2 (index bit 0 first),
//       every add / sub an fp32 round-to-nearest-even op (explicit __fadd_rn / __fsub_rn);
//   y = fp32(t * fp32(1/sqrt(k)));   a = max |y| over the whole tensor;
//   INT8: q = clamp(rne(fp32(y * fp32(127/a))), -127, 127),  scale = fp32(a / 127)
//   FP8 : q = e4m3_rne_satfinite(fp32(y * fp32(448/a))),     scale = fp32(a / 448)
//   a == 0 -> scale 1 and zero codes; a not finite -> HQ_ERR_NONFINITE in the status word.
//
// Data movement (HBM-bound; log2(k) <= 8 adds per element against 3-5 bytes moved):
//   pass 1 rotates and reduces the absmax into one partial per CTA, pass 2 reduces the
//   partials, rotates again and writes the 1-byte codes.  Pass 2 walks the tensor in the
//   reverse order of pass 1 so its first reads hit what pass 1 left in L2.
//   * along the contiguous dimension (dim = 1): each thread owns 8 consecutive elements
//     (one 16-byte bf16 load or two fp32 loads), bits 0-2 of the in-block index live in
//     registers, bits 3.. across lanes (warp shuffles); 8 code bytes per thread, 256
//     contiguous bytes per warp.
//   * along the strided dimension (dim = 0): a CTA stages a 256-row x 128-byte tile in
//     shared memory (16-byte chunks XOR-swizzled by row group so the column gather is
//     conflict-free), each thread then owns 8 consecutive rows of 8 (bf16) or 4 (fp32)
//     columns; the codes are written transposed (rotated dimension innermost), 256
//     contiguous bytes per warp per column.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cfloat>
#include <cstdint>

namespace hq {

enum QuantMode : int { kModeAbsmax = 0, kModeInt8 = 1, kModeFp8 = 2 };

constexpr int kQuantThreads = 256;

// ------------------------------------------------------------------ element loads

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <bool STREAM>
__device__ __forceinline__ uint4 ld16(const void* p) {
  return STREAM ? __ldcs(reinterpret_cast<const uint4*>(p)) : __ldg(reinterpret_cast<const uint4*>(p));
}

template <typename SrcT, bool STREAM>
__device__ __forceinline__ void load8(const SrcT* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16, false>(const __nv_bfloat16* p, float (&v)[8]) {
  unpack_bf16x8(ld16<false>(p), v);
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16, true>(const __nv_bfloat16* p, float (&v)[8]) {
  unpack_bf16x8(ld16<true>(p), v);
}
template <>
__device__ __forceinline__ void load8<float, false>(const float* p, float (&v)[8]) {
  const uint4 a = ld16<false>(p), b = ld16<false>(p + 4);
  v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y); v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
  v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y); v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
}
template <>
__device__ __forceinline__ void load8<float, true>(const float* p, float (&v)[8]) {
  const uint4 a = ld16<true>(p), b = ld16<true>(p + 4);
  v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y); v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
  v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y); v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
}

// ------------------------------------------------------------------ butterflies

// Stages h = 1, 2, 4 over the 8 register-resident elements (in-block index bits 0..2).
__device__ __forceinline__ void butterfly_regs8(float (&v)[8]) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & h) continue;
      const float u = v[i], w = v[i + h];
      v[i] = __fadd_rn(u, w);
      v[i + h] = __fsub_rn(u, w);
    }
  }
}

// Stages h = 8, 16, ..., K/2: the partner element sits in the lane whose index differs in
// bit log2(h/8).  The lower-index holder keeps u + v, the upper one u - v.
template <int K, int NV>
__device__ __forceinline__ void butterfly_lanes(float (&v)[NV], int lane) {
#pragma unroll
  for (int m = 1; m < K / 8; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float p = __shfl_xor_sync(0xFFFFFFFFu, v[i], m);
      v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
    }
  }
}

// ------------------------------------------------------------------ quantizers

__device__ __forceinline__ uint32_t code_int8(float y, float inv) {
  int q = __float2int_rn(__fmul_rn(y, inv));
  q = max(-127, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}

__device__ __forceinline__ uint32_t code_fp8(float y, float inv) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fmul_rn(y, inv), __NV_SATFINITE, __NV_E4M3));
}

template <int MODE>
__device__ __forceinline__ uint2 codes8(const float (&y)[8], float inv, bool zero) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    b[i] = zero ? 0u : (MODE == kModeInt8 ? code_int8(y[i], inv) : code_fp8(y[i], inv));
  return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                    b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}

// ------------------------------------------------------------------ reductions

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, m));
  return v;
}

// Block-wide max; every thread gets the result.  `scratch` holds >= 32 floats.
__device__ __forceinline__ float block_max(float v, float* scratch) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[w] = v;
  __syncthreads();
  v = lane < static_cast<int>(blockDim.x >> 5) ? scratch[lane] : 0.0f;
  return warp_max(v);
}

// Pass-1 epilogue: one partial per CTA, +inf when any rotated value was not finite.
__device__ __forceinline__ void write_partial(float amax, bool bad, float* partials, float* scratch) {
  const float m = block_max(bad ? INFINITY : amax, scratch);
  if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

struct QuantParams {
  float inv;    // QMAX / a
  bool zero;    // a == 0: all codes zero
  bool abort;   // a not finite: nothing is written
};

// Pass-2 prologue: reduce the partials to a, publish the scale (CTA 0), set the status
// word on a non-finite tensor.
template <int MODE>
__device__ __forceinline__ QuantParams finish_absmax(const float* partials, int n_partials,
                                                     float* scale_out, float* scratch,
                                                     unsigned int* status) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < n_partials; i += blockDim.x) m = fmaxf(m, partials[i]);
  const float a = block_max(m, scratch);
  constexpr float QMAX = MODE == kModeInt8 ? 127.0f : 448.0f;
  QuantParams p;
  p.abort = !(a <= FLT_MAX);
  p.zero = (a == 0.0f);
  p.inv = (p.abort || p.zero) ? 0.0f : __fdiv_rn(QMAX, a);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (p.abort) {
      atomicCAS(status, 0u, 5u /* HQ_ERR_NONFINITE */);
      *scale_out = __int_as_float(0x7FC00000);
    } else {
      *scale_out = p.zero ? 1.0f : __fdiv_rn(a, QMAX);
    }
  }
  return p;
}

// ------------------------------------------------------------------ dim = 1 (contiguous)

// A warp-chunk is 32 lanes x 8 elements = 256 consecutive elements: a whole number of
// k-blocks for every k <= 256.  Each warp processes U consecutive warp-chunks per step.
constexpr int kRowsUnroll = 4;

template <typename SrcT, int K, int MODE>
__global__ void __launch_bounds__(kQuantThreads)
fwhtq_rows_kernel(const SrcT* __restrict__ src, int64_t n_chunks8, uint8_t* __restrict__ codes,
                  float* __restrict__ partials, int n_partials, float* __restrict__ scale_out,
                  unsigned int* __restrict__ status) {
  static_assert(K >= 16 && K <= 256 && (K & (K - 1)) == 0, "k must be a power of two in [16,256]");
  constexpr int U = kRowsUnroll;
  constexpr bool QUANT = MODE != kModeAbsmax;
  __shared__ float scratch[32];
  const int lane = threadIdx.x & 31;
  const float c = __frsqrt_rn(static_cast<float>(K));

  QuantParams qp{0.0f, false, false};
  if (QUANT) {
    qp = finish_absmax<MODE>(partials, n_partials, scale_out, scratch, status);
    if (qp.abort) return;
  }

  const int64_t warps_per_cta = kQuantThreads / 32;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * warps_per_cta + (threadIdx.x >> 5);
  const int64_t tw = static_cast<int64_t>(gridDim.x) * warps_per_cta;
  const int64_t n_wchunks = (n_chunks8 + 31) / 32;
  const int64_t n_groups = (n_wchunks + U - 1) / U;

  float amax = 0.0f;
  bool bad = false;
  if (gw < n_groups) {
    const int64_t last = gw + tw * ((n_groups - 1 - gw) / tw);
    // pass 1 walks forward, pass 2 backward (L2 reuse of the tail pass 1 read last)
    for (int64_t g = QUANT ? last : gw; QUANT ? g >= 0 : g < n_groups; g += QUANT ? -tw : tw) {
      float v[U][8];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t ch = (g * U + u) * 32 + lane;
        if (ch < n_chunks8) {
          load8<SrcT, QUANT>(src + ch * 8, v[u]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[u][i] = 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        butterfly_regs8(v[u]);
        butterfly_lanes<K, 8>(v[u], lane);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = __fmul_rn(v[u][i], c);
      }
      if (!QUANT) {
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float ay = fabsf(v[u][i]);
            bad |= !(ay <= FLT_MAX);
            amax = fmaxf(amax, ay);
          }
      } else {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int64_t ch = (g * U + u) * 32 + lane;
          if (ch < n_chunks8)
            __stcs(reinterpret_cast<uint2*>(codes + ch * 8), codes8<MODE>(v[u], qp.inv, qp.zero));
        }
      }
    }
  }
  if (!QUANT) write_partial(amax, bad, partials, scratch);
}

// ------------------------------------------------------------------ dim = 0 (strided)

constexpr int kColsTileRows = 256;   // rows per tile: 32 lanes x 8 registers
constexpr int kColsTileBytes = 128;  // bytes of each source row per tile (8 x 16-byte chunks)

template <typename SrcT, int K, int MODE>
__global__ void __launch_bounds__(kQuantThreads)
fwhtq_cols_kernel(const SrcT* __restrict__ src, int64_t rows, int64_t cols,
                  uint8_t* __restrict__ codes, float* __restrict__ partials, int n_partials,
                  float* __restrict__ scale_out, unsigned int* __restrict__ status) {
  static_assert(K >= 16 && K <= 256 && (K & (K - 1)) == 0, "k must be a power of two in [16,256]");
  constexpr bool QUANT = MODE != kModeAbsmax;
  constexpr int CPC = 16 / static_cast<int>(sizeof(SrcT));  // columns per 16-byte chunk
  constexpr int TCOLS = 8 * CPC;                            // columns per tile
  __shared__ __align__(16) uint4 tile[kColsTileRows][8];
  __shared__ float scratch[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float c = __frsqrt_rn(static_cast<float>(K));

  QuantParams qp{0.0f, false, false};
  if (QUANT) {
    qp = finish_absmax<MODE>(partials, n_partials, scale_out, scratch, status);
    if (qp.abort) return;
  }

  const int64_t n_rt = (rows + kColsTileRows - 1) / kColsTileRows;
  const int64_t n_ct = (cols + TCOLS - 1) / TCOLS;
  const int64_t n_tiles = n_rt * n_ct;
  float amax = 0.0f;
  bool bad = false;

  if (static_cast<int64_t>(blockIdx.x) < n_tiles) {
    const int64_t G = gridDim.x;
    const int64_t b = blockIdx.x;
    const int64_t last = b + G * ((n_tiles - 1 - b) / G);
    for (int64_t t = QUANT ? last : b; QUANT ? t >= 0 : t < n_tiles; t += QUANT ? -G : G) {
      const int64_t r0 = (t / n_ct) * kColsTileRows;
      const int64_t c0 = (t % n_ct) * TCOLS;
      __syncthreads();  // previous tile's gather is done before the tile is overwritten
      {
        const int ch = threadIdx.x & 7;
#pragma unroll
        for (int j = 0; j < kColsTileRows * 8 / kQuantThreads; ++j) {
          const int r = (threadIdx.x >> 3) + 32 * j;
          const int64_t gr = r0 + r, gc = c0 + ch * CPC;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (gr < rows && gc < cols) val = ld16<QUANT>(src + gr * cols + gc);
          tile[r][ch ^ ((r >> 3) & 7)] = val;
        }
      }
      __syncthreads();
      // thread (warp w, lane l): rows 8l..8l+7 of the w-th 16-byte column chunk
      float v[8][CPC];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 raw = tile[8 * lane + i][warp ^ (lane & 7)];
        if constexpr (CPC == 8) {
          float t8[8];
          unpack_bf16x8(raw, t8);
#pragma unroll
          for (int j = 0; j < CPC; ++j) v[i][j] = t8[j];
        } else {
          v[i][0] = __uint_as_float(raw.x); v[i][1] = __uint_as_float(raw.y);
          v[i][2] = __uint_as_float(raw.z); v[i][3] = __uint_as_float(raw.w);
        }
      }
      // register stages over the row index (bits 0..2), per column
#pragma unroll
      for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (i & h) continue;
#pragma unroll
          for (int j = 0; j < CPC; ++j) {
            const float u = v[i][j], w = v[i + h][j];
            v[i][j] = __fadd_rn(u, w);
            v[i + h][j] = __fsub_rn(u, w);
          }
        }
      }
      // lane stages over row-index bits 3..log2(K)-1
#pragma unroll
      for (int m = 1; m < K / 8; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < CPC; ++j) {
            const float p = __shfl_xor_sync(0xFFFFFFFFu, v[i][j], m);
            v[i][j] = upper ? __fsub_rn(p, v[i][j]) : __fadd_rn(v[i][j], p);
          }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < CPC; ++j) v[i][j] = __fmul_rn(v[i][j], c);

      if (!QUANT) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < CPC; ++j) {
            const float ay = fabsf(v[i][j]);
            bad |= !(ay <= FLT_MAX);
            amax = fmaxf(amax, ay);
          }
      } else {
        const int64_t row = r0 + 8 * lane;
        if (row < rows) {
#pragma unroll
          for (int j = 0; j < CPC; ++j) {
            const int64_t col = c0 + warp * CPC + j;
            if (col < cols) {
              float y8[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) y8[i] = v[i][j];
              __stcs(reinterpret_cast<uint2*>(codes + col * rows + row), codes8<MODE>(y8, qp.inv, qp.zero));
            }
          }
        }
      }
    }
  }
  if (!QUANT) write_partial(amax, bad, partials, scratch);
}

}  // namespace hq
