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
//   partials, rotates again and writes the 1-byte codes.  Consecutive passes over the same
//   tensor walk it in opposite directions so each starts on what the previous left in L2.
//   * along the contiguous dimension (dim = 1, fwhtq_rows_kernel): each thread owns 32
//     consecutive elements (one warp step = 1024 elements), so in-block index bits 0..4 are
//     register bits; for k >= 64 the warp swaps its values through a 4 KB shared-memory slice
//     so that the remaining stages run in registers too (no shuffles); 32 code bytes per
//     thread.
//   * along the strided dimension (dim = 0, fwhtq_cols_bf16_kernel for bf16): a CTA stages
//     256-row x 64-column tiles in shared memory (cp.async, 3-tile ring); ldmatrix.trans gives
//     each thread 64 rows of one column.  The absmax, INT8 and FP8 passes use the exchange
//     layout (xrotate): position bits 6, 7 start in lane bits and are brought into registers by
//     swapping half of the registers with the partner lane; the codes are written transposed
//     (rotated dimension innermost) in 32-byte segments.
//     fp32 sources use a simpler shared-memory tile kernel (fwhtq_cols_f32_kernel).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp6.h>
#include <cuda_fp4.h>
#include "sm100_ptx.cuh"
#include <cfloat>
#include <cstdint>
#include <type_traits>

namespace hq {

// kModeLowp: the FP6 / FP4 minifloats, the format (2 = e3m2, 3 = e2m3, 4 = e2m1, as the
// library's format enum) passed at run time as `lp_fmt`.
enum QuantMode : int { kModeAbsmax = 0, kModeInt8 = 1, kModeFp8 = 2, kModeLowp = 3 };

// Largest finite value of a minifloat format (the QMAX its codes are scaled to).
__device__ __forceinline__ float lowp_max(int lp_fmt) { return lp_fmt == 2 ? 28.0f : lp_fmt == 3 ? 7.5f : 6.0f; }

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

// ------------------------------------------------------------------ quantizers

__device__ __forceinline__ uint32_t code_int8(float y, float inv) {
  int q = __float2int_rn(__fmul_rn(y, inv));
  q = max(-127, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}

__device__ __forceinline__ uint32_t code_fp8(float y, float inv) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fmul_rn(y, inv), __NV_SATFINITE, __NV_E4M3));
}

// One minifloat code (nearest-even, saturating), value in the low bits of the byte.
__device__ __forceinline__ uint32_t code_lowp_z(float z, int lp_fmt) {
  if (lp_fmt == 4) return static_cast<uint32_t>(__nv_cvt_float_to_fp4(z, __NV_E2M1, cudaRoundNearest)) & 0xFu;
  return static_cast<uint32_t>(__nv_cvt_float_to_fp6(z, lp_fmt == 2 ? __NV_E3M2 : __NV_E2M3, cudaRoundNearest));
}

template <int MODE>
__device__ __forceinline__ uint2 codes8(const float (&y)[8], float inv, bool zero, int lp_fmt = 0) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    b[i] = zero ? 0u
                : (MODE == kModeInt8 ? code_int8(y[i], inv)
                   : MODE == kModeFp8 ? code_fp8(y[i], inv)
                                      : code_lowp_z(__fmul_rn(y[i], inv), lp_fmt));
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
// CG: the partials were written by other CTAs of the same launch (read through L2, past L1).
template <int MODE, bool CG = false>
__device__ __forceinline__ QuantParams finish_absmax(const float* partials, int n_partials,
                                                     float* scale_out, float* scratch,
                                                     unsigned int* status, int lp_fmt = 0) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < n_partials; i += blockDim.x) m = fmaxf(m, CG ? __ldcg(partials + i) : partials[i]);
  const float a = block_max(m, scratch);
  const float QMAX = MODE == kModeInt8 ? 127.0f : MODE == kModeFp8 ? 448.0f : lowp_max(lp_fmt);
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

// ------------------------------------------------------------------ packed-fp32 helpers

// Every helper is one fp32 round-to-nearest-even op per lane (f32x2 on sm_100), so results
// are bit-identical to the scalar __fadd_rn / __fsub_rn / __fmul_rn sequence.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);  // a - b, one rounding
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// Butterfly stages h = 1, 2, ..., H/2 over NV float2 registers holding 2*NV consecutive
// in-block positions (register index = position).  h = 1 pairs the halves of one float2.
template <int H, int NV>
__device__ __forceinline__ void stages_low(float2 (&v)[NV]) {
  if constexpr (H >= 2) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float a = v[i].x, b = v[i].y;
      v[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
  }
#pragma unroll
  for (int h2 = 1; h2 < H / 2; h2 <<= 1) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      if (i & h2) continue;
      const float2 a = v[i], b = v[i + h2];
      v[i] = add2(a, b);
      v[i + h2] = sub2(a, b);
    }
  }
}

// Stages whose partner lives in another lane (xor mask m): the lower holder keeps a + b, the
// upper one b' - a' = fma(-1, own, partner), a single rounding either way.
template <int NV>
__device__ __forceinline__ void stage_lanes(float2 (&v)[NV], int m, int lane) {
  const float sg = (lane & m) ? -1.0f : 1.0f;
  const float2 s2 = make_float2(sg, sg);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float2 p;
    p.x = __shfl_xor_sync(0xFFFFFFFFu, v[i].x, m);
    p.y = __shfl_xor_sync(0xFFFFFFFFu, v[i].y, m);
    v[i] = __ffma2_rn(s2, v[i], p);
  }
}

// max over |x| that turns any NaN into NaN (three-input max on sm_100).
__device__ __forceinline__ float absmax3(float m, float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m), "f"(fabsf(a)), "f"(fabsf(b)));
  return r;
}

// Partial of pass 1 from a per-thread max of the *unnormalised* |t|: the normalisation is
// a positive scaling, and fp32 rounding is monotone, so max|fp32(t*c)| = fp32(max|t| * c).
__device__ __forceinline__ void write_partial_unnormalised(float amax_t, float c, float* partials,
                                                           float* scratch) {
  const float m = block_max(amax_t != amax_t ? INFINITY : amax_t, scratch);
  if (threadIdx.x == 0) partials[blockIdx.x] = __fmul_rn(m, c);
}

// Codes of 4 consecutive elements packed little-endian into one word.
template <int MODE>
__device__ __forceinline__ uint32_t codes4(float2 z0, float2 z1) {
  if constexpr (MODE == kModeInt8) {
    // z + 1.5*2^23 rounds to an integer with ties to even (|z| <= 127.00001 < 2^22); the low
    // byte of the sum's bit pattern is that integer in two's complement.  |z| <= 127 after
    // rounding because |y| <= a and inv = fp32(127/a), so no clamp is needed.  The add is the
    // scalar __fadd_rn, which is never contracted with the multiply that produced z: a fused
    // multiply-add would round y*inv only once and flip codes whose product lies within an
    // ulp of a half-integer.
    constexpr float mg = 12582912.0f;
    const uint32_t b0 = __float_as_uint(__fadd_rn(z0.x, mg)), b1 = __float_as_uint(__fadd_rn(z0.y, mg));
    const uint32_t b2 = __float_as_uint(__fadd_rn(z1.x, mg)), b3 = __float_as_uint(__fadd_rn(z1.y, mg));
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
  } else {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(z0, __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(z1, __NV_SATFINITE, __NV_E4M3);
    return lo | (hi << 16);
  }
}

// Scaling of a rotated value t to the code grid.  The definition is z = fp32(fp32(t * c) * inv).
// When c = 1/sqrt(k) is a power of two (k = 16, 64, 256) and inv <= 2^100 this equals
// fp32(t * ci) with ci = c * inv (exact): if t * c is a normal number it is exact, so one
// rounding of t * c * inv remains either way; otherwise |z| <= 2^-126 * 2^100 under both forms,
// which is the zero code for INT8 and e4m3 alike (with the sign of t).
struct CodeScale {
  float2 c2, inv2, ci2;
  bool one_mul;
};

template <int K>
__device__ __forceinline__ CodeScale code_scale(float c, float inv) {
  CodeScale s;
  s.c2 = make_float2(c, c);
  s.inv2 = make_float2(inv, inv);
  const float ci = __fmul_rn(c, inv);
  s.ci2 = make_float2(ci, ci);
  s.one_mul = (K == 16 || K == 64 || K == 256) && inv <= 0x1p100f;
  return s;
}

// Codes of 4 consecutive rotated values (t0.x, t0.y, t1.x, t1.y) at the scale of cs, in its
// one-multiply form (ONE_MUL, valid when cs.one_mul) or its two-multiply form.
template <int MODE, bool ONE_MUL>
__device__ __forceinline__ uint32_t scaled_codes4(float2 t0, float2 t1, const CodeScale& cs, int lp_fmt);

// Codes of 4 consecutive elements for any mode (the minifloats' format at run time).
template <int MODE>
__device__ __forceinline__ uint32_t codes4x(float2 z0, float2 z1, int lp_fmt) {
  if constexpr (MODE != kModeLowp) {
    return codes4<MODE>(z0, z1);
  } else {
    if (lp_fmt == 4) {
      // two codes per byte from the conversion, one per byte in the layout
      const uint32_t a = __nv_cvt_float2_to_fp4x2(z0, __NV_E2M1, cudaRoundNearest);
      const uint32_t b = __nv_cvt_float2_to_fp4x2(z1, __NV_E2M1, cudaRoundNearest);
      return (a & 0xFu) | ((a & 0xF0u) << 4) | ((b & 0xFu) << 16) | ((b & 0xF0u) << 20);
    }
    const __nv_fp6_interpretation_t f = lp_fmt == 2 ? __NV_E3M2 : __NV_E2M3;
    const uint32_t lo = __nv_cvt_float2_to_fp6x2(z0, f, cudaRoundNearest);
    const uint32_t hi = __nv_cvt_float2_to_fp6x2(z1, f, cudaRoundNearest);
    return (lo & 0xFFFFu) | (hi << 16);
  }
}

template <int MODE, bool ONE_MUL>
__device__ __forceinline__ uint32_t scaled_codes4(float2 t0, float2 t1, const CodeScale& cs, int lp_fmt) {
  return ONE_MUL ? codes4x<MODE>(mul2(t0, cs.ci2), mul2(t1, cs.ci2), lp_fmt)
                 : codes4x<MODE>(mul2(mul2(t0, cs.c2), cs.inv2), mul2(mul2(t1, cs.c2), cs.inv2), lp_fmt);
}

// Tensor-core operand layout of the minifloat codes: each group of 16 consecutive codes along
// the rotated dimension fills one 16-byte chunk, packed LSB-first (code i in bits
// [b*i, b*i + b), b = 6 or 4) from byte 0, the rest of the chunk zero; kind::f8f6f4 reads FP6 /
// FP4 operands from shared memory in this form.

// Codes of 4 consecutive elements (one per byte, low bits) compressed to 24 (FP6) or 16 (FP4)
// bits, code 0 lowest.
__device__ __forceinline__ uint32_t lowp_compress4(uint32_t w, int lp_fmt) {
  if (lp_fmt == 4) return (w & 0xFu) | ((w >> 4) & 0xF0u) | ((w >> 8) & 0xF00u) | ((w >> 12) & 0xF000u);
  return (w & 0x3Fu) | ((w >> 2) & 0xFC0u) | ((w >> 4) & 0x3F000u) | ((w >> 6) & 0xFC0000u);
}

// One 16-byte chunk from the compressed codes of 4 consecutive 4-element pieces.
__device__ __forceinline__ uint4 lowp_chunk(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3, int lp_fmt) {
  if (lp_fmt == 4) return make_uint4(p0 | (p1 << 16), p2 | (p3 << 16), 0u, 0u);
  return make_uint4(p0 | (p1 << 24), (p1 >> 8) | (p2 << 16), (p2 >> 16) | (p3 << 8), 0u);
}

// 16 codes (one per byte in w0..w3) -> their chunk.
__device__ __forceinline__ uint4 lowp_pack16(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, int lp_fmt) {
  return lowp_chunk(lowp_compress4(w0, lp_fmt), lowp_compress4(w1, lp_fmt), lowp_compress4(w2, lp_fmt),
                    lowp_compress4(w3, lp_fmt), lp_fmt);
}

// ------------------------------------------------------------------ sign flags

// Randomized variant (a sign diagonal D before the blocks, t = H_k D x): `neg` holds one byte
// per position of the rotated dimension, bit 0 set negating that position.  The flip is an
// exact change of the source's sign bit before the butterflies, applied as an XOR mask to the
// raw words.

// Masks for 16 consecutive bf16 positions held as 8 bf16x2 words (word j: positions 2j in the
// low half, 2j + 1 in the high half); f = the 16 flag bytes.
__device__ __forceinline__ void sign_masks_bf16x16(uint4 f, uint32_t (&m)[8]) {
  const uint32_t w[4] = {f.x & 0x01010101u, f.y & 0x01010101u, f.z & 0x01010101u, f.w & 0x01010101u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[2 * i] = __byte_perm(w[i], 0u, 0x1404) << 7;      // flag bytes 0, 1 -> bits 15, 31
    m[2 * i + 1] = __byte_perm(w[i], 0u, 0x3424) << 7;  // flag bytes 2, 3 -> bits 15, 31
  }
}

// Masks for 4 consecutive fp32 positions (one word each) from 4 flag bytes.
__device__ __forceinline__ void sign_masks_f32x4(uint32_t f, uint32_t (&m)[4]) {
  m[0] = (f << 31) & 0x80000000u;
  m[1] = (f << 23) & 0x80000000u;
  m[2] = (f << 15) & 0x80000000u;
  m[3] = (f << 7) & 0x80000000u;
}

// ------------------------------------------------------------------ dim = 1 (contiguous)

// Each thread owns 32 consecutive elements (one warp step = 1024 elements), so in-block index
// bits 0..4 are register bits.  For k >= 64 the warp exchanges its 1024 values through a
// 4 KB shared-memory slice so that each thread then holds index bits {0, 1, 5, 6, 7}
// (bits 2, 3, 4 and the 256-element group become lane bits) and the stages for bits 5.. run
// in registers too: no shuffles.  The slice is XOR-swizzled at 16-byte granularity,
// chunk c -> c ^ ((c >> 3) & 7), which makes both the write and the read conflict-free.
constexpr int kRowsPerThread = 32;
constexpr int kRowsWarpElems = 32 * kRowsPerThread;

template <typename SrcT>
struct RowsRaw {
  static constexpr int W = 16 * static_cast<int>(sizeof(SrcT)) / 2;  // 32-bit words per thread
};

template <bool LAST_USE>
__device__ __forceinline__ void ld_32B(const void* p, uint32_t* r) {
  if (LAST_USE)
    asm volatile("ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
  else
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}

// (the L2 eviction hint exists only for the 32-byte form)
template <bool LAST_USE>
__device__ __forceinline__ void ld_16B(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "l"(p));
}

// Load a thread's 32 elements starting at element `e` (two halves of 16; a half past the end
// of the tensor reads as zeros).  WIDE: 32-byte loads (source 32-byte aligned).
template <typename SrcT, bool WIDE, bool LAST_USE>
__device__ __forceinline__ void load_rows32(const SrcT* src, int64_t n, int64_t e,
                                            uint32_t (&raw)[RowsRaw<SrcT>::W]) {
  constexpr int HW = RowsRaw<SrcT>::W / 2;  // words per half (8 for bf16, 16 for fp32)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t eh = e + 16 * h;
    if (eh < n) {
      const char* p = reinterpret_cast<const char*>(src + eh);
#pragma unroll
      for (int q = 0; q < HW; q += (WIDE ? 8 : 4)) {
        if (WIDE) ld_32B<LAST_USE>(p + 4 * q, raw + h * HW + q);
        else ld_16B<LAST_USE>(p + 4 * q, raw + h * HW + q);
      }
    } else {
#pragma unroll
      for (int q = 0; q < HW; ++q) raw[h * HW + q] = 0u;
    }
  }
}

template <typename SrcT>
__device__ __forceinline__ void unpack_rows32(const uint32_t (&raw)[RowsRaw<SrcT>::W], float2 (&v)[16]) {
  if constexpr (sizeof(SrcT) == 2) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      v[i] = make_float2(__uint_as_float(raw[i] << 16), __uint_as_float(raw[i] & 0xFFFF0000u));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = make_float2(__uint_as_float(raw[2 * i]), __uint_as_float(raw[2 * i + 1]));
  }
}

// Warp-level exchange: before, thread t holds elements 32t + r (r = register index 0..31);
// after, thread t holds elements 4*(t&7) + (r&3) + 32*(r>>2) + 256*(t>>3).
__device__ __forceinline__ void exchange_rows(float2 (&v)[16], float4* slice, int lane) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    slice[8 * lane + (j ^ (lane & 7))] = make_float4(v[2 * j].x, v[2 * j].y, v[2 * j + 1].x, v[2 * j + 1].y);
  __syncwarp();
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const float4 f = slice[(((lane & 7) ^ b) + 8 * b) + 64 * (lane >> 3)];
    v[2 * b] = make_float2(f.x, f.y);
    v[2 * b + 1] = make_float2(f.z, f.w);
  }
  __syncwarp();
}

template <typename SrcT, int K, int MODE, bool WIDE, bool SIGNED>
__global__ void __launch_bounds__(kQuantThreads, sizeof(SrcT) == 2 ? 3 : 1)
fwhtq_rows_kernel(const SrcT* __restrict__ src, int64_t n, uint8_t* __restrict__ codes,
                  float* __restrict__ partials, int n_partials, float* __restrict__ scale_out,
                  unsigned int* __restrict__ status, int reverse, const uint8_t* __restrict__ neg,
                  int64_t cols, int lp_fmt) {
  // programmatic dependent launch: nothing is read or written before the previous grid in the
  // stream has completed; the next grid may be scheduled from here on
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  static_assert(K >= 16 && K <= 256 && (K & (K - 1)) == 0, "k must be a power of two in [16,256]");
  constexpr bool QUANT = MODE != kModeAbsmax;
  constexpr bool EXCH = K >= 64;
  constexpr int RW = RowsRaw<SrcT>::W;
  __shared__ __align__(16) float4 xch[EXCH ? kQuantThreads * 8 : 1];
  __shared__ float scratch[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float c = __frsqrt_rn(static_cast<float>(K));

  QuantParams qp{0.0f, false, false};
  if (QUANT) {
    qp = finish_absmax<MODE>(partials, n_partials, scale_out, scratch, status, lp_fmt);
    if (qp.abort) return;
  }
  const CodeScale cs = code_scale<K>(c, qp.inv);

  const int64_t wpc = kQuantThreads / 32;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * wpc + warp;
  const int64_t tw = static_cast<int64_t>(gridDim.x) * wpc;
  const int64_t n_units = (n + kRowsWarpElems - 1) / kRowsWarpElems;
  float amax = 0.0f;
  if (gw < n_units) {
    // alternate passes over a tensor walk it in opposite directions, so each pass starts on
    // what the previous one left in L2
    const int64_t last = gw + tw * ((n_units - 1 - gw) / tw);
    const int64_t first = reverse ? last : gw;
    const int64_t step = reverse ? -tw : tw;
    // the loads of unit u + step go out while u is computed (one unit of registers, so that
    // three CTAs fit per SM)
    auto valid = [&](int64_t u) { return reverse ? u >= 0 : u < n_units; };
    // column of this thread's first element in the current unit (sign flags only): tracked
    // incrementally, the units of a thread being `step` apart
    int64_t col = 0, dcol = 0;
    if constexpr (SIGNED) {
      col = (first * kRowsWarpElems + 32 * lane) % cols;
      dcol = ((step * kRowsWarpElems) % cols + cols) % cols;
    }
    auto body = [&](uint32_t (&raw)[RW], int64_t u) {
      if constexpr (SIGNED) {
        // each 16-element half lies in one row (cols is a multiple of 16)
        const int64_t c1 = col + 16 >= cols ? col + 16 - cols : col + 16;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 f = __ldg(reinterpret_cast<const uint4*>(neg + (h == 0 ? col : c1)));
          if constexpr (sizeof(SrcT) == 2) {
            uint32_t m[8];
            sign_masks_bf16x16(f, m);
#pragma unroll
            for (int j = 0; j < 8; ++j) raw[8 * h + j] ^= m[j];
          } else {
            const uint32_t fw[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t m[4];
              sign_masks_f32x4(fw[q], m);
#pragma unroll
              for (int j = 0; j < 4; ++j) raw[16 * h + 4 * q + j] ^= m[j];
            }
          }
        }
        col = col + dcol >= cols ? col + dcol - cols : col + dcol;
      }
      float2 v[16];
      unpack_rows32<SrcT>(raw, v);
      const int64_t nu = u + step;
      if (valid(nu)) load_rows32<SrcT, WIDE, QUANT>(src, n, nu * kRowsWarpElems + 32 * lane, raw);
      stages_low<(K < 32 ? K : 32), 16>(v);
      if constexpr (EXCH) {
        exchange_rows(v, xch + warp * 256, lane);
        // index bits 5.. are register-index bits 2.. = float2-index bits 1..
#pragma unroll
        for (int h2 = 2; h2 < K / 16; h2 <<= 1) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (i & h2) continue;
            const float2 a = v[i], b = v[i + h2];
            v[i] = add2(a, b);
            v[i + h2] = sub2(a, b);
          }
        }
      }
      if constexpr (!QUANT) {
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = absmax3(amax, v[i].x, v[i].y);
      } else {
        const int64_t ub = u * kRowsWarpElems;
        uint32_t w[8];
        if (cs.one_mul) {
#pragma unroll
          for (int j = 0; j < 8; ++j) w[j] = codes4x<MODE>(mul2(v[2 * j], cs.ci2), mul2(v[2 * j + 1], cs.ci2), lp_fmt);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            w[j] = codes4x<MODE>(mul2(mul2(v[2 * j], cs.c2), cs.inv2), mul2(mul2(v[2 * j + 1], cs.c2), cs.inv2), lp_fmt);
        }
        if (qp.zero) {
#pragma unroll
          for (int j = 0; j < 8; ++j) w[j] = 0u;
        }
        const bool full = ub + kRowsWarpElems <= n;  // all but a ragged last unit
        if constexpr (MODE == kModeLowp) {
          // minifloats: 16-code groups packed into 16-byte chunks (n is a multiple of 16)
          if constexpr (!EXCH) {
            const int64_t e = ub + 32 * lane;
            if (full || e < n) *reinterpret_cast<uint4*>(codes + e) = lowp_pack16(w[0], w[1], w[2], w[3], lp_fmt);
            if (full || e + 16 < n)
              *reinterpret_cast<uint4*>(codes + e + 16) = lowp_pack16(w[4], w[5], w[6], w[7], lp_fmt);
          } else {
            // word b of lane l holds codes e0 + 32b + 0..3 with e0 = 4 (l & 7) + ...: a group's
            // four words sit in lanes 4g .. 4g + 3, gathered into the first of them
            const int64_t e0 = ub + 256 * (lane >> 3) + 4 * (lane & 7);
#pragma unroll
            for (int b = 0; b < 8; ++b) {
              const uint32_t p = lowp_compress4(w[b], lp_fmt);
              const uint32_t p1 = __shfl_down_sync(0xFFFFFFFFu, p, 1);
              const uint32_t p2 = __shfl_down_sync(0xFFFFFFFFu, p, 2);
              const uint32_t p3 = __shfl_down_sync(0xFFFFFFFFu, p, 3);
              if ((lane & 3) == 0 && (full || e0 + 32 * b < n))
                *reinterpret_cast<uint4*>(codes + e0 + 32 * b) = lowp_chunk(p, p1, p2, p3, lp_fmt);
            }
          }
        } else if constexpr (!EXCH) {
          const int64_t e = ub + 32 * lane;
          if (full || e < n) *reinterpret_cast<uint4*>(codes + e) = make_uint4(w[0], w[1], w[2], w[3]);
          if (full || e + 16 < n) *reinterpret_cast<uint4*>(codes + e + 16) = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
          const int64_t e0 = ub + 256 * (lane >> 3) + 4 * (lane & 7);
          if (full) {
#pragma unroll
            for (int b = 0; b < 8; ++b) *reinterpret_cast<uint32_t*>(codes + e0 + 32 * b) = w[b];
          } else {
#pragma unroll
            for (int b = 0; b < 8; ++b)
              if (e0 + 32 * b < n) *reinterpret_cast<uint32_t*>(codes + e0 + 32 * b) = w[b];
          }
        }
      }
    };
    uint32_t raw[RW];
    load_rows32<SrcT, WIDE, QUANT>(src, n, first * kRowsWarpElems + 32 * lane, raw);
    for (int64_t u = first; valid(u); u += step) body(raw, u);
  }
  if (!QUANT) write_partial_unnormalised(amax, c, partials, scratch);
}

// max(m, fl(|a| + |b|), fl(|c| + |d|)), NaN-propagating.  For a butterfly pair (u, v) the two
// outputs satisfy max(|fl(u + v)|, |fl(u - v)|) = fl(|u| + |v|) (one of them is the sum of the
// magnitudes, the other the difference, and rounding is monotone and sign-symmetric), so the
// absmax pass never forms the last stage's outputs.
__device__ __forceinline__ float max_abs_sums(float m, float a, float b, float c, float d) {
  return absmax3(m, __fadd_rn(fabsf(a), fabsf(b)), __fadd_rn(fabsf(c), fabsf(d)));
}

// Running maxima of the absmax pass: eight independent chains, so consecutive max
// instructions do not wait on each other.
constexpr int kAcc = 8;

__device__ __forceinline__ void st_global_32B(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                              uint32_t f, uint32_t g, uint32_t h) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d),
               "r"(e), "r"(f), "r"(g), "r"(h)
               : "memory");
}

// ------------------------------------------------------------------ exchange layout
//
// The absmax, INT8 and FP8 passes hold a thread's 64 values of one k-block slice as v[j].x =
// in-block position j and v[j].y = position j + 32 (j = position bits 0..4, the float2 half =
// bit 5), so every butterfly stage except the one on bit 5 pairs two different float2
// registers and runs as packed f32x2 operations.  For k = 128 / 256 the position bits 6 / 6, 7
// start in lane bits; they are brought into registers by exchanging half of the registers with
// the partner lane (one shuffle per two values instead of one per value):
//   before the exchange, register bit r holds position bit Q and lane bit l holds bit P; lane
//   l-value b keeps the registers with r-bit 0 and swaps those with r-bit 1 for the partner's.
//   Afterwards the lane bit holds Q and the register bit holds P.  For this to need no selects,
//   register bit r is stored "swizzled", holding Q XOR b before and P XOR b after the exchange
//   (the loads place the data so, from lane-dependent shared-memory addresses).
// A butterfly stage on a swizzled register bit pairs R0 (r-bit 0) and R1: with b = 0 they hold
// positions 0 and 1 of the pair, with b = 1 positions 1 and 0, so R0' = fma(s, R0, R1) and
// R1' = fma(-s, R1, R0) with s = +1 (b = 0) or -1 (b = 1) give u + v and u - v at the right
// places.  Each is one fp32 rounding of the exact sum or difference: bit-identical to the plain
// stage.
// Exchanged bits: k = 256: register bit 3 (position 3) with the lane bit of position 6 ("A"),
// register bit 4 (position 4) with the lane bit of position 7 ("B"); k = 128: register bit 4
// with lane bit A.  Afterwards a thread holds 8 (k = 256) or 16 (k = 128) consecutive
// positions per group of registers, and 4 / 2 lanes together hold 32 consecutive code bytes.

// Plain stage on register bit log2(H): pairs (v[i], v[i + H]).
template <int H>
__device__ __forceinline__ void xstage(float2 (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i & H) continue;
    const float2 a = v[i], b = v[i + H];
    v[i] = add2(a, b);
    v[i + H] = sub2(a, b);
  }
}

// Stage on a swizzled register bit (s2 = (s, s), ns2 = (-s, -s)).
template <int H>
__device__ __forceinline__ void xstage_sw(float2 (&v)[32], float2 s2, float2 ns2) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i & H) continue;
    const float2 a = v[i], b = v[i + H];
    v[i] = __ffma2_rn(s2, a, b);
    v[i + H] = __ffma2_rn(ns2, b, a);
  }
}

// Stage on position bit 5 (the two halves of every float2).
__device__ __forceinline__ void xstage_halves(float2 (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float a = v[i].x, b = v[i].y;
    v[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
}

// Registers with bit log2(H) set are swapped with lane ^ m's.
template <int H>
__device__ __forceinline__ void xexchange(float2 (&v)[32], int m) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (!(i & H)) continue;
    v[i].x = __shfl_xor_sync(0xFFFFFFFFu, v[i].x, m);
    v[i].y = __shfl_xor_sync(0xFFFFFFFFu, v[i].y, m);
  }
}

// Last stage folded into the running maxima (see max_abs_sums): pairs on register bit log2(H),
// or the two halves of every float2.
template <int H>
__device__ __forceinline__ void xfold(const float2 (&v)[32], float (&am)[kAcc]) {
  int n = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i & H) continue;
    am[n % kAcc] = max_abs_sums(am[n % kAcc], v[i].x, v[i + H].x, v[i].y, v[i + H].y);
    ++n;
  }
}
__device__ __forceinline__ void xfold_halves(const float2 (&v)[32], float (&am)[kAcc]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2)
    am[(i / 2) % kAcc] = max_abs_sums(am[(i / 2) % kAcc], v[i].x, v[i].y, v[i + 1].x, v[i + 1].y);
}

// Whole rotation of a thread's values in the exchange layout (stages in position-bit order
// 0, 1, ..., log2 K - 1).  ABSMAX: the last stage is folded into `am` instead.
template <int K, bool ABSMAX>
__device__ __forceinline__ void xrotate(float2 (&v)[32], float2 sA, float2 nsA, float2 sB, float2 nsB, int mA, int mB,
                                        float (&am)[kAcc]) {
  xstage<1>(v);
  xstage<2>(v);
  if constexpr (K == 16) {
    xstage<4>(v);
    if constexpr (ABSMAX) xfold<8>(v, am); else xstage<8>(v);
  } else if constexpr (K == 32) {
    xstage<4>(v);
    xstage<8>(v);
    if constexpr (ABSMAX) xfold<16>(v, am); else xstage<16>(v);
  } else if constexpr (K == 64) {
    xstage<4>(v);
    xstage<8>(v);
    xstage<16>(v);
    if constexpr (ABSMAX) xfold_halves(v, am); else xstage_halves(v);
  } else if constexpr (K == 128) {
    xstage<4>(v);
    xstage<8>(v);
    xstage_sw<16>(v, sA, nsA);
    xstage_halves(v);
    xexchange<16>(v, mA);
    if constexpr (ABSMAX) xfold<16>(v, am); else xstage_sw<16>(v, sA, nsA);
  } else {
    xstage<4>(v);
    xstage_sw<8>(v, sA, nsA);
    xstage_sw<16>(v, sB, nsB);
    xstage_halves(v);
    xexchange<8>(v, mA);
    xstage_sw<8>(v, sA, nsA);
    xexchange<16>(v, mB);
    if constexpr (ABSMAX) xfold<16>(v, am); else xstage_sw<16>(v, sB, nsB);
  }
}

// Code words of a thread's rotated values: wx[q] = codes of positions 4q .. 4q + 3 (the .x
// halves of v[4q .. 4q + 3]), wy[q] the same for the .y halves, little-endian.
template <int MODE, bool ONE_MUL>
__device__ __forceinline__ void xcodes_at(const float2 (&v)[32], const CodeScale& cs, bool zero, uint32_t (&wx)[8],
                                          uint32_t (&wy)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float2 z[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      z[i] = ONE_MUL ? mul2(v[4 * q + i], cs.ci2) : mul2(mul2(v[4 * q + i], cs.c2), cs.inv2);
    if constexpr (MODE == kModeInt8) {
      // z + 1.5 * 2^23: the low byte is rne(z) in two's complement (see codes4).  The add is
      // the scalar __fadd_rn: with a packed add the compiler fused it with the packed multiply
      // into one fused multiply-add, which rounds y * inv only once (a product 74.50000000019
      // whose fp32 rounding is the tie 74.5 then gave 75 instead of the even 74).
      constexpr float mg = 12582912.0f;
      uint32_t bx[4], by[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        bx[i] = __float_as_uint(__fadd_rn(z[i].x, mg));
        by[i] = __float_as_uint(__fadd_rn(z[i].y, mg));
      }
      wx[q] = __byte_perm(__byte_perm(bx[0], bx[1], 0x0040), __byte_perm(bx[2], bx[3], 0x0040), 0x5410);
      wy[q] = __byte_perm(__byte_perm(by[0], by[1], 0x0040), __byte_perm(by[2], by[3], 0x0040), 0x5410);
    } else {
      const uint32_t x01 = __nv_cvt_float2_to_fp8x2(make_float2(z[0].x, z[1].x), __NV_SATFINITE, __NV_E4M3);
      const uint32_t x23 = __nv_cvt_float2_to_fp8x2(make_float2(z[2].x, z[3].x), __NV_SATFINITE, __NV_E4M3);
      const uint32_t y01 = __nv_cvt_float2_to_fp8x2(make_float2(z[0].y, z[1].y), __NV_SATFINITE, __NV_E4M3);
      const uint32_t y23 = __nv_cvt_float2_to_fp8x2(make_float2(z[2].y, z[3].y), __NV_SATFINITE, __NV_E4M3);
      wx[q] = x01 | (x23 << 16);
      wy[q] = y01 | (y23 << 16);
    }
    if (zero) wx[q] = wy[q] = 0u;
  }
}

// The scale's one-multiply form is chosen once for all of the thread's values (a branch on a
// warp-uniform flag), so each value takes one multiply by fp32(c * inv) or two.
template <int MODE>
__device__ __forceinline__ void xcodes(const float2 (&v)[32], const CodeScale& cs, bool zero, uint32_t (&wx)[8],
                                       uint32_t (&wy)[8]) {
  if (cs.one_mul) xcodes_at<MODE, true>(v, cs, zero, wx, wy);
  else xcodes_at<MODE, false>(v, cs, zero, wx, wy);
}

__device__ __forceinline__ void st_global_8B(void* p, uint32_t a, uint32_t b) {
  asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_global_16B(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Stores of a thread's code words.  k <= 64: the thread's 64 codes are consecutive (x half,
// then y half) at pos0 relative to `base`.  k = 128 / 256: groups of 16 / 8 consecutive codes
// whose 32-byte segments are shared by the 2 / 4 lanes of the exchanged lane bits (A, B; p =
// the thread's value of them).  Those lanes first swap code words so that each ends with whole
// segments: register group g of lane p holds segment pieces of segment pair g ^ p (the swizzle),
// so in round r every lane sends its group r to lane p ^ r and receives pieces of its own
// segment pair p; the pieces are then put in address order (piece q comes from lane q, i.e.
// from round q ^ p) with two layers of selects.  Each lane then writes its segment pair
// (position bits 6, 7 = p; 5 = the half) as two 32-byte stores.  pos_of(h) gives the in-tile
// position of the thread's segment for half h; ok(pos) whether it lies inside the tensor.
__device__ __forceinline__ uint32_t sel(bool c, uint32_t a, uint32_t b) { return c ? a : b; }

// One 32-byte segment: a single 32-byte store when the address is 32-byte aligned (w32), else
// two 16-byte stores.
__device__ __forceinline__ void store_seg32(uint8_t* d, const uint32_t (&w)[8], bool w32) {
  if (w32) {
    st_global_32B(d, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
  } else {
    st_global_16B(d, w[0], w[1], w[2], w[3]);
    st_global_16B(d + 16, w[4], w[5], w[6], w[7]);
  }
}

template <int K, class Pos, class Ok>
__device__ __forceinline__ void xstore(uint8_t* base, const uint32_t (&wx)[8], const uint32_t (&wy)[8], int p, int mA,
                                       int mB, Pos pos_of, Ok ok, bool w32) {
  uint32_t o[2][8];
  if constexpr (K <= 64) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o[0][i] = wx[i];
      o[1][i] = wy[i];
    }
  } else if constexpr (K == 128) {
    // groups g = 0, 1 (4 words per half); round 1 swaps group 1 with lane ^ mA
    uint32_t s0[8], s1[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s0[i] = wx[i];
      s0[4 + i] = wy[i];
      s1[i] = __shfl_xor_sync(0xFFFFFFFFu, wx[4 + i], mA);
      s1[4 + i] = __shfl_xor_sync(0xFFFFFFFFu, wy[4 + i], mA);
    }
    const bool sw = p & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[0][i] = sel(sw, s1[i], s0[i]);
      o[0][4 + i] = sel(sw, s0[i], s1[i]);
      o[1][i] = sel(sw, s1[4 + i], s0[4 + i]);
      o[1][4 + i] = sel(sw, s0[4 + i], s1[4 + i]);
    }
  } else {
    // groups g = 0..3 (2 words per half); round r swaps group r with lane ^ (A if r & 1, B if r & 2)
    uint32_t sl[4][4];  // slot: x word 0, x word 1, y word 0, y word 1
    sl[0][0] = wx[0]; sl[0][1] = wx[1]; sl[0][2] = wy[0]; sl[0][3] = wy[1];
#pragma unroll
    for (int r = 1; r < 4; ++r) {
      const int m = ((r & 1) ? mA : 0) | ((r & 2) ? mB : 0);
      sl[r][0] = __shfl_xor_sync(0xFFFFFFFFu, wx[2 * r], m);
      sl[r][1] = __shfl_xor_sync(0xFFFFFFFFu, wx[2 * r + 1], m);
      sl[r][2] = __shfl_xor_sync(0xFFFFFFFFu, wy[2 * r], m);
      sl[r][3] = __shfl_xor_sync(0xFFFFFFFFu, wy[2 * r + 1], m);
    }
    // piece q of the segment = slot q ^ p: swap by bit 0 of p, then by bit 1
    const bool b0 = p & 1, b1 = p & 2;
    uint32_t t[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      t[0][i] = sel(b0, sl[1][i], sl[0][i]);
      t[1][i] = sel(b0, sl[0][i], sl[1][i]);
      t[2][i] = sel(b0, sl[3][i], sl[2][i]);
      t[3][i] = sel(b0, sl[2][i], sl[3][i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sl[0][i] = sel(b1, t[2][i], t[0][i]);
      sl[1][i] = sel(b1, t[3][i], t[1][i]);
      sl[2][i] = sel(b1, t[0][i], t[2][i]);
      sl[3][i] = sel(b1, t[1][i], t[3][i]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      o[0][2 * q] = sl[q][0];
      o[0][2 * q + 1] = sl[q][1];
      o[1][2 * q] = sl[q][2];
      o[1][2 * q + 1] = sl[q][3];
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t ps = pos_of(h);
    if (ok(ps)) store_seg32(base + ps, o[h], w32);
  }
}

// Sign masks of 8 consecutive bf16 positions (4 bf16x2 words) from their 8 flag bytes.
__device__ __forceinline__ void sign_masks_bf16x8(uint2 f, uint32_t (&m)[4]) {
  const uint32_t w[2] = {f.x & 0x01010101u, f.y & 0x01010101u};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    m[2 * i] = __byte_perm(w[i], 0u, 0x1404) << 7;
    m[2 * i + 1] = __byte_perm(w[i], 0u, 0x3424) << 7;
  }
}

// v[8q + 2i], v[8q + 2i + 1] from words i of chunk q: .x from the chunk's x-half words, .y from
// its y-half words.
__device__ __forceinline__ void xunpack(int q, const uint32_t (&wxq)[4], const uint32_t (&wyq)[4], float2 (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[8 * q + 2 * i] = make_float2(__uint_as_float(wxq[i] << 16), __uint_as_float(wyq[i] << 16));
    v[8 * q + 2 * i + 1] = make_float2(__uint_as_float(wxq[i] & 0xFFFF0000u), __uint_as_float(wyq[i] & 0xFFFF0000u));
  }
}

// ------------------------------------------------------------------ dim = 0, bf16 source

// A CTA tile is 256 rows x 64 bf16 columns (32 KB); a 3-tile ring in shared memory is filled
// by cp.async (zero-filled past the tensor's edge), two tiles ahead of the one computed.  Warp w owns the tile's 8 columns of 16-byte
// chunk w; ldmatrix.trans turns four 8x8 blocks at a time into column-major fragments so that
// thread t holds 64 consecutive rows (64*(t&3) + 0..63) of column 8w + t/4: in-block row bits
// 0..5 are register bits, bits 6 and 7 lane bits (shuffles only for k = 128, 256).  The
// codes of a thread are 64 contiguous bytes of the transposed output.
constexpr int kColsTileRows2 = 256;
constexpr int kColsTileCols2 = 64;
constexpr int kColsStages2 = 3;
constexpr size_t kColsSmemBytes2 = size_t(kColsStages2) * kColsTileRows2 * 128;  // 3 x 32 KB tiles

// 16-byte chunk swizzle of tile row rho: row bit 0 -> bit 0, row bits 6, 7 -> bits 1, 2, so
// the 8 rows one ldmatrix matrix reads (rows differing in bits 0, 6, 7) hit distinct banks.
__device__ __forceinline__ int cols_swz(int rho) { return (rho & 1) | ((rho >> 5) & 6); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

// Row and column block of a tile index t = tr * n_ct + tc that advances by a fixed step (either
// sign): one 64-bit division at the start, then an add with one carry per step (a 64-bit
// division per tile cost a few instructions per element in the strided kernel's integer work).
struct TileWalk {
  int64_t tr, tc, dr, dc, n_ct;
  __device__ __forceinline__ void init(int64_t t, int64_t step, int64_t nct) {
    n_ct = nct;
    tr = t / nct;
    tc = t - tr * nct;
    if (tc < 0) { tc += nct; --tr; }  // floor division for a t before the first tile
    dr = step / nct;
    dc = step - dr * nct;
    if (dc < 0) { dc += nct; --dr; }
  }
  __device__ __forceinline__ void advance() {
    tr += dr;
    tc += dc;
    if (tc >= n_ct) { tc -= n_ct; ++tr; }
  }
};

template <int K, int MODE, bool SIGNED>
__global__ void __launch_bounds__(kQuantThreads)
fwhtq_cols_bf16_kernel(const __nv_bfloat16* __restrict__ src, int64_t rows, int64_t cols,
                       uint8_t* __restrict__ codes, float* __restrict__ partials, int n_partials,
                       float* __restrict__ scale_out, unsigned int* __restrict__ status, int reverse,
                       const uint8_t* __restrict__ neg, int lp_fmt) {
  // programmatic dependent launch: nothing is read or written before the previous grid in the
  // stream has completed; the next grid may be scheduled from here on
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  static_assert(K >= 16 && K <= 256 && (K & (K - 1)) == 0, "k must be a power of two in [16,256]");
  constexpr bool QUANT = MODE != kModeAbsmax;
  extern __shared__ __align__(128) uint4 tiles[];  // [3][256 rows][8 chunks]
  __shared__ float scratch[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float c = __frsqrt_rn(static_cast<float>(K));

  QuantParams qp{0.0f, false, false};
  if (QUANT) {
    qp = finish_absmax<MODE>(partials, n_partials, scale_out, scratch, status, lp_fmt);
    if (qp.abort) return;
  }
  const CodeScale cs = code_scale<K>(c, qp.inv);

  const int64_t n_rt = (rows + kColsTileRows2 - 1) / kColsTileRows2;
  const int64_t n_ct = (cols + kColsTileCols2 - 1) / kColsTileCols2;
  const int64_t n_tiles = n_rt * n_ct;
  float amax = 0.0f;
  float am[kAcc];  // exchange layout: independent running maxima of the unnormalised |t|
#pragma unroll
  for (int j = 0; j < kAcc; ++j) am[j] = 0.0f;
  // 32-byte code stores when every segment address is 32-byte aligned (k >= 128: rows is a
  // multiple of 128)
  const bool w32 = (reinterpret_cast<uintptr_t>(codes) & 31u) == 0;

  // load tile (tr, tc): thread T copies 16-byte chunk (T & 7) of rows (T >> 3) + 32 j
  auto issue = [&](int buf, int64_t tr, int64_t tc) {
    const int64_t r0 = tr * kColsTileRows2, c0 = tc * kColsTileCols2;
    const int ch = threadIdx.x & 7;
    const int64_t gc = c0 + 8 * ch;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int rho = (threadIdx.x >> 3) + 32 * j;
      const int64_t gr = r0 + rho;
      const bool ok = gr < rows && gc < cols;
      const __nv_bfloat16* g = ok ? src + gr * cols + gc : src;
      cp_async16(ptx::smem_u32(&tiles[(buf * kColsTileRows2 + rho) * 8 + (ch ^ cols_swz(rho))]), g, ok ? 16u : 0u);
    }
    cp_async_commit();
  };

  const int64_t G = gridDim.x, b0 = blockIdx.x;
  if (b0 < n_tiles) {
    const int64_t last = b0 + G * ((n_tiles - 1 - b0) / G);
    const int64_t first = reverse ? last : b0;
    const int64_t step = reverse ? -G : G;
    auto valid = [&](int64_t t) { return reverse ? t >= 0 : t < n_tiles; };
    int buf = 0;
    TileWalk cur, ahead;  // tile t and tile t + 2 step
    cur.init(first, step, n_ct);
    ahead.init(first + 2 * step, step, n_ct);
    issue(0, cur.tr, cur.tc);
    if (valid(first + step)) {
      TileWalk next;
      next.init(first + step, step, n_ct);
      issue(1, next.tr, next.tc);
    }
    for (int64_t t = first; valid(t); t += step, cur.advance(), ahead.advance()) {
      // keep two tiles in flight; wait only for this tile's copies
      if (valid(t + 2 * step)) {
        issue(buf == 0 ? 2 : buf - 1, ahead.tr, ahead.tc);
        cp_async_wait<2>();
      } else if (valid(t + step)) {
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      if constexpr (MODE != kModeLowp) {
        // exchange layout (see xrotate): a thread receives rows of column 8 warp + lane / 4
        // whose position bits 6, 7 are its lane bits 0, 1; gather q of the x half reads 8-row
        // group (q ^ sw) of each 64-row quarter, the y half group 4 + (q ^ sw), with the swizzle
        // sw of the thread receiving the row this lane addresses (matrix row lane & 7 goes to
        // lane bits (lane & 7) >> 1)
        const int m = lane >> 3, qr = lane & 7;
        const int sw_addr = K == 256 ? (qr >> 1) : K == 128 ? 2 * ((qr >> 1) & 1) : 0;
        const int a = lane & 3;
        const int sw_own = K == 256 ? a : K == 128 ? 2 * (a & 1) : 0;
        float2 v[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t rx[4], ry[4];
          const int kx = q ^ sw_addr, ky = 4 + (q ^ sw_addr);
          const int rhox = (qr & 1) + 2 * m + 8 * kx + 64 * (qr >> 1);
          const int rhoy = (qr & 1) + 2 * m + 8 * ky + 64 * (qr >> 1);
          ldmatrix_x4_trans(ptx::smem_u32(&tiles[(buf * kColsTileRows2 + rhox) * 8 + (warp ^ cols_swz(rhox))]), rx);
          ldmatrix_x4_trans(ptx::smem_u32(&tiles[(buf * kColsTileRows2 + rhoy) * 8 + (warp ^ cols_swz(rhoy))]), ry);
          if constexpr (SIGNED) {
            // flags of the thread's own rows: 8-row group (q ^ sw_own) and the one 32 rows on
            // (16-row chunks are wholly inside or outside: rows is a multiple of 16)
            const int64_t r0t = cur.tr * kColsTileRows2 + 64 * a + 8 * (q ^ sw_own);
            uint32_t mx[4], my[4];
            sign_masks_bf16x8(r0t < rows ? __ldg(reinterpret_cast<const uint2*>(neg + r0t)) : make_uint2(0u, 0u), mx);
            sign_masks_bf16x8(r0t + 32 < rows ? __ldg(reinterpret_cast<const uint2*>(neg + r0t + 32)) : make_uint2(0u, 0u),
                              my);
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
              rx[mm] ^= mx[mm];
              ry[mm] ^= my[mm];
            }
          }
          xunpack(q, rx, ry, v);
        }
        __syncthreads();  // buffer free before the copies issued next iteration reuse it
        const float gA = (lane & 1) ? -1.0f : 1.0f, gB = (lane & 2) ? -1.0f : 1.0f;
        const float2 sA = make_float2(gA, gA), nsA = make_float2(-gA, -gA);
        const float2 sB = make_float2(gB, gB), nsB = make_float2(-gB, -gB);
        xrotate<K, !QUANT>(v, sA, nsA, sB, nsB, 1, 2, am);
        if constexpr (QUANT) {
          if (!qp.abort) {  // uniform: every lane takes part in the code-word exchange
            const int64_t r0 = cur.tr * kColsTileRows2, c0 = cur.tc * kColsTileCols2;
            const int64_t col = c0 + 8 * warp + (lane >> 2);
            uint32_t wx[8], wy[8];
            xcodes<MODE>(v, cs, qp.zero, wx, wy);
            uint8_t* o = codes + col * rows + r0;
            if constexpr (K <= 64) {
              // the thread's 64 consecutive rows, stored per 16 rows (rows is a multiple of 16)
              const int64_t rb = 64 * a;
              if (col < cols) {
                if (r0 + rb < rows) st_global_16B(o + rb, wx[0], wx[1], wx[2], wx[3]);
                if (r0 + rb + 16 < rows) st_global_16B(o + rb + 16, wx[4], wx[5], wx[6], wx[7]);
                if (r0 + rb + 32 < rows) st_global_16B(o + rb + 32, wy[0], wy[1], wy[2], wy[3]);
                if (r0 + rb + 48 < rows) st_global_16B(o + rb + 48, wy[4], wy[5], wy[6], wy[7]);
              }
            } else {
              const bool col_in = col < cols;
              auto pos_of = [&](int h) -> int64_t {
                if constexpr (K == 128) return 32 * h + 64 * (a & 1) + 128 * (a >> 1);
                else return 32 * h + 64 * a;
              };
              auto ok_pos = [&](int64_t pr) { return col_in && r0 + pr < rows; };
              xstore<K>(o, wx, wy, K == 256 ? a : (a & 1), 1, 2, pos_of, ok_pos, w32);
            }
          }
        }
        buf = buf == 2 ? 0 : buf + 1;
        continue;
      }
      // gather: 8 x (ldmatrix.x4.trans) -> 64 consecutive rows of one column per thread
      float2 v[32];
      {
        // sign flags of the thread's rows r0t + 0..63 (16-row chunks wholly inside or outside
        // the tensor: rows is a multiple of 16); rows past the end stay unflipped zeros
        uint32_t sm[SIGNED ? 32 : 1];
        if constexpr (SIGNED) {
          const int64_t r0t = cur.tr * kColsTileRows2 + 64 * (lane & 3);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t m8[8];
            const uint4 f = r0t + 16 * c < rows ? __ldg(reinterpret_cast<const uint4*>(neg + r0t + 16 * c))
                                                : make_uint4(0u, 0u, 0u, 0u);
            sign_masks_bf16x16(f, m8);
#pragma unroll
            for (int j = 0; j < 8; ++j) sm[8 * c + j] = m8[j];
          }
        }
        const int m = lane >> 3, q = lane & 7;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          const int rho = (q & 1) + 2 * m + 8 * kc + 64 * (q >> 1);
          uint32_t r[4];
          ldmatrix_x4_trans(ptx::smem_u32(&tiles[(buf * kColsTileRows2 + rho) * 8 + (warp ^ cols_swz(rho))]), r);
#pragma unroll
          for (int mm = 0; mm < 4; ++mm) {
            const uint32_t rw = SIGNED ? r[mm] ^ sm[(4 * kc + mm) % (SIGNED ? 32 : 1)] : r[mm];
            v[4 * kc + mm] = make_float2(__uint_as_float(rw << 16), __uint_as_float(rw & 0xFFFF0000u));
          }
        }
      }
      __syncthreads();  // buffer free before the copies issued next iteration reuse it
      stages_low<(K < 64 ? K : 64), 32>(v);
      if constexpr (K >= 128) stage_lanes<32>(v, 1, lane);
      if constexpr (K >= 256) stage_lanes<32>(v, 2, lane);
      if constexpr (!QUANT) {
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = absmax3(amax, v[i].x, v[i].y);
      } else {
        const int64_t r0 = cur.tr * kColsTileRows2, c0 = cur.tc * kColsTileCols2;
        const int64_t col = c0 + 8 * warp + (lane >> 2);
        const int64_t row = r0 + 64 * (lane & 3);
        if (col < cols) {
          uint8_t* o = codes + col * rows + row;
          // the scale's form chosen once for the thread's values (a warp-uniform flag)
          auto emit = [&](auto one_tag) {
            constexpr bool ONE = decltype(one_tag)::value;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (row + 16 * j < rows) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i = 8 * j + 2 * e;
                  w[e] = qp.zero ? 0u : scaled_codes4<MODE, ONE>(v[i], v[i + 1], cs, lp_fmt);
                }
                *reinterpret_cast<uint4*>(o + 16 * j) = MODE == kModeLowp ? lowp_pack16(w[0], w[1], w[2], w[3], lp_fmt)
                                                                          : make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          };
          if (cs.one_mul) emit(std::true_type{});
          else emit(std::false_type{});
        }
      }
      buf = buf == 2 ? 0 : buf + 1;
    }
  }
  if constexpr (!QUANT && MODE != kModeLowp) {
#pragma unroll
    for (int j = 0; j < kAcc; ++j) amax = absmax3(amax, am[j], 0.0f);
  }
  if (!QUANT) write_partial_unnormalised(amax, c, partials, scratch);
}

// ------------------------------------------------------------------ dim = 0, fp32 source

constexpr int kColsTileRows = 256;   // rows per tile: 32 lanes x 8 registers
constexpr int kColsTileBytes = 128;  // bytes of each source row per tile (8 x 16-byte chunks)

template <typename SrcT, int K, int MODE, bool SIGNED>
__global__ void __launch_bounds__(kQuantThreads)
fwhtq_cols_f32_kernel(const SrcT* __restrict__ src, int64_t rows, int64_t cols,
                  uint8_t* __restrict__ codes, float* __restrict__ partials, int n_partials,
                  float* __restrict__ scale_out, unsigned int* __restrict__ status, int reverse,
                  const uint8_t* __restrict__ neg, int lp_fmt) {
  // programmatic dependent launch: nothing is read or written before the previous grid in the
  // stream has completed; the next grid may be scheduled from here on
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  static_assert(K >= 16 && K <= 256 && (K & (K - 1)) == 0, "k must be a power of two in [16,256]");
  static_assert(!SIGNED || sizeof(SrcT) == 4, "sign masks of this kernel are for fp32 words");
  constexpr bool QUANT = MODE != kModeAbsmax;
  constexpr int CPC = 16 / static_cast<int>(sizeof(SrcT));  // columns per 16-byte chunk
  constexpr int TCOLS = 8 * CPC;                            // columns per tile
  __shared__ __align__(16) uint4 tile[kColsTileRows][8];
  __shared__ float scratch[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float c = __frsqrt_rn(static_cast<float>(K));

  QuantParams qp{0.0f, false, false};
  if (QUANT) {
    qp = finish_absmax<MODE>(partials, n_partials, scale_out, scratch, status, lp_fmt);
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
    const int64_t first = reverse ? last : b, step = reverse ? -G : G;
    TileWalk cur;
    cur.init(first, step, n_ct);
    for (int64_t t = first; reverse ? t >= 0 : t < n_tiles; t += step, cur.advance()) {
      const int64_t r0 = cur.tr * kColsTileRows;
      const int64_t c0 = cur.tc * TCOLS;
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
      uint32_t sm[8];  // sign masks of the 8 rows (8-row groups are wholly inside or outside)
      if constexpr (SIGNED) {
        const int64_t r8 = r0 + 8 * lane;
        const uint2 f = r8 < rows ? __ldg(reinterpret_cast<const uint2*>(neg + r8)) : make_uint2(0u, 0u);
        uint32_t m4[4];
        sign_masks_f32x4(f.x, m4);
#pragma unroll
        for (int i = 0; i < 4; ++i) sm[i] = m4[i];
        sign_masks_f32x4(f.y, m4);
#pragma unroll
        for (int i = 0; i < 4; ++i) sm[4 + i] = m4[i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 raw = tile[8 * lane + i][warp ^ (lane & 7)];
        if constexpr (SIGNED) {
          raw.x ^= sm[i];
          raw.y ^= sm[i];
          raw.z ^= sm[i];
          raw.w ^= sm[i];
        }
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
      } else if constexpr (MODE == kModeLowp) {
        // minifloats: lanes 2m and 2m + 1 hold rows 16m .. 16m + 15 of a column, one 16-byte chunk
        // (rows is a multiple of 16, so both lanes are inside the tensor or both past its end)
        const int64_t row = r0 + 8 * lane;
#pragma unroll
        for (int j = 0; j < CPC; ++j) {
          const int64_t col = c0 + warp * CPC + j;
          float y8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) y8[i] = v[i][j];
          const uint2 c8 = codes8<MODE>(y8, qp.inv, qp.zero, lp_fmt);
          const uint32_t px = lowp_compress4(c8.x, lp_fmt), py = lowp_compress4(c8.y, lp_fmt);
          const uint32_t qx = __shfl_down_sync(0xFFFFFFFFu, px, 1), qy = __shfl_down_sync(0xFFFFFFFFu, py, 1);
          if ((lane & 1) == 0 && row < rows && col < cols)
            __stcs(reinterpret_cast<uint4*>(codes + col * rows + row), lowp_chunk(px, py, qx, qy, lp_fmt));
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
              __stcs(reinterpret_cast<uint2*>(codes + col * rows + row), codes8<MODE>(y8, qp.inv, qp.zero, lp_fmt));
            }
          }
        }
      }
    }
  }
  if (!QUANT) write_partial(amax, bad, partials, scratch);
}

}  // namespace hq
