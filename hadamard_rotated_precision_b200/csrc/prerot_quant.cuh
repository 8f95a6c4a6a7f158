// Tensor-wise quantization of values that are already rotated: no transform, only the absmax
// and the codes.  This is the next layer's operand when this layer's GEMM applied the next
// layer's rotation in its epilogue (the output rotated along its columns, fp32).
//
// Method: "Training Transformers with 4-bit Integers", section 3.3 (the Hadamard blocks are
// applied before quantization; here they were applied by the producing GEMM) and "HALO:
// Hadamard-Assisted Lower-Precision Optimization for LLMs", Approach (tensor-wise scale).
// Numerics as the rotating quantizer after its rotation: a = max |y| over the tensor,
// inv = fp32(QMAX / a), code = RNE(fp32(y * inv)) (INT8 clamp-free, e4m3 saturating),
// scale = fp32(a / QMAX); a == 0 gives scale 1 and zero codes, a non-finite a the status
// HQ_ERR_NONFINITE and no codes.
//
// Two passes over the fp32 tensor, each a grid-stride stream of 16-byte loads:
//   pass 1 (kModeAbsmax): per-CTA partial maxima;
//   pass 2 (kModeInt8 / kModeFp8): every CTA reduces the partials, then writes 4 codes per
//   16-byte load (one 32-bit store).
#pragma once
#include <cstdint>
#include "fwht_quant.cuh"

namespace hq {
namespace prerot {

constexpr int kThreads = 256;

template <int MODE>
__global__ void __launch_bounds__(kThreads) prerot_quant_kernel(const float* __restrict__ y, int64_t n4,
                                                                uint8_t* __restrict__ codes,
                                                                float* __restrict__ partials, int n_partials,
                                                                float* __restrict__ scale,
                                                                unsigned int* __restrict__ status) {
  static_assert(MODE == kModeAbsmax || MODE == kModeInt8 || MODE == kModeFp8, "INT8 / e4m3 codes");
  __shared__ float scratch[32];
  const float4* y4 = reinterpret_cast<const float4*>(y);
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  const int64_t first = int64_t(blockIdx.x) * kThreads + threadIdx.x;
  if constexpr (MODE == kModeAbsmax) {
    float m0 = 0.0f, m1 = 0.0f;  // two chains; max.NaN keeps any NaN
    for (int64_t i = first; i < n4; i += stride) {
      const float4 v = __ldcs(y4 + i);
      m0 = absmax3(m0, v.x, v.y);
      m1 = absmax3(m1, v.z, v.w);
    }
    float m = absmax3(m0, m1, 0.0f);
    m = m != m ? INFINITY : m;  // NaN -> +inf: the pass-2 reduction sees a non-finite a
    write_partial(m, false, partials, scratch);
  } else {
    const QuantParams q = finish_absmax<MODE>(partials, n_partials, scale, scratch, status);
    if (q.abort) return;
    const float2 inv2 = make_float2(q.inv, q.inv);
    uint32_t* c4 = reinterpret_cast<uint32_t*>(codes);
    for (int64_t i = first; i < n4; i += stride) {
      const float4 v = __ldcs(y4 + i);
      c4[i] = q.zero ? 0u : codes4<MODE>(mul2(make_float2(v.x, v.y), inv2), mul2(make_float2(v.z, v.w), inv2));
    }
  }
}

}  // namespace prerot
}  // namespace hq
