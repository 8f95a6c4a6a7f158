// Dense tensor-core throughput probe: tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32 per
// instruction; kind::i8 or kind::f8f6f4 with e4m3 operands) with both operand tiles resident in
// shared memory and the accumulator in TMEM, so no global-memory traffic limits it.  One CTA
// pair per TPC; CTA 0 of each pair issues every MMA back to back into one accumulator and
// commits once at the end.  The host times the launch with CUDA events: that is the measured
// dense INT8 / FP8 peak used as the GEMMs' roofline denominator (no counterpart on the pages,
// which quote no B200 figure; it replaces the nominal-ratio estimate bf16 peak x 2).
//
// Operand bytes are pseudo-random (a fixed integer hash of the byte offset, e4m3 codes with
// bit 6 clear so no NaN and |x| <= 1.875): the tensor pipe's power draw, and so its clock under
// the power cap, depends on the data, and zeros would flatter it.
#pragma once
#include <cstdint>
#include "gemm_tcgen05.cuh"
#include "sm100_ptx.cuh"

namespace hq {
namespace peak {

constexpr int kThreads = 128;
constexpr uint32_t kTileBytes = 128u * 128u;  // 128 rows x 128 bytes, 128-byte swizzle atoms
// More shared memory than the probe uses, so that no two CTAs share an SM.
constexpr size_t kSmemBytes = 140 * 1024;
static_assert(1024 + 2 * size_t(kTileBytes) + 64 <= kSmemBytes, "operand tiles, barrier, TMEM holder");
// The second CTA of a pair waits through the whole run: n_blocks <= 2^24 is at most about 5 s
// of MMAs at the lowest clocks seen under the power cap, well inside this limit.
constexpr uint64_t kDrainLimitNs = 30000000000ull;

// Instruction descriptor of the CTA-pair MMA: M = 256, N = 256, dense, K-major A and B.
template <int FMT>
__host__ __device__ constexpr uint32_t peak_idesc() {
  return (uint32_t(FMT == gemm::kInt8 ? 2 : 1) << 4) | (uint32_t(FMT == gemm::kInt8 ? 1 : 0) << 7) |
         (uint32_t(FMT == gemm::kInt8 ? 1 : 0) << 10) | (uint32_t(256 >> 3) << 17) | (uint32_t(256 >> 4) << 24);
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) mma_peak_kernel(int64_t n_blocks, unsigned int* __restrict__ status) {
  extern __shared__ uint8_t raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a = base;
  uint8_t* b = base + kTileBytes;
  uint64_t* bar_p = reinterpret_cast<uint64_t*>(base + 2 * kTileBytes);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bar_p + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();

  // operands: 32 KB of hashed bytes, 16 per thread and step
  for (uint32_t off = 16u * threadIdx.x; off < 2 * kTileBytes; off += 16u * kThreads) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t h = (off + 4u * j + 0x9E3779B9u * (rank + 1)) * 0x85EBCA6Bu;
      h ^= h >> 13;
      h *= 0xC2B2AE35u;
      h ^= h >> 16;
      w[j] = FMT == gemm::kInt8 ? h : (h & 0xBFBFBFBFu);
    }
    ptx::st_shared_v4(ptx::smem_u32(base + off), w[0], w[1], w[2], w[3]);
  }
  ptx::fence_proxy_async_smem();  // generic-proxy writes visible to the tensor core
  if (warp == 0 && lane == 0) {
    ptx::mbar_init(ptx::smem_u32(bar_p), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(holder), 256);
    ptx::tmem_relinquish_pair();
  }
  __syncthreads();
  ptx::tc_fence_before_sync();
  ptx::cluster_sync();
  ptx::tc_fence_after_sync();
  const uint32_t tmem = *holder;

  if (rank == 0 && warp == 0 && lane == 0) {
    const uint32_t idesc = peak_idesc<FMT>();
    const uint32_t sa = ptx::smem_u32(a), sb = ptx::smem_u32(b);
    for (int64_t kb = 0; kb < n_blocks; ++kb) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = gemm::smem_desc_sw128(sa + 32u * kk);
        const uint64_t bd = gemm::smem_desc_sw128(sb + 32u * kk);
        if (FMT == gemm::kInt8) ptx::mma_i8_pair(tmem, ad, bd, idesc, (kb | kk) ? 1u : 0u);
        else ptx::mma_f8_pair(tmem, ad, bd, idesc, (kb | kk) ? 1u : 0u);
      }
    }
    ptx::tc_commit_pair_mc(ptx::smem_u32(bar_p), 0x3);
  }
  // both CTAs wait (bounded) for the last MMA before their tensor memory is released
  if (threadIdx.x == 0) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(ptx::smem_u32(bar_p), 0)) {
      if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) {
        atomicCAS(status, 0u, 6u /* HQ_ERR_TIMEOUT */);
        break;
      }
    }
  }
  __syncthreads();
  ptx::tc_fence_before_sync();
  ptx::cluster_sync();
  ptx::tc_fence_after_sync();
  if (warp == 1) ptx::tmem_dealloc_pair(tmem, 256);
}

}  // namespace peak
}  // namespace hq
