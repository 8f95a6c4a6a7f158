// Low-precision GEMM on the 5th-generation tensor cores with a fused dequantization epilogue.
//
//   C[i][j] = sum_l A[i][l] * B[j][l]          A: [M][K] codes, B: [N][K] codes (both K-major)
//   out[i][j] = bf16( fp32(C[i][j]) * fp32(s_a * s_b) )       (or the raw accumulator)
//
// Method: "Training Transformers with 4-bit Integers", section 3.1 (the integer product is
// computed on integer tensor cores and dequantized back to floating point by the scales)
// and section 3.3 (the Hadamard rotation of both operands cancels in the product, so the
// GEMM runs directly on the rotated codes); "HALO: Hadamard-Assisted Lower-Precision
// Optimization for LLMs" (INT8 / FP8 operands with one tensor-wise scale each).
//
// Kernel shape (one CTA per SM, persistent over output tiles):
//   tile 128 x 256, K step 128 bytes (one 128-byte swizzle atom per operand row), 4-stage
//   shared-memory ring fed by TMA (no multicast), tcgen05.mma (kind::i8 / kind::f8f6f4,
//   M=128 N=256 K=32) issued by one thread into a TMEM accumulator, two accumulators
//   (2 x 256 TMEM columns) so the epilogue of tile t overlaps the main loop of tile t+1.
//   warp 0: TMA producer; warp 1: TMEM allocator + MMA issuer; warps 2-5: epilogue
//   (warp w reads TMEM lanes 32*(w%4) .. +31 = output rows of that quarter tile).
// Every wait on an mbarrier is bounded (about a second); on expiry the kernel records
// HQ_ERR_TIMEOUT in the status word, the other roles stop, in-flight copies and MMAs are
// drained with bounded waits, TMEM is freed and the CTA exits.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100_ptx.cuh"

namespace hq {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes == elements for 8-bit operands
constexpr int STAGES = 4;
constexpr int UMMA_K = 32;  // K of one tcgen05.mma for 8-bit operands
constexpr int A_STAGE_BYTES = BM * BK;
constexpr int B_STAGE_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int ACC_BUFS = 2;
constexpr int TMEM_COLS = ACC_BUFS * BN;  // 512: the whole tensor memory of the SM
constexpr int NUM_THREADS = 192;
constexpr int NUM_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
constexpr size_t SMEM_BYTES = 1024 + size_t(STAGES) * STAGE_BYTES + NUM_BARS * 8 + 16;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;  // 1 s per wait

enum Fmt : int { kInt8 = 0, kFp8 = 1 };
// kOutF32: the dequantized value fp32(acc) * fp32(s_a * s_b) without the bf16 rounding (for an
// output that is still rotated and is de-rotated in fp32 afterwards).
enum Out : int { kOutBf16 = 0, kOutAcc = 1, kOutF32 = 2 };

// Instruction descriptor: dense, D = s32 (int8) / f32 (fp8), A = B = s8 / e4m3, both K-major,
// N = 256, M = 128.
template <int FMT>
__host__ __device__ constexpr uint32_t instr_desc() {
  return (uint32_t(FMT == kInt8 ? 2 : 1) << 4)     // D format
         | (uint32_t(FMT == kInt8 ? 1 : 0) << 7)   // A format
         | (uint32_t(FMT == kInt8 ? 1 : 0) << 10)  // B format
         | (uint32_t(BN >> 3) << 17)               // N / 8
         | (uint32_t(BM >> 4) << 24);              // M / 16
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row core groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  return uint64_t((saddr & 0x3FFFFu) >> 4)      // start address
         | (uint64_t(1) << 16)                   // leading-dimension offset (unused, 1)
         | (uint64_t(1024 >> 4) << 32)           // stride offset between 8-row groups
         | (uint64_t(1) << 46)                   // descriptor version (sm_100)
         | (uint64_t(2) << 61);                  // 128-byte swizzle
}

struct Shared {
  uint8_t* a;
  uint8_t* b;
  uint8_t* epi;  // pair kernel: bf16 output boxes staged for TMA stores
  uint64_t* bars;
  uint32_t* tmem_holder;
  volatile int* abort_flag;
};

__device__ __forceinline__ Shared carve(uint8_t* raw) {
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  Shared s;
  s.a = base;
  s.b = base + STAGES * A_STAGE_BYTES;
  s.epi = nullptr;
  s.bars = reinterpret_cast<uint64_t*>(s.b + STAGES * B_STAGE_BYTES);
  s.tmem_holder = reinterpret_cast<uint32_t*>(s.bars + NUM_BARS);
  s.abort_flag = reinterpret_cast<volatile int*>(s.tmem_holder + 1);
  return s;
}

// Bounded wait; gives up when the flag is raised by another role or after WAIT_LIMIT_NS.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned int* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
      *abort_flag = 1;
      atomicCAS(status, 0u, 6u /* HQ_ERR_TIMEOUT */);
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (used to drain work already in flight).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, unsigned int* status) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
      atomicCAS(status, 0u, 6u);
      return;
    }
  }
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int& m_blk, int& n_blk) {
  m_blk = tile % num_m;  // M fastest: concurrent CTAs share B tiles and sweep A
  n_blk = tile / num_m;
}

template <int FMT, int OUT>
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], void* out, int64_t row,
                                            int col0, int N, float sab) {
  if (OUT == kOutBf16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + row * N + col0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (col0 + 8 * q + 8 > N) break;
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 8 * q + 2 * e;
        float x0, x1;
        if (FMT == kInt8) {
          x0 = __int2float_rn(static_cast<int>(r[i]));
          x1 = __int2float_rn(static_cast<int>(r[i + 1]));
        } else {
          x0 = __uint_as_float(r[i]);
          x1 = __uint_as_float(r[i + 1]);
        }
        const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(x0, sab), __fmul_rn(x1, sab));
        pk[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(o + 8 * q) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  } else if (OUT == kOutF32) {
    float* o = reinterpret_cast<float*>(out) + row * N + col0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (col0 + 4 * q + 4 > N) break;
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t u = r[4 * q + e];
        x[e] = __fmul_rn(FMT == kInt8 ? __int2float_rn(static_cast<int>(u)) : __uint_as_float(u), sab);
      }
      *reinterpret_cast<float4*>(o + 4 * q) = make_float4(x[0], x[1], x[2], x[3]);
    }
  } else {
    uint32_t* o = reinterpret_cast<uint32_t*>(out) + row * N + col0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (col0 + 4 * q + 4 > N) break;
      *reinterpret_cast<uint4*>(o + 4 * q) = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
    }
  }
}

template <int FMT, int OUT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
            const float* __restrict__ scale_a, const float* __restrict__ scale_b, void* __restrict__ out,
            int M, int N, int K, unsigned int* __restrict__ status, int skip_first_load, uint32_t ab_code) {
  extern __shared__ uint8_t smem_raw[];
  const Shared sh = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + BK - 1) / BK;

  auto bar = [&](int i) { return ptx::smem_u32(sh.bars + i); };
  auto full_bar = [&](int s) { return bar(s); };
  auto empty_bar = [&](int s) { return bar(STAGES + s); };
  auto tfull_bar = [&](int b) { return bar(2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar(2 * STAGES + ACC_BUFS + b); };
  const uint32_t drain_bar = bar(2 * STAGES + 2 * ACC_BUFS);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < ACC_BUFS; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 4);  // one arrive per epilogue warp
    }
    ptx::mbar_init(drain_bar, 1);
    *sh.abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmap_a);
    ptx::prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(sh.tmem_holder), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *sh.tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(tile, num_m, m_blk, n_blk);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, sh.abort_flag, status)) { ok = false; break; }
          if (skip_first_load && tile == static_cast<int>(blockIdx.x) && kb == 0) {
            // test hook: leave the first stage un-armed so the MMA warp's bounded wait on it
            // expires (HQ_ERR_TIMEOUT) and every role takes the abort path
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            continue;
          }
          ptx::mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          ptx::tma_load_2d(ptx::smem_u32(sh.a + stage * A_STAGE_BYTES), &tmap_a, kb * BK, m_blk * BM, full_bar(stage));
          ptx::tma_load_2d(ptx::smem_u32(sh.b + stage * B_STAGE_BYTES), &tmap_b, kb * BK, n_blk * BN, full_bar(stage));
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // every copy this thread started has landed before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) drain_wait(full_bar(s), (issued_parity >> s) & 1u, status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // ab_code: the A and B element format of kind::f8f6f4 (e4m3 0, e2m3 3, e3m2 4, e2m1 5)
      const uint32_t idesc = instr_desc<FMT>() | (ab_code << 7) | (ab_code << 10);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!wait_bounded(tempty_bar(acc), acc_phase ^ 1u, sh.abort_flag, status)) break;
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, sh.abort_flag, status)) { ok = false; break; }
          ptx::tc_fence_after_sync();
          const uint32_t a_addr = ptx::smem_u32(sh.a + stage * A_STAGE_BYTES);
          const uint32_t b_addr = ptx::smem_u32(sh.b + stage * B_STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint64_t ad = smem_desc_sw128(a_addr + kk * UMMA_K);
            const uint64_t bd = smem_desc_sw128(b_addr + kk * UMMA_K);
            const uint32_t accumulate = (kb > 0 || kk > 0) ? 1u : 0u;
            if (FMT == kInt8) ptx::mma_i8(d_tmem, ad, bd, idesc, accumulate);
            else ptx::mma_f8(d_tmem, ad, bd, idesc, accumulate);
          }
          ptx::tc_commit(empty_bar(stage));  // frees the smem stage once these MMAs retire
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        ptx::tc_commit(tfull_bar(acc));  // accumulator complete
        if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
      }
      // all MMAs issued by this thread have retired before TMEM is released
      ptx::tc_commit(drain_bar);
      drain_wait(drain_bar, 0, status);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int quarter = warp & 3;
    const float sab = (OUT == kOutBf16) ? __fmul_rn(*scale_a, *scale_b) : 0.0f;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int m_blk, n_blk;
      tile_coords(tile, num_m, m_blk, n_blk);
      int ok = 0;
      if (lane == 0) ok = wait_bounded(tfull_bar(acc), acc_phase, sh.abort_flag, status) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      ptx::tc_fence_after_sync();
      const int64_t row = int64_t(m_blk) * BM + quarter * 32 + lane;
      const uint32_t t_row = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(t_row + uint32_t(c * 32), r);
        ptx::tmem_ld_wait();
        const int col0 = n_blk * BN + c * 32;
        if (row < M && col0 < N) store_chunk<FMT, OUT>(r, out, row, col0, N, sab);
      }
      ptx::tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(tempty_bar(acc));
      if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
    }
  }

  ptx::tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}


// ---------------------------------------------------------------- output rotation in the epilogue
//
// For the fp32 output (kOutF32) the epilogue can apply blockdiag(H_k / sqrt(k)) along the
// output's columns before storing: an epilogue thread owns one output row of the tile in TMEM,
// so a k-block of columns is in its registers.  Arithmetic as the library's rotation:
// z = fp32(acc) * sab, Sylvester butterflies h = 1 .. k/2 (index bit 0 first, fp32 RNE), then
// one multiply by fp32(1/sqrt(k)).

// Dequantized fp32 values of 32 consecutive accumulator columns of this thread's row.
template <int FMT>
__device__ __forceinline__ void load_dequant32(uint32_t taddr, float sab, float* v) {
  uint32_t r[32];
  ptx::tmem_ld_32x32b_x32(taddr, r);
  ptx::tmem_ld_wait(r);
#pragma unroll
  for (int i = 0; i < 32; ++i)
    v[i] = __fmul_rn(FMT == kInt8 ? __int2float_rn(static_cast<int>(r[i])) : __uint_as_float(r[i]), sab);
}

// Butterfly stages h = 1 .. H/2 over NV consecutive values (blocks of H).
template <int NV, int H>
__device__ __forceinline__ void butterflies(float* v) {
#pragma unroll
  for (int h = 1; h < H; h <<= 1) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      if (i & h) continue;
      const float u = v[i], w = v[i + h];
      v[i] = __fadd_rn(u, w);
      v[i + h] = __fsub_rn(u, w);
    }
  }
}

// o[0 .. n) = v * c for the first n of NV values (n a multiple of 4; unrolled, so v stays in
// registers).
template <int NV>
__device__ __forceinline__ void store_f32_scaled(float* o, const float* v, int n, float c) {
#pragma unroll
  for (int q = 0; q < NV; q += 4)
    if (q < n)
      *reinterpret_cast<float4*>(o + q) =
          make_float4(__fmul_rn(v[q], c), __fmul_rn(v[q + 1], c), __fmul_rn(v[q + 2], c), __fmul_rn(v[q + 3], c));
}

// k <= 128: chunks of max(k, 32) columns, each rotated in registers and stored.
template <int FMT, int RK, int TILE_N>
__device__ __forceinline__ void epi_rot_cols(uint32_t t_row, float sab, float c, float* out_row, int col_base,
                                             bool row_ok, int N) {
  constexpr int W = RK < 32 ? 32 : RK;
#pragma unroll 1
  for (int b = 0; b < TILE_N / W; ++b) {
    float v[W];
#pragma unroll
    for (int q = 0; q < W / 32; ++q) load_dequant32<FMT>(t_row + uint32_t(b * W + 32 * q), sab, v + 32 * q);
    butterflies<W, RK>(v);
    const int col0 = col_base + b * W;
    // N % k == 0: whole blocks (a 32-column chunk of k = 16 blocks may end at N after one)
    if (row_ok && col0 < N) store_f32_scaled<W>(out_row + col0, v, N - col0, c);
  }
}

// k = 256 (the tile's whole width): stages h = 1 .. 64 on each 128-column half, written back to
// the accumulator as fp32 bits, then the last stage pairs column j with j + 128.
template <int FMT, int TILE_N>
__device__ __forceinline__ void epi_rot_cols256(uint32_t t_row, float sab, float c, float* out_row, int col_base,
                                                bool row_ok, int N) {
  static_assert(TILE_N == 256, "k = 256 spans the whole tile");
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf) {
    float v[128];
#pragma unroll
    for (int q = 0; q < 4; ++q) load_dequant32<FMT>(t_row + uint32_t(128 * hf + 32 * q), sab, v + 32 * q);
    butterflies<128, 128>(v);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[32 * q + i]);
      ptx::tmem_st_32x32b_x32(t_row + uint32_t(128 * hf + 32 * q), r);
    }
  }
  ptx::tmem_st_wait();
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    uint32_t a[32], b[32];
    ptx::tmem_ld_32x32b_x32(t_row + uint32_t(32 * q), a);
    ptx::tmem_ld_32x32b_x32(t_row + uint32_t(128 + 32 * q), b);
    ptx::tmem_ld_wait(a);
    ptx::reg_fence(b);
    float lo[32], hi[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float u = __uint_as_float(a[i]), w = __uint_as_float(b[i]);
      lo[i] = __fadd_rn(u, w);
      hi[i] = __fsub_rn(u, w);
    }
    if (row_ok && col_base < N) {
      store_f32_scaled<32>(out_row + col_base + 32 * q, lo, 32, c);
      store_f32_scaled<32>(out_row + col_base + 128 + 32 * q, hi, 32, c);
    }
  }
}

// ====================================================================== CTA-pair variant
//
// A cluster of two CTAs on the two SMs of a TPC computes a 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32 per instruction): CTA r of the pair holds
// rows 128 r .. 128 r + 127 of the A tile and rows 128 r .. of the B tile (its half of N) in
// its own shared memory, and the 128 x 256 accumulator of its rows in its own TMEM.  Per CTA a
// stage is 16 KB of A + 16 KB of B (half of the single-CTA kernel's B traffic per output), so
// six stages fit.  Only CTA 0 issues MMAs; both CTAs load their own tiles (no multicast), the
// loads of both count on CTA 0's "full" barrier, and CTA 0's commits arrive on the barriers of
// both CTAs.  Epilogue warps of both CTAs report a drained accumulator to CTA 0.
namespace pair {

constexpr int BM = 256;    // rows per pair tile (128 per CTA)
constexpr int HALF = 128;  // A rows per CTA

// Row `lane` of a 32 x 64 bf16 output box in shared memory (128-byte swizzle: 16-byte chunk q,
// columns 8q .. 8q+7, at q ^ (lane & 7)) from 64 accumulators (r0: columns 0-31, r1: 32-63):
// bf16(fp32(acc) * sab).
template <int FMT>
__device__ __forceinline__ void write_box_row(uint32_t box, int lane, const uint32_t (&r0)[32],
                                              const uint32_t (&r1)[32], float sab) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = 8 * (q & 3) + 2 * e;
      const uint32_t u0 = q < 4 ? r0[i] : r1[i], u1 = q < 4 ? r0[i + 1] : r1[i + 1];
      float x0, x1;
      if (FMT == kInt8) {
        x0 = __int2float_rn(static_cast<int>(u0));
        x1 = __int2float_rn(static_cast<int>(u1));
      } else {
        x0 = __uint_as_float(u0);
        x1 = __uint_as_float(u1);
      }
      const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(x0, sab), __fmul_rn(x1, sab));
      pk[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    ptx::st_shared_v4(box + uint32_t(lane * 128 + ((q ^ (lane & 7)) << 4)), pk[0], pk[1], pk[2], pk[3]);
  }
}

// Tile geometry for an N tile of BN_ (256 or 128) columns: each CTA holds BN_/2 rows of B.
// The bf16 epilogue stages output boxes of 32 rows x 64 columns (4 KB, 128-byte swizzle) in
// shared memory for TMA stores.  Default shape: a 192 KB operand ring, four epilogue warps
// (one per 32-lane quarter of TMEM) and two boxes per warp.  SHORT_K (contractions of at most
// kShortKBlocks k-blocks, where a tile's main loop is shorter than writing its output): a
// 160 KB ring and eight epilogue warps, two per TMEM quarter, each owning half of the tile's
// columns with room for its whole share, so the accumulator is released as soon as it has
// been read and the stores stream out while the next tiles are computed.
constexpr int kShortStages = 5;  // SHORT_K operand ring: stages of 32 KB (BN = 256)
constexpr int kShortBoxes = 2;   // SHORT_K output boxes per epilogue warp

template <int BN_, bool SHORT_K = false>
struct Geo {
  static constexpr int EPI_WARPS = SHORT_K ? 8 : 4;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;  // producer, MMA issuer, epilogue
  static constexpr int BN = BN_;
  static constexpr int B_ROWS = BN_ / 2;
  static constexpr int A_STAGE_BYTES = HALF * BK;
  static constexpr int B_STAGE_BYTES = B_ROWS * BK;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;  // per CTA
  static constexpr int STAGES = ((SHORT_K ? kShortStages : 6) * (16384 + 16384)) / STAGE_BYTES;
  static constexpr int TMEM_COLS = ACC_BUFS * BN_;                      // 512 or 256
  static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
  static constexpr int BOX_COLS = 64;
  static constexpr int BOX_BYTES = 32 * BOX_COLS * 2;
  static constexpr int CHUNKS = BN_ / BOX_COLS / (EPI_WARPS / 4);  // 64-column chunks per tile and warp
  static constexpr int NB = SHORT_K ? (CHUNKS < kShortBoxes ? CHUNKS : kShortBoxes) : 2;  // boxes per epilogue warp
  static constexpr bool WHOLE = SHORT_K && NB == CHUNKS;  // the boxes hold the warp's whole tile share
  static constexpr int EPI_BYTES = EPI_WARPS * NB * BOX_BYTES;
  static constexpr size_t SMEM_BYTES =
      1024 + size_t(STAGES) * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
  static_assert(SMEM_BYTES <= 232448, "more dynamic shared memory than a B200 CTA may have");
};

// Tile order of the pair kernel: bands of kRasterBand M-blocks; within a band the M-block
// varies fastest, then the N-block.  The tiles in flight together (one per CTA pair) then read
// kRasterBand A panels and about pairs / kRasterBand B panels (256 rows x K each), which stay
// in L2 while the band sweeps N, so A is read from DRAM about once and B once per band.  With
// the M-fastest order over the whole of M, the A panels of every M-block were read again for
// each N-block column once A exceeded what L2 keeps beside the output stream (12288 x 4096 x
// 8192: 1054 MB of DRAM reads for 134 MB of operands).  A GEMM with at most kRasterBand
// M-blocks is one band, i.e. the plain M-fastest order.
constexpr int kRasterBand = 16;

__device__ __forceinline__ void pair_tile_coords(int tile, int num_m, int num_n, int& m_blk, int& n_blk) {
  const int band = tile / (kRasterBand * num_n);
  const int m0 = band * kRasterBand;
  const int gb = min(kRasterBand, num_m - m0);
  const int idx = tile - band * kRasterBand * num_n;
  m_blk = m0 + idx % gb;
  n_blk = idx / gb;
}

constexpr int kShortKBlocks = 8;  // K <= 1024 bytes: the SHORT_K shape

template <int FMT, int BN_>
__host__ __device__ constexpr uint32_t instr_desc() {
  return (uint32_t(FMT == kInt8 ? 2 : 1) << 4) | (uint32_t(FMT == kInt8 ? 1 : 0) << 7) |
         (uint32_t(FMT == kInt8 ? 1 : 0) << 10) | (uint32_t(BN_ >> 3) << 17) | (uint32_t(BM >> 4) << 24);
}

template <class G>
__device__ __forceinline__ Shared carve(uint8_t* raw) {
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  Shared s;
  s.a = base;
  s.b = base + G::STAGES * G::A_STAGE_BYTES;
  s.epi = s.b + G::STAGES * G::B_STAGE_BYTES;  // 1024-byte aligned
  s.bars = reinterpret_cast<uint64_t*>(s.epi + G::EPI_BYTES);
  s.tmem_holder = reinterpret_cast<uint32_t*>(s.bars + G::NUM_BARS);
  s.abort_flag = reinterpret_cast<volatile int*>(s.tmem_holder + 1);
  return s;
}

// MN: both operands MN-major, i.e. stored contraction-outermost (A as [K][M], B as [K][N]; the
// kind::i8 and e4m3 inputs allow it).  A TMA box is then 128 contraction rows of 128 bytes
// along M (or N): one 128-byte swizzle atom wide, so the smem descriptor keeps its 1024-byte
// stride between 8-row groups (now groups along the contraction), and one MMA's 32-deep slice
// starts 32 rows = 4096 bytes further on.  Needs BN_ = 256 (128 B rows per CTA).
template <int FMT, int OUT, int BN_, bool SHORT_K, bool MN = false>
__global__ void __launch_bounds__(Geo<BN_, SHORT_K>::THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const __grid_constant__ CUtensorMap tmap_out, const float* __restrict__ scale_a,
                 const float* __restrict__ scale_b, void* __restrict__ out, int M, int N, int K,
                 unsigned int* __restrict__ status, int split_from, uint32_t* __restrict__ part_ws,
                 int* __restrict__ counters, uint32_t ab_code, int rot_k) {
  // rot_k (kOutF32 only; 0 = none): rotate the output along its columns in blocks of rot_k
  // before storing (see epi_rot_cols)
  using G = Geo<BN_, SHORT_K>;
  static_assert(!MN || (BN_ == 256 && !SHORT_K && OUT != kOutBf16), "MN-major operands: 256-wide tiles, direct stores");
  static_assert(!SHORT_K || OUT == kOutBf16, "SHORT_K: bf16 output through TMA stores");
  constexpr int BN = G::BN, STAGES = G::STAGES, A_STAGE_BYTES = G::A_STAGE_BYTES;
  constexpr int B_STAGE_BYTES = G::B_STAGE_BYTES, STAGE_BYTES = G::STAGE_BYTES, TMEM_COLS = G::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  const Shared sh = carve<G>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + BK - 1) / BK;
  // Work items: tiles below split_from whole (items 0 .. F-1, tile = item), the tiles from
  // split_from on in two halves of the k-blocks (item F + j: tile F + j % T, half j / T, so both
  // halves of a tile run in the same wave).  split_from >= num_tiles: no split; 0: every tile
  // split; in between: only the last, partial wave's tiles, so that it takes half a tile-time.
  // A half writes its partial accumulator to part_ws; the warp slab that finishes second adds
  // the other half and writes the output (bf16 output only).
  const int split_f = SHORT_K ? num_tiles : min(split_from, num_tiles);  // SHORT_K never splits
  const int split_t = num_tiles - split_f;
  const int num_items = split_f + 2 * split_t;
  const int kb_half = (num_kb + 1) / 2;
  struct Item { int tile, half, kb_begin, kb_end; bool part; };
  auto item_at = [&](int item) {
    Item it;
    if (item < split_f) {
      it.tile = item; it.half = 0; it.kb_begin = 0; it.kb_end = num_kb; it.part = false;
    } else {
      const int j = item - split_f;
      it.tile = split_f + j % split_t;
      it.half = j / split_t;
      it.kb_begin = it.half ? kb_half : 0;
      it.kb_end = it.half ? num_kb : kb_half;
      it.part = true;
    }
    return it;
  };

  auto bar = [&](int i) { return ptx::smem_u32(sh.bars + i); };
  auto full_bar = [&](int s) { return bar(s); };
  auto empty_bar = [&](int s) { return bar(STAGES + s); };
  auto tfull_bar = [&](int b) { return bar(2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar(2 * STAGES + ACC_BUFS + b); };
  const uint32_t drain_bar = bar(2 * STAGES + 2 * ACC_BUFS);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);   // used in CTA 0: its producer's arrive + both CTAs' bytes
      ptx::mbar_init(empty_bar(s), 1);  // CTA 0's commit, multicast to both CTAs
    }
    for (int b = 0; b < ACC_BUFS; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 2 * G::EPI_WARPS);  // used in CTA 0: every epilogue warp of both CTAs
    }
    ptx::mbar_init(drain_bar, 1);
    *sh.abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmap_a);
    ptx::prefetch_tmap(&tmap_b);
    if (OUT == kOutBf16) ptx::prefetch_tmap(&tmap_out);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(sh.tmem_holder), TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before_sync();
  ptx::cluster_sync();  // both CTAs' barriers initialised before any remote arrive or copy
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *sh.tmem_holder;
  // programmatic dependent launch: the set-up above overlaps the previous grid's tail; codes,
  // scales and the output are touched only once that grid has completed
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int item = pair_id; item < num_items && ok; item += num_pairs) {
        const Item it = item_at(item);
        int m_blk, n_blk;
        pair_tile_coords(it.tile, num_m, num_n, m_blk, n_blk);
        for (int kb = it.kb_begin; kb < it.kb_end; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, sh.abort_flag, status)) { ok = false; break; }
          const uint32_t fb = ptx::mapa_shared(full_bar(stage), 0);
          if (leader) ptx::mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          const int a_mn = m_blk * BM + int(rank) * HALF, b_mn = n_blk * BN + int(rank) * G::B_ROWS;
          ptx::tma_load_2d_pair(ptx::smem_u32(sh.a + stage * A_STAGE_BYTES), &tmap_a, MN ? a_mn : kb * BK,
                                MN ? kb * BK : a_mn, fb);
          ptx::tma_load_2d_pair(ptx::smem_u32(sh.b + stage * B_STAGE_BYTES), &tmap_b, MN ? b_mn : kb * BK,
                                MN ? kb * BK : b_mn, fb);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // CTA 0 sees both CTAs' copies complete on its barriers; CTA 1 is held by the final
      // cluster barrier until CTA 0 got here
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) drain_wait(full_bar(s), (issued_parity >> s) & 1u, status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (CTA 0)
    if (lane == 0 && leader) {
      // ab_code: the A and B element format of kind::f8f6f4 (e4m3 0, e2m3 3, e3m2 4, e2m1 5)
      // bits 15 / 16: A / B MN-major
      const uint32_t idesc = instr_desc<FMT, BN_>() | (ab_code << 7) | (ab_code << 10) | (MN ? (3u << 15) : 0u);
      constexpr uint32_t kk_step = MN ? UMMA_K * 128 : UMMA_K;  // bytes between consecutive MMAs' slices
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int item = pair_id; item < num_items && ok; item += num_pairs) {
        const Item it = item_at(item);
        const int kb_begin = it.kb_begin, kb_end = it.kb_end;
        if (!wait_bounded(tempty_bar(acc), acc_phase ^ 1u, sh.abort_flag, status)) break;
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, sh.abort_flag, status)) { ok = false; break; }
          ptx::tc_fence_after_sync();
          const uint32_t a_addr = ptx::smem_u32(sh.a + stage * A_STAGE_BYTES);
          const uint32_t b_addr = ptx::smem_u32(sh.b + stage * B_STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint64_t ad = smem_desc_sw128(a_addr + kk * kk_step);
            const uint64_t bd = smem_desc_sw128(b_addr + kk * kk_step);
            const uint32_t accumulate = (kb > kb_begin || kk > 0) ? 1u : 0u;
            if (FMT == kInt8) ptx::mma_i8_pair(d_tmem, ad, bd, idesc, accumulate);
            else ptx::mma_f8_pair(d_tmem, ad, bd, idesc, accumulate);
          }
          ptx::tc_commit_pair_mc(empty_bar(stage), 0x3);  // both CTAs' stage is free
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        ptx::tc_commit_pair_mc(tfull_bar(acc), 0x3);  // both halves of the accumulator ready
        if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
      }
      ptx::tc_commit_pair(drain_bar);
      drain_wait(drain_bar, 0, status);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;  // the TMEM lanes this warp may read: 32 * quarter ..
    const int ew = warp - 2;       // epilogue warp 0 .. EPI_WARPS - 1
    const int chunk0 = (ew >> 2) * G::CHUNKS;  // first 64-column chunk of this warp's columns
    const float sab = (OUT != kOutAcc) ? __fmul_rn(*scale_a, *scale_b) : 0.0f;
    // bf16 output: chunk j (64 columns) of this warp's 32 rows goes TMEM -> registers -> a
    // swizzled 32 x 64 box in shared memory -> TMA store (asynchronous).  Box b of the warp's
    // NB boxes is rewritten only once the store that last used it has read it.  SHORT_K: the
    // warp's boxes hold its whole share of the tile; they are all written, made visible to the
    // TMA engine with one proxy fence and stored as one group.
    const uint32_t epi_base = ptx::smem_u32(sh.epi) + uint32_t(ew) * uint32_t(G::NB * G::BOX_BYTES);
    int box_group[G::NB];  // commit index of the store that last used each box (-1: none)
#pragma unroll
    for (int b = 0; b < G::NB; ++b) box_group[b] = -1;
    int ncommit = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int item = pair_id; item < num_items; item += num_pairs) {
      const Item it = item_at(item);
      int m_blk, n_blk;
      pair_tile_coords(it.tile, num_m, num_n, m_blk, n_blk);
      int ok = 0;
      if (lane == 0) ok = wait_bounded(tfull_bar(acc), acc_phase, sh.abort_flag, status) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      ptx::tc_fence_after_sync();
      const int row0 = m_blk * BM + int(rank) * HALF + quarter * 32;  // first row of this warp
      const uint32_t t_row = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN);
      if constexpr (OUT == kOutBf16) {
        // split contraction: publish this half's partial slab (32 rows x BN, stored so that a
        // warp's 16-byte stores are contiguous), then count it; the half that counts second
        // adds the other's partial to its own and writes the output, the first is done.
        const uint32_t* peer = nullptr;
        int* slab_counter = nullptr;
        bool emit = true;
        if (it.part) {
          const size_t slab_words = size_t(32) * BN;
          // [split tile][rank][quarter], the split tiles counted from split_from
          const size_t slab = size_t(it.tile - split_f) * 8 + size_t(rank) * 4 + quarter;
          uint32_t* mine = part_ws + (size_t(it.half) * split_t * 8 + slab) * slab_words;
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t r[32];
            ptx::tmem_ld_32x32b_x32(t_row + uint32_t(c * 32), r);
            ptx::tmem_ld_wait(r);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              ptx::st_global_cg_v4(mine + size_t((c * 8 + v) * 32 + lane) * 4, r[4 * v], r[4 * v + 1], r[4 * v + 2],
                                   r[4 * v + 3]);
          }
          __threadfence();
          __syncwarp();
          slab_counter = counters + slab;
          int prev = 0;
          if (lane == 0) prev = atomicAdd(slab_counter, 1);
          prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
          emit = prev == 1;
          if (emit) {
            __threadfence();  // the other half's partial is visible
            peer = part_ws + (size_t(1 - it.half) * split_t * 8 + slab) * slab_words;
          } else {  // the accumulator has been read: the MMA may reuse it
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(tempty_bar(acc), 0));
          }
        }
        if constexpr (G::WHOLE) {  // the previous tile's stores have read every box
          if (lane == 0 && ncommit > 0) ptx::bulk_wait_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < G::CHUNKS && emit; ++j) {
          uint32_t r0[32], r1[32];
          ptx::tmem_ld_32x32b_x32(t_row + uint32_t((chunk0 + j) * 64), r0);
          ptx::tmem_ld_32x32b_x32(t_row + uint32_t((chunk0 + j) * 64 + 32), r1);
          ptx::tmem_ld_wait(r0);
          ptx::reg_fence(r1);
          if (peer) {  // own + other half: one rounding per element (fp32) or exact (int32)
#pragma unroll
            for (int v = 0; v < 16; ++v) {
              const int c = 2 * j + (v >> 3);
              const uint4 q = ptx::ld_global_cg_v4(peer + size_t((c * 8 + (v & 7)) * 32 + lane) * 4);
              uint32_t* rr = (v < 8 ? r0 : r1) + 4 * (v & 7);
              const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                rr[e] = FMT == kInt8 ? rr[e] + qq[e] : __float_as_uint(__fadd_rn(__uint_as_float(rr[e]), __uint_as_float(qq[e])));
            }
          }
          if (j == G::CHUNKS - 1) {  // the accumulator has been read: the MMA may reuse it
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(tempty_bar(acc), 0));
          }
          const int b = j % G::NB;
          const uint32_t box = epi_base + uint32_t(b * G::BOX_BYTES);
          if constexpr (!G::WHOLE) {
            if (lane == 0 && box_group[b] >= 0) {
              if (ncommit - 1 - box_group[b] >= G::NB - 1) ptx::bulk_wait_read<G::NB - 1>();
              else ptx::bulk_wait_read<0>();
            }
            __syncwarp();
          }
          write_box_row<FMT>(box, lane, r0, r1, sab);
          if constexpr (!G::WHOLE) {
            ptx::fence_proxy_async_smem();  // the box is visible to the TMA engine
            __syncwarp();
            const int col0 = n_blk * BN + (chunk0 + j) * G::BOX_COLS;
            if (col0 < N && row0 < M) {  // boxes reaching past the edge are clipped by TMA
              if (lane == 0) {
                ptx::tma_store_2d(&tmap_out, box, col0, row0);
                ptx::bulk_commit();
              }
              box_group[b] = ncommit++;
            }
          }
        }
        if constexpr (G::WHOLE) {
          ptx::fence_proxy_async_smem();  // the boxes are visible to the TMA engine
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int j = 0; j < G::CHUNKS; ++j) {
              const int col0 = n_blk * BN + (chunk0 + j) * G::BOX_COLS;
              if (col0 < N && row0 < M)  // boxes reaching past the edge are clipped by TMA
                ptx::tma_store_2d(&tmap_out, epi_base + uint32_t(j * G::BOX_BYTES), col0, row0);
            }
            ptx::bulk_commit();
          }
          ++ncommit;
        }
        if (peer && lane == 0) *slab_counter = 0;  // both halves counted: ready for the next launch
      } else {
        const int64_t row = int64_t(row0) + lane;
        bool done = false;
        if constexpr (OUT == kOutF32 && BN_ == 256) {
          if (rot_k != 0) {
            const float c = __frsqrt_rn(static_cast<float>(rot_k));  // fp32(1/sqrt(k)), correctly rounded
            float* orow = reinterpret_cast<float*>(out) + row * N;
            const int cb = n_blk * BN;
            const bool rok = row < M;
            switch (rot_k) {
              case 16: epi_rot_cols<FMT, 16, BN_>(t_row, sab, c, orow, cb, rok, N); break;
              case 32: epi_rot_cols<FMT, 32, BN_>(t_row, sab, c, orow, cb, rok, N); break;
              case 64: epi_rot_cols<FMT, 64, BN_>(t_row, sab, c, orow, cb, rok, N); break;
              case 128: epi_rot_cols<FMT, 128, BN_>(t_row, sab, c, orow, cb, rok, N); break;
              default: epi_rot_cols256<FMT, BN_>(t_row, sab, c, orow, cb, rok, N); break;
            }
            done = true;
          }
        }
        if (!done) {
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t r[32];
            ptx::tmem_ld_32x32b_x32(t_row + uint32_t(c * 32), r);
            ptx::tmem_ld_wait();
            const int col0 = n_blk * BN + c * 32;
            if (row < M && col0 < N) store_chunk<FMT, OUT>(r, out, row, col0, N, sab);
          }
        }
        ptx::tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(tempty_bar(acc), 0));
      }
      if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
    }
    // every store of this warp has completed (and its shared memory been read) before exit
    if (OUT == kOutBf16 && lane == 0) ptx::bulk_wait<0>();
  }

  ptx::tc_fence_before_sync();
  ptx::cluster_sync();  // no CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace pair

}  // namespace gemm
}  // namespace hq
