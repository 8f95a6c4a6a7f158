// Both rotations of one bf16 matrix from a single read per pass: the block-Hadamard rotation
// along the columns (codes [rows][cols]) and along the rows (codes written transposed,
// [cols][rows]), each with its own tensor-wise absmax scale.
//
// Method: "Training Transformers with 4-bit Integers", section 3.3 (block-diagonal Hadamard
// rotation before quantization) and "HALO: Hadamard-Assisted Lower-Precision Optimization
// for LLMs" (Approach: every operand of the three linear-layer GEMMs is rotated along that
// GEMM's contraction dimension, so X, W and dY are each needed in two rotations; quantized
// rotated tensors are stored and reused).  The arithmetic is the same as in fwht_quant.cuh
// (Sylvester FWHT, index bit 0 first, fp32 round-to-nearest-even adds, normalisation by
// fp32(1/sqrt(k)), tensor-wise absmax, INT8 / e4m3 codes), so the codes are bit-identical to
// the single-rotation kernels'.
//
// Data movement: the tensor is cut into 256 x 256 tiles (a tile holds whole k-blocks in both
// directions for every k <= 256).  TMA streams each tile into shared memory as four 32 KB
// strips of 64 columns x 256 rows, through a 7-strip ring.  Eight warps read every strip
// twice from shared memory; the warp that is the last to finish with a strip issues the copy
// that refills its slot:
//   row role  (rotation along the columns): a thread takes 64 consecutive columns of one row
//             (one strip row), so in-block index bits 0..5 are register bits and bits 6, 7
//             are the strip, i.e. lane bits 3, 4;
//   col role  (rotation along the rows): four ldmatrix.trans x4 gathers per 32 rows give a
//             thread 64 consecutive rows of one column (bits 0..5 in registers, bits 6, 7 in
//             lane bits 0, 1).
// The absmax, INT8 and FP8 passes compute in the exchange layout of fwht_quant.cuh (xrotate:
// packed f32x2 butterflies, the lane bits brought into registers by swapping half of the
// registers with the partner lane, 32-byte code segments); the FP6 / FP4 code pass keeps
// butterfly shuffles across lanes (rotate64) and packs its codes per 16-code group.
// Pass 1 reduces both rotations' absmax into one partial per CTA and role; pass 2 reduces
// the partials, rotates again and writes both code tensors.  HBM traffic per element and
// pass is one 2-byte read (plus two 1-byte code writes in pass 2), against two reads when
// each rotation runs on its own.
//
// Shared-memory layout of a strip: the copy is a 3-D box over the view (col, a, b) of the
// tensor with row = 64a + b, dims ordered (col, a, b), so strip row rho = 4b + a holds tile
// row 64a + b.  With the 128-byte swizzle (16-byte chunk index XOR rho & 7) the eight rows
// one ldmatrix matrix reads (a = 0..3, b even/odd) and the eight rows one quarter-warp of
// the row role reads are in distinct chunks: both gathers are bank-conflict-free.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>
#include "fwht_quant.cuh"
#include "sm100_ptx.cuh"

namespace hq {
namespace dual {

// Eight warps at up to 255 registers each (no spills, 64 values per thread in flight) measured
// as fast as sixteen at 128 for k = 256 and faster for smaller k.  The step code also handles
// sixteen warps (two row steps and two column steps per warp and tile).
constexpr int kComputeWarps = 8;
static_assert(kComputeWarps == 8 || kComputeWarps == 16, "8 or 16 warps");
constexpr int kSteps = 32 / kComputeWarps;    // row steps and column steps per warp and tile
constexpr int kThreads = 32 * kComputeWarps;
constexpr int kTile = 256;                          // rows and columns of a tile
constexpr int kStripCols = 64;                      // 128 bytes of bf16 per strip row
constexpr int kStripsPerTile = kTile / kStripCols;  // 4
constexpr uint32_t kStripBytes = uint32_t(kTile) * kStripCols * 2;  // 32 KB
constexpr int kSlots = 7;                                           // strips in the ring
constexpr size_t kSmemBytes = 1024 + size_t(kSlots) * kStripBytes + kSlots * 8;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait

// Bounded wait: false once another warp raised the abort flag or after kWaitLimitNs (which
// raises the flag and records HQ_ERR_TIMEOUT).
__device__ __forceinline__ bool wait_full(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicCAS(status, 0u, 6u /* HQ_ERR_TIMEOUT */);
      return false;
    }
  }
}

// Rotation of a thread's 64 values (v[i] = positions 2i, 2i+1 of bits 0..5) for block size K:
// register stages for bits 0..min(log2 K, 6) - 1, then the lane stages (bit 6: lane xor m6,
// bit 7: lane xor m7).  ABSMAX: the last stage is folded into the running maxima `am` of the
// unnormalised |t| instead (v is left partly rotated); otherwise v ends fully rotated.
template <int K, bool ABSMAX>
__device__ __forceinline__ void rotate64(float2 (&v)[32], int lane, int m6, int m7, float (&am)[kAcc]) {
  if constexpr (K <= 64) {
    if constexpr (ABSMAX) {
      stages_low<K / 2, 32>(v);
      constexpr int h2 = K / 4;  // float2 distance of the last stage's pairs
      int n = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (i & h2) continue;
        am[n % kAcc] = max_abs_sums(am[n % kAcc], v[i].x, v[i + h2].x, v[i].y, v[i + h2].y);
        ++n;
      }
    } else {
      stages_low<K, 32>(v);
    }
  } else {
    stages_low<64, 32>(v);
    if constexpr (K == 256) stage_lanes<32>(v, m6, lane);
    const int ml = K == 256 ? m7 : m6;
    if constexpr (ABSMAX) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float px = __shfl_xor_sync(0xFFFFFFFFu, v[i].x, ml);
        const float py = __shfl_xor_sync(0xFFFFFFFFu, v[i].y, ml);
        am[i % kAcc] = max_abs_sums(am[i % kAcc], v[i].x, px, v[i].y, py);
      }
    } else {
      stage_lanes<32>(v, ml, lane);
    }
  }
}

// Codes of a thread's 64 rotated values, 64 contiguous bytes at dst (W32: two 32-byte stores,
// each a whole sector; dst 32-byte aligned).
template <int MODE, bool W32>
__device__ __forceinline__ void store_codes64(uint8_t* dst, const float2 (&v)[32], const CodeScale& cs, bool zero,
                                              int lp_fmt) {
  uint32_t w[16];
  if (cs.one_mul) {
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = codes4x<MODE>(mul2(v[2 * j], cs.ci2), mul2(v[2 * j + 1], cs.ci2), lp_fmt);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      w[j] = codes4x<MODE>(mul2(mul2(v[2 * j], cs.c2), cs.inv2), mul2(mul2(v[2 * j + 1], cs.c2), cs.inv2), lp_fmt);
  }
  if (zero) {
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = 0u;
  }
  if constexpr (MODE == kModeLowp) {
    // minifloats: four 16-code groups, each packed into its 16-byte chunk
    uint4 ch[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) ch[q] = lowp_pack16(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3], lp_fmt);
    if constexpr (W32) {
      st_global_32B(dst, ch[0].x, ch[0].y, ch[0].z, ch[0].w, ch[1].x, ch[1].y, ch[1].z, ch[1].w);
      st_global_32B(dst + 32, ch[2].x, ch[2].y, ch[2].z, ch[2].w, ch[3].x, ch[3].y, ch[3].z, ch[3].w);
    } else {
      uint4* o = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int q = 0; q < 4; ++q) o[q] = ch[q];
    }
  } else if constexpr (W32) {
    st_global_32B(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    st_global_32B(dst + 32, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
  } else {
    uint4* o = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float2& f) {
  f = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}


// ONCHIP (INT8 / FP8 codes; a cooperative launch of at most one CTA per SM and one tile per
// CTA): both passes in one launch.  Each CTA keeps its tile in shared memory, runs the absmax
// pass over it, writes its partial maxima, meets the other CTAs at a grid barrier on
// *grid_counter (zeroed by the host before the launch; every wait bounded), reduces all the
// partials and runs the code pass over the same resident tile: the source is read from HBM
// once, and there is one launch instead of two.
template <int K, int MODE, bool W32, bool SIGNED, bool ONCHIP = false>
__global__ void __launch_bounds__(kThreads, 1)
fwhtq_dual_kernel(const __grid_constant__ CUtensorMap map, int64_t rows, int64_t cols,
                  uint8_t* __restrict__ codes_c, uint8_t* __restrict__ codes_r,
                  float* __restrict__ part_c, float* __restrict__ part_r, int n_partials,
                  float* __restrict__ scale_c, float* __restrict__ scale_r,
                  unsigned int* __restrict__ status, int reverse,
                  const uint8_t* __restrict__ neg_c, const uint8_t* __restrict__ neg_r, int lp_fmt,
                  unsigned int* __restrict__ grid_counter) {
  // programmatic dependent launch: nothing is read or written before the previous grid in the
  // stream has completed; the next grid may be scheduled from here on
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  // SIGNED: sign flags per column (neg_c) and per row (neg_r); either may be null (all clear)
  static_assert(K >= 16 && K <= 256 && (K & (K - 1)) == 0, "k must be a power of two in [16,256]");
  static_assert(!ONCHIP || MODE == kModeInt8 || MODE == kModeFp8, "single-launch form: INT8 / FP8 codes");
  constexpr bool QUANT = MODE != kModeAbsmax;
  extern __shared__ uint8_t dsmem[];
  __shared__ float scratch[32];
  __shared__ float red[2 * kComputeWarps];
  __shared__ int abort_flag;
  __shared__ int grid_ok;  // ONCHIP: the grid barrier completed in time
  __shared__ unsigned int released[kSlots];  // warps done with the slot, over all rounds
  __shared__ int issued_round[kSlots];       // round of the slot's latest copy (-1: none)
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(base);
  const uint32_t bars = sbase + kSlots * kStripBytes;  // full[kSlots]
  auto full_bar = [&](int s) { return bars + 8u * s; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int64_t n_ct = (cols + kTile - 1) / kTile;
  const int64_t n_tiles = ((rows + kTile - 1) / kTile) * n_ct;
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t my_tiles = b < n_tiles ? (n_tiles - 1 - b) / G + 1 : 0;
  const int64_t n_strips = my_tiles * kStripsPerTile;
  // alternate passes walk the tiles in opposite orders, so each starts on what the previous
  // one left in L2
  auto tile_of = [&](int64_t i) { return reverse ? b + G * (my_tiles - 1 - i) : b + G * i; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      released[s] = 0u;
      issued_round[s] = -1;
    }
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int64_t q) {
    const int64_t t = tile_of(q / kStripsPerTile);
    const int s = static_cast<int>(q % kStripsPerTile);
    const int slot = static_cast<int>(q % kSlots);
    issued_round[slot] = static_cast<int>(q / kSlots);
    ptx::mbar_arrive_expect_tx(full_bar(slot), kStripBytes);
    ptx::tma_load_3d(sbase + slot * kStripBytes, &map, static_cast<int32_t>(kStripCols * (kStripsPerTile * (t % n_ct) + s)),
                     static_cast<int32_t>(4 * (t / n_ct)), 0, full_bar(slot));
  };
  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&map);
    for (int64_t q = 0; q < (n_strips < kSlots ? n_strips : kSlots); ++q) issue(q);
  }
  // A warp is done with strip q: the last of the kComputeWarps warps to say so for this use of
  // the slot refills it with strip q + kSlots.  Each warp's reads of the strip are ordered before its
  // count (syncwarp, then a CTA fence), and the counting warp's fence orders all of them
  // before its copy is issued.
  auto release = [&](int64_t q) {
    __syncwarp();
    if (lane == 0) {
      const int slot = static_cast<int>(q % kSlots);
      __threadfence_block();
      const unsigned int done = atomicAdd(&released[slot], 1u) + 1u;
      if (done == static_cast<unsigned int>(kComputeWarps) * static_cast<unsigned int>(q / kSlots + 1)) {
        __threadfence_block();
        ptx::fence_proxy_async_smem();
        if (q + kSlots < n_strips && !abort_flag) issue(q + kSlots);
      }
    }
  };

  const float c = __frsqrt_rn(static_cast<float>(K));
  QuantParams qc{0.0f, false, false}, qr{0.0f, false, false};
  if constexpr (QUANT && !ONCHIP) {
    qc = finish_absmax<MODE>(part_c, n_partials, scale_c, scratch, status, lp_fmt);
    qr = finish_absmax<MODE>(part_r, n_partials, scale_r, scratch, status, lp_fmt);
  }
  int64_t work_tiles = (qc.abort && qr.abort) ? 0 : my_tiles;

  CodeScale csc = code_scale<K>(c, qc.inv), csr = code_scale<K>(c, qr.inv);
  float amc[kAcc], amr[kAcc];
#pragma unroll
  for (int j = 0; j < kAcc; ++j) amc[j] = amr[j] = 0.0f;

  // row role lane constants: strip sr = lane >> 3, row selector x = lane & 7
  const int x = lane & 7, sr = lane >> 3;
  const uint32_t swr = 4u * (x & 1) + (x >> 1);
  // col role: the tile's 32 (strip, 8-column chunk) pairs p = warp + kComputeWarps * j go to
  // strip p >> 3, chunk p & 7 (the chunk is warp & 7 for every j); lane constants: matrix row
  // i = lane & 7 (same swizzle), matrix mm = lane >> 3
  const int grp = warp >> 3;
  const uint32_t col_lane_off = (8u * (lane >> 3) + swr) * 128u + ((static_cast<uint32_t>(warp & 7) ^ swr) << 4);
  // exchange layout (absmax, INT8, FP8 passes): chunk / gather swizzles and stage signs
  constexpr bool XL = MODE != kModeLowp;
  // row role: position bits 3, 4 of the loaded chunk XOR (A, B) = strip bits (k = 256), bit 4
  // XOR A (k = 128)
  const int row_sw = K == 256 ? sr : K == 128 ? 2 * (sr & 1) : 0;
  // col role: the receiving thread's swizzle (its lane bits 0, 1), and that of the thread
  // receiving the matrix row this lane addresses (row x of a matrix goes to lane bits x >> 1)
  const int col_sw = K == 256 ? (lane & 3) : K == 128 ? 2 * (lane & 1) : 0;
  const int col_sw_addr = K == 256 ? (x >> 1) : K == 128 ? 2 * ((x >> 1) & 1) : 0;
  const float rgA = (sr & 1) ? -1.0f : 1.0f, rgB = (sr & 2) ? -1.0f : 1.0f;
  const float cgA = (lane & 1) ? -1.0f : 1.0f, cgB = (lane & 2) ? -1.0f : 1.0f;
  const float2 rsA = make_float2(rgA, rgA), rnsA = make_float2(-rgA, -rgA);
  const float2 rsB = make_float2(rgB, rgB), rnsB = make_float2(-rgB, -rgB);
  const float2 csA = make_float2(cgA, cgA), cnsA = make_float2(-cgA, -cgA);
  const float2 csB = make_float2(cgB, cgB), cnsB = make_float2(-cgB, -cgB);

  // One sweep over this CTA's tiles: the absmax pass (Q false: both roles' running maxima)
  // or the code pass (Q true).
  auto sweep = [&](auto q_tag) {
    constexpr bool Q = decltype(q_tag)::value;
    for (int64_t i = 0; i < work_tiles; ++i) {
      const int64_t t = tile_of(i);
      const int64_t row0 = (t / n_ct) * kTile, col0 = (t % n_ct) * kTile;
      const int64_t q0 = i * kStripsPerTile;
      const int slot0 = static_cast<int>(q0 % kSlots);
      auto slot_of = [&](int s) { return slot0 + s < kSlots ? slot0 + s : slot0 + s - kSlots; };
      bool ok = true;
  #pragma unroll
      for (int s = 0; s < kStripsPerTile; ++s) {
        const int64_t q = q0 + s;
        ok = ok && wait_full(full_bar(slot_of(s)), static_cast<uint32_t>((q / kSlots) & 1), &abort_flag, status);
      }
      if (!ok) break;

      if constexpr (XL) {
        // ---- row role (exchange layout): a thread reads one strip row (64 columns) of its strip
        // sr; position bits 6, 7 of the column are lane bits 3, 4 (A = bit 3, B = bit 4)
        const uint32_t my_strip = sbase + static_cast<uint32_t>(slot_of(sr)) * kStripBytes;
  #pragma unroll 1
        for (int st = 0; st < kSteps; ++st) {
          const int g = warp + kComputeWarps * st;  // 0..31: tile rows {2g, 2g+1} + 64 * {0..3}
          const uint32_t rowaddr = my_strip + (8u * g + swr) * 128u;
          float2 v[32];
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t cq = static_cast<uint32_t>(q ^ row_sw);  // chunk of the x half; the y half's is 4 + cq
            uint4 rx = ptx::ld_shared_v4(rowaddr + ((cq ^ swr) << 4));
            uint4 ry = ptx::ld_shared_v4(rowaddr + (((4u + cq) ^ swr) << 4));
            if constexpr (SIGNED) {
              const int64_t c0 = col0 + kStripCols * sr + 8 * cq;
              uint32_t mx[4], my[4];
              const bool in = neg_c != nullptr && c0 < cols;
              sign_masks_bf16x8(in ? __ldg(reinterpret_cast<const uint2*>(neg_c + c0)) : make_uint2(0u, 0u), mx);
              sign_masks_bf16x8(in ? __ldg(reinterpret_cast<const uint2*>(neg_c + c0 + 32)) : make_uint2(0u, 0u), my);
              rx.x ^= mx[0]; rx.y ^= mx[1]; rx.z ^= mx[2]; rx.w ^= mx[3];
              ry.x ^= my[0]; ry.y ^= my[1]; ry.z ^= my[2]; ry.w ^= my[3];
            }
            const uint32_t wxq[4] = {rx.x, rx.y, rx.z, rx.w}, wyq[4] = {ry.x, ry.y, ry.z, ry.w};
            xunpack(q, wxq, wyq, v);
          }
          if (kSteps == 2 && st == 1) {
            release(q0 + 1 - grp);
            release(q0 + 3 - grp);
          }
          xrotate<K, !Q>(v, rsA, rnsA, rsB, rnsB, 8, 16, amc);
          if constexpr (Q) {
            const int64_t r = row0 + 64 * (x >> 1) + (x & 1) + 2 * g;
            if (!qc.abort) {  // uniform: every lane takes part in the code-word exchange
              const bool row_in = r < rows;
              uint32_t wx[8], wy[8];
              xcodes<MODE>(v, csc, qc.zero, wx, wy);
              // segment of half h: k <= 64 the thread's strip; k = 128 position bit 6 = A, bit 7 =
              // the strip's bit 1; k = 256 bits 6, 7 = the strip
              auto pos_of = [&](int h) -> int64_t {
                if constexpr (K <= 64) return int64_t(kStripCols) * sr + 32 * h;
                else if constexpr (K == 128) return 32 * h + 64 * (sr & 1) + 128 * (sr >> 1);
                else return 32 * h + 64 * sr;
              };
              auto ok_pos = [&](int64_t pc) { return row_in && col0 + pc < cols; };
              xstore<K>(codes_c + r * cols + col0, wx, wy, K == 256 ? sr : (sr & 1), 8, 16, pos_of, ok_pos, W32);
            }
          }
        }

        // ---- col role (exchange layout): ldmatrix.trans gathers; a thread receives rows of one
        // column whose position bits 6, 7 are its lane bits 0, 1 (A = bit 0, B = bit 1)
  #pragma unroll 1
        for (int j2 = 0; j2 < kSteps; ++j2) {
          const int s = grp + (kComputeWarps / 8) * j2;
          const uint32_t lbase = sbase + static_cast<uint32_t>(slot_of(s)) * kStripBytes + col_lane_off;
          float2 v[32];
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            // gather q of the x half reads call (q ^ sw) of 32 rows, the y half call 4 + (q ^ sw);
            // the swizzle is that of the thread receiving the row this lane addresses
            uint32_t rx[4], ry[4];
            ldmatrix_x4_trans(lbase + 4096u * static_cast<uint32_t>(q ^ col_sw_addr), rx);
            ldmatrix_x4_trans(lbase + 4096u * static_cast<uint32_t>(4 + (q ^ col_sw_addr)), ry);
            if constexpr (SIGNED) {
              const int64_t r0t = row0 + 64 * (lane & 3) + 8 * (q ^ col_sw);
              uint32_t mx[4], my[4];
              const bool in = neg_r != nullptr && r0t < rows;
              sign_masks_bf16x8(in ? __ldg(reinterpret_cast<const uint2*>(neg_r + r0t)) : make_uint2(0u, 0u), mx);
              sign_masks_bf16x8(in ? __ldg(reinterpret_cast<const uint2*>(neg_r + r0t + 32)) : make_uint2(0u, 0u), my);
  #pragma unroll
              for (int mm = 0; mm < 4; ++mm) {
                rx[mm] ^= mx[mm];
                ry[mm] ^= my[mm];
              }
            }
            xunpack(q, rx, ry, v);
          }
          release(q0 + s);
          xrotate<K, !Q>(v, csA, cnsA, csB, cnsB, 1, 2, amr);
          if constexpr (Q) {
            const int64_t gc = col0 + kStripCols * s + 8 * (warp & 7) + (lane >> 2);
            if (!qr.abort) {  // uniform: every lane takes part in the code-word exchange
              const bool col_in = gc < cols;
              uint32_t wx[8], wy[8];
              xcodes<MODE>(v, csr, qr.zero, wx, wy);
              const int a = lane & 3;
              auto pos_of = [&](int h) -> int64_t {
                if constexpr (K <= 64) return 64 * a + 32 * h;
                else if constexpr (K == 128) return 32 * h + 64 * (a & 1) + 128 * (a >> 1);
                else return 32 * h + 64 * a;
              };
              auto ok_pos = [&](int64_t pr) { return col_in && row0 + pr < rows; };
              xstore<K>(codes_r + gc * rows + row0, wx, wy, K == 256 ? a : (a & 1), 1, 2, pos_of, ok_pos, W32);
            }
          }
        }
      } else {
        // ---- row role: rotation along the columns, kSteps steps of 8 rows x 256 columns per warp
        const uint32_t my_strip = sbase + static_cast<uint32_t>(slot_of(sr)) * kStripBytes;
    #pragma unroll 1
        for (int st = 0; st < kSteps; ++st) {
          const int g = warp + kComputeWarps * st;  // 0..31: tile rows {2g, 2g+1} + 64 * {0..3}
          const uint32_t rowaddr = my_strip + (8u * g + swr) * 128u;
          // sign flags of the thread's 64 columns (the randomized variant; cols is a multiple of 64,
          // so they are all inside the tensor or all past its end)
          uint32_t sm[SIGNED ? 32 : 1];
        (void)sm;
          if constexpr (SIGNED) {
            const int64_t c0 = col0 + kStripCols * sr;
    #pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t m8[8];
              sign_masks_bf16x16(neg_c != nullptr && c0 < cols ? __ldg(reinterpret_cast<const uint4*>(neg_c + c0 + 16 * c))
                                                               : make_uint4(0u, 0u, 0u, 0u), m8);
    #pragma unroll
              for (int j = 0; j < 8; ++j) sm[8 * c + j] = m8[j];
            }
          }
          float2 v[32];
    #pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 raw = ptx::ld_shared_v4(rowaddr + ((static_cast<uint32_t>(j) ^ swr) << 4));
            if constexpr (SIGNED) {
              raw.x ^= sm[(4 * j) % (SIGNED ? 32 : 1)];
              raw.y ^= sm[(4 * j + 1) % (SIGNED ? 32 : 1)];
              raw.z ^= sm[(4 * j + 2) % (SIGNED ? 32 : 1)];
              raw.w ^= sm[(4 * j + 3) % (SIGNED ? 32 : 1)];
            }
            unpack_bf16x2(raw.x, v[4 * j]);
            unpack_bf16x2(raw.y, v[4 * j + 1]);
            unpack_bf16x2(raw.z, v[4 * j + 2]);
            unpack_bf16x2(raw.w, v[4 * j + 3]);
          }
          if (kSteps == 2 && st == 1) {
            // this warp's last reads of the two strips it has no column step on (with 16 warps a
            // warp's column steps cover strips grp and grp + 2; with 8 warps all four)
            release(q0 + 1 - grp);
            release(q0 + 3 - grp);
          }
          if constexpr (!Q) {
            rotate64<K, true>(v, lane, 8, 16, amc);
          } else {
            rotate64<K, false>(v, lane, 8, 16, amc);
            const int64_t r = row0 + 64 * (x >> 1) + (x & 1) + 2 * g;
            const int64_t cc = col0 + kStripCols * sr;
            if (!qc.abort && r < rows && cc < cols) store_codes64<MODE, W32>(codes_c + r * cols + cc, v, csc, qc.zero, lp_fmt);
          }
        }

        // ---- col role: rotation along the rows, 8 columns of one strip per step
    #pragma unroll 1
        for (int j2 = 0; j2 < kSteps; ++j2) {
          const int s = grp + (kComputeWarps / 8) * j2;
          const uint32_t lbase = sbase + static_cast<uint32_t>(slot_of(s)) * kStripBytes + col_lane_off;
          // sign flags of the thread's 64 rows (rows is a multiple of 64)
          uint32_t sm[SIGNED ? 32 : 1];
        (void)sm;
          if constexpr (SIGNED) {
            const int64_t r0t = row0 + 64 * (lane & 3);
    #pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t m8[8];
              sign_masks_bf16x16(neg_r != nullptr && r0t < rows ? __ldg(reinterpret_cast<const uint4*>(neg_r + r0t + 16 * c))
                                                                : make_uint4(0u, 0u, 0u, 0u), m8);
    #pragma unroll
              for (int j = 0; j < 8; ++j) sm[8 * c + j] = m8[j];
            }
          }
          float2 v[32];
    #pragma unroll
          for (int n = 0; n < 8; ++n) {
            uint32_t r4[4];
            ldmatrix_x4_trans(lbase + 4096u * n, r4);
    #pragma unroll
            for (int mm = 0; mm < 4; ++mm)
              unpack_bf16x2(SIGNED ? r4[mm] ^ sm[(4 * n + mm) % (SIGNED ? 32 : 1)] : r4[mm], v[4 * n + mm]);
          }
          release(q0 + s);
          if constexpr (!Q) {
            rotate64<K, true>(v, lane, 1, 2, amr);
          } else {
            rotate64<K, false>(v, lane, 1, 2, amr);
            const int64_t gc = col0 + kStripCols * s + 8 * (warp & 7) + (lane >> 2);
            const int64_t gr = row0 + 64 * (lane & 3);
            if (!qr.abort && gc < cols && gr < rows) store_codes64<MODE, W32>(codes_r + gc * rows + gr, v, csr, qr.zero, lp_fmt);
          }
        }
      }
    }

  };
  // The CTA's partial maxima of both rotations (the unnormalised |t| times fp32(1/sqrt(k)),
  // +inf when any rotated value was not finite).
  auto write_partials = [&]() {
    float mc = amc[0], mr = amr[0];
#pragma unroll
    for (int j = 1; j < kAcc; ++j) {
      mc = absmax3(mc, amc[j], 0.0f);
      mr = absmax3(mr, amr[j], 0.0f);
    }
    mc = mc != mc ? INFINITY : mc;
    mr = mr != mr ? INFINITY : mr;
    mc = warp_max(mc);
    mr = warp_max(mr);
    if (lane == 0) {
      red[warp] = mc;
      red[kComputeWarps + warp] = mr;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < kComputeWarps; ++w) {
        mc = fmaxf(mc, red[w]);
        mr = fmaxf(mr, red[kComputeWarps + w]);
      }
      mc = fmaxf(mc, red[0]);
      mr = fmaxf(mr, red[kComputeWarps]);
      part_c[b] = __fmul_rn(mc, c);
      part_r[b] = __fmul_rn(mr, c);
    }
  };

  if constexpr (ONCHIP) {
    sweep(std::false_type{});
    write_partials();
    // grid barrier: every CTA's partials are written before any CTA reduces them (each CTA
    // fences its write, then counts; all wait, bounded, for the count to reach the grid)
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      atomicAdd(grid_counter, 1u);
      const uint64_t t0 = ptx::globaltimer_ns();
      int ok = 1;
      while (*reinterpret_cast<volatile unsigned int*>(grid_counter) < gridDim.x) {
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
          atomicCAS(status, 0u, 6u /* HQ_ERR_TIMEOUT */);
          ok = 0;
          break;
        }
      }
      __threadfence();
      grid_ok = ok;
    }
    __syncthreads();
    if (grid_ok) {
      qc = finish_absmax<MODE, true>(part_c, static_cast<int>(gridDim.x), scale_c, scratch, status, lp_fmt);
      qr = finish_absmax<MODE, true>(part_r, static_cast<int>(gridDim.x), scale_r, scratch, status, lp_fmt);
    } else {
      qc.abort = qr.abort = true;
    }
    csc = code_scale<K>(c, qc.inv);
    csr = code_scale<K>(c, qr.inv);
    work_tiles = (qc.abort && qr.abort) ? 0 : my_tiles;
    sweep(std::true_type{});
  } else {
    sweep(std::integral_constant<bool, QUANT>{});
  }

  // every copy issued has landed before the CTA exits (all are consumed above unless a wait
  // gave up or both rotations were abandoned)
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      if (issued_round[s] < 0) continue;
      const uint32_t par = static_cast<uint32_t>(issued_round[s] & 1);
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(full_bar(s), par)) {
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
          atomicCAS(status, 0u, 6u);
          break;
        }
      }
    }
  }
  if constexpr (!QUANT) write_partials();
}

}  // namespace dual
}  // namespace hq
