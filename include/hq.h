/*
 * hq.h -- C ABI of libhq.so: Hadamard-rotated, tensor-wise quantized INT8 / FP8 linear layer
 * for NVIDIA B200 (sm_100a).
 *
 * The method (web pages on the subject):
 *  - "Training Transformers with 4-bit Integers", section 3.3 "Hadamard Quantization": both
 *    operands of a matmul are multiplied by a block-diagonal matrix of k x k Hadamard blocks
 *    H_k before quantization; the transform cancels in the product.  Section 3.1: symmetric
 *    integer range, integer product dequantized back to floating point by the scales.
 *  - "HALO: Hadamard-Assisted Lower-Precision Optimization for LLMs", "Approach": in the
 *    forward pass X and W are rotated on the right (along d_in); in the backward pass the
 *    output gradient is rotated on the left (along tokens) for the weight gradient (HALO-2);
 *    tensor-wise scales; INT8 or FP8 operands ("Key results", "Limitations").
 *
 * Besides the three rotated GEMMs of a layer: a backward placement that reuses the forward's
 * codes (hq_linear_fwd_keep / hq_linear_bwd_reuse), the next layer's rotation in a GEMM's
 * epilogue (hq_gemm_rotout / hq_quantize_prerotated), the randomized Hadamard variant (*_rht)
 * and the split quantization passes of quantized weight communication.
 *
 * Readings taken where the pages are silent (all implemented identically by the test oracle):
 *  - H_k is Sylvester's natural-order Hadamard matrix, normalised by fp32(1/sqrt(k)); the
 *    transform is an fp32 FWHT with stages h = 1, 2, ..., k/2, no fused multiply-add.
 *  - Every rotation runs along the contraction dimension of its GEMM (forward: K; dX: N;
 *    dW: the tokens M), with the same k everywhere.
 *  - Tensor-wise absmax a of the rotated tensor.  INT8: codes clamp(rne(y*fp32(127/a)),
 *    -127, 127), scale fp32(a/127).  FP8 (E4M3FN): codes e4m3_rne_satfinite(y*fp32(448/a)),
 *    scale fp32(a/448).  a == 0: scale 1, codes 0.
 *  - Epilogue: out = bf16_rne(fp32(acc) * fp32(scale_a * scale_b)).
 *
 * Conventions for every call:
 *  - All tensors are dense row-major device buffers owned by the caller; the library never
 *    allocates or frees memory.  Its only state, per device: the status word, the side
 *    stream and three events the multi-kernel layer calls fork to (created on first use),
 *    and hq_quantize_noalloc's fixed scratch array.
 *  - Every device pointer must be 16-byte aligned (else HQ_ERR_ALIGN).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream).
 *    Argument errors are returned synchronously before anything is launched.  Errors found
 *    on the device (non-finite operand, an internal wait that expired) are recorded in the
 *    status word and returned by hq_get_error(); outputs are unspecified after an error.
 *  - Codes take 1 byte per element (int8 two's complement, e4m3 bits, or the FP6 / FP4
 *    minifloats in the tensor cores' packed layout, see hq_fmt) and are stored with the rotated
 *    (contraction) dimension innermost.  Scales are one fp32 each, in device memory.
 *  - k is one of 16, 32, 64, 128, 256.
 */
#ifndef HQ_H_
#define HQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HQ_API __attribute__((visibility("default")))
#else
#define HQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* hq_stream_t;

typedef enum {
  HQ_OK = 0,
  HQ_ERR_ARG = 1,         /* null pointer, unknown enum value, negative size, bad k or dim */
  HQ_ERR_SHAPE = 2,       /* rotated dim not a multiple of k, other dim not a multiple of 16,
                             or a size limit exceeded */
  HQ_ERR_DTYPE = 3,       /* unknown source dtype */
  HQ_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
  HQ_ERR_NONFINITE = 5,   /* device: a rotated operand contained NaN or Inf */
  HQ_ERR_TIMEOUT = 6,     /* device: a bounded wait inside a kernel expired */
  HQ_ERR_CUDA = 7,        /* a CUDA runtime call failed (hq_last_cuda_error() tells which) */
  HQ_ERR_WORKSPACE = 8,   /* workspace pointer missing or smaller than required */
  HQ_ERR_UNSUPPORTED = 9  /* the current device is not sm_100 */
} hq_status;

/* Code formats.  Every code is one byte; the scale is fp32(a / max) with a the tensor's absmax.
 *   HQ_INT8      symmetric integers -127..127 (max 127), GEMM on kind::i8, int32 accumulators
 *   HQ_FP8_E4M3  E4M3FN (max 448), kind::f8f6f4, fp32 accumulators
 *   HQ_FP6_E3M2  FP6 sign | 3 exponent (bias 3) | 2 mantissa, max 28, value in bits 5..0
 *   HQ_FP6_E2M3  FP6 sign | 2 exponent (bias 1) | 3 mantissa, max 7.5, value in bits 5..0
 *   HQ_FP4_E2M1  FP4 sign | 2 exponent (bias 1) | 1 mantissa, max 6, value in bits 3..0
 * FP6 and FP4 are the formats HALO names below FP8 (its GPUs had no FP6 matmul, so it
 * lower-bounded them with FP8); B200's kind::f8f6f4 multiplies them directly, one code per
 * byte in shared memory.  The minifloats have subnormals and no infinities or NaN; codes are
 * nearest-even with saturation to +-max, the upper bits of each byte zero. */
typedef enum {
  HQ_INT8 = 0,
  HQ_FP8_E4M3 = 1,
  HQ_FP6_E3M2 = 2,
  HQ_FP6_E2M3 = 3,
  HQ_FP4_E2M1 = 4
} hq_fmt;
typedef enum { HQ_F32 = 0, HQ_BF16 = 1 } hq_dtype;
typedef enum {
  HQ_OUT_BF16 = 0, /* dequantized bf16 */
  HQ_OUT_ACC = 1   /* raw accumulators: int32 for HQ_INT8, fp32 for HQ_FP8_E4M3 */
} hq_out;

/* Largest contraction length the INT8 path accepts: 127*127*K must stay below 2^31 so the
 * int32 accumulator cannot overflow. */
#define HQ_MAX_K_INT8 133143

/* ------------------------------------------------------------------------------------------
 * hq_quantize -- rotate a matrix along one dimension with blockdiag(H_k)/sqrt(k) and quantize
 * it tensor-wise ("Training Transformers with 4-bit Integers", section 3.3; HALO "Approach").
 *
 *   src     [rows][cols], dtype `dt` (fp32 or bf16).
 *   dim     1: rotate along cols (cols % k == 0);  codes are [rows][cols].
 *           0: rotate along rows (rows % k == 0);  codes are [cols][rows] (transposed so the
 *              rotated dimension is innermost); cols must be a multiple of 16.
 *   codes   rows*cols bytes, device.      scale   1 fp32, device (dequantization step).
 *   workspace / ws_bytes: >= hq_quantize_workspace_bytes() bytes of device scratch (partial
 *           maxima); contents need no initialisation and are not preserved.
 * Runs two kernels on `stream`: rotation + absmax partials, then rotation + codes.
 * rows == 0 or cols == 0 writes scale = 1 and no codes.
 * ---------------------------------------------------------------------------------------- */
HQ_API size_t hq_quantize_workspace_bytes(void);
HQ_API hq_status hq_quantize(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k,
                      hq_fmt fmt, void* codes, float* scale, void* workspace, size_t ws_bytes,
                      hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * hq_gemm -- low-precision GEMM on the tcgen05 tensor cores with the dequantization epilogue
 * ("Training Transformers with 4-bit Integers", section 3.1: INT32 product dequantized).
 *
 *   A [M][K] codes, B [N][K] codes (both contraction-innermost, as hq_quantize writes them),
 *   scale_a / scale_b: device fp32 scalars (may be NULL when out_kind == HQ_OUT_ACC).
 *   out [M][N]: bf16  = bf16(fp32(acc) * fp32(scale_a*scale_b))   (HQ_OUT_BF16)
 *               int32 / fp32 raw accumulators                     (HQ_OUT_ACC)
 *   K and N must be multiples of 16 (K <= HQ_MAX_K_INT8 for INT8); M is free.
 *   K == 0 writes zeros; M == 0 or N == 0 does nothing.
 * ---------------------------------------------------------------------------------------- */
HQ_API hq_status hq_gemm(const void* A, const float* scale_a, const void* B, const float* scale_b,
                  int64_t M, int64_t N, int64_t K, hq_fmt fmt, hq_out out_kind, void* out,
                  hq_stream_t stream);

/* hq_gemm_ws -- hq_gemm with device scratch for splitting tiles along the contraction (the
 * layer calls use the same).  With at least hq_gemm_workspace_bytes(M, N, K) bytes (16-byte
 * aligned; contents need no initialisation and are not preserved) a bf16-output GEMM whose
 * last wave of 256 x 256 tiles fills at most half the CTA pairs splits those tiles in two
 * halves of the k-blocks, and one with too few tiles for the pairs splits all of them; each
 * half's fp32 / int32 partial is added to the other's once (INT8 results are unchanged, FP8
 * ones round once more).  A NULL workspace, or a smaller one, runs hq_gemm. */
HQ_API size_t hq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
HQ_API hq_status hq_gemm_ws(const void* A, const float* scale_a, const void* B, const float* scale_b,
                            int64_t M, int64_t N, int64_t K, hq_fmt fmt, hq_out out_kind, void* out,
                            void* workspace, size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * The three GEMMs of one linear layer Y = X W^T with M tokens, K = d_in, N = d_out, each
 * with both operands rotated along its contraction dimension and quantized tensor-wise
 * (HALO-2: right-hand rotation of X and W forward, left-hand rotation of dY for dW).
 *   X [M][K], W [N][K], dY [M][N] in dtype `dt`; outputs bf16.
 *   M, K, N: multiples of k (and of 16).
 *   workspace: >= hq_linear_workspace_bytes(M, K, N) bytes of device scratch (codes, scales,
 *   partial maxima); no initialisation needed, not preserved between calls.
 * Each call launches 5 kernels on `stream` (2 per quantization + the GEMM).
 * ---------------------------------------------------------------------------------------- */
HQ_API size_t hq_linear_workspace_bytes(int64_t M, int64_t K, int64_t N);

/* One workspace size for every layer-level call of a shape: the largest of
 * hq_linear_workspace_bytes, hq_linear_fwd_bwd_workspace_bytes, the saved-codes pair
 * (hq_linear_fwd_save / hq_linear_bwd) and the reuse placement (hq_linear_fwd_keep /
 * hq_linear_bwd_reuse) for M, K, N.  Every code format stores one byte per element, so `fmt`
 * only has to be a valid format; 0 for negative sizes or an unknown format. */
HQ_API size_t hq_workspace_bytes(int64_t M, int64_t K, int64_t N, hq_fmt fmt);

/* Y[M][N] = (X H)(W H)^T: X and W rotated along K.  The forward that also keeps X's codes
 * rotated along the tokens for the weight gradient (the HALO training flow, where the
 * activation is stored quantized) is the separate call hq_linear_fwd_save; its backward,
 * which takes those codes instead of X, is hq_linear_bwd. */
HQ_API hq_status hq_linear_fwd(const void* X, const void* W, hq_dtype dt, int64_t M, int64_t K,
                        int64_t N, int k, hq_fmt fmt, void* Y, void* workspace, size_t ws_bytes,
                        hq_stream_t stream);

/* dX[M][K] = (dY H)(W^T H)^T: dY rotated along N (its columns), W along N (its rows). */
HQ_API hq_status hq_linear_bwd_dx(const void* dY, const void* W, hq_dtype dt, int64_t M, int64_t K,
                           int64_t N, int k, hq_fmt fmt, void* dX, void* workspace,
                           size_t ws_bytes, hq_stream_t stream);

/* dW[N][K] = (dY^T H)(X^T H)^T: dY and X rotated along the tokens M (left-hand rotation). */
HQ_API hq_status hq_linear_bwd_dw(const void* dY, const void* X, hq_dtype dt, int64_t M, int64_t K,
                           int64_t N, int k, hq_fmt fmt, void* dW, void* workspace,
                           size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * hq_quantize_dual -- both rotations of one matrix in one call ("HALO" Approach: quantized
 * rotated tensors are kept and reused; each operand of the layer is needed rotated along each
 * of its two dimensions).  Results are bit-identical to two hq_quantize calls:
 *   codes_c [rows][cols] + scale_c: rotated along cols  (hq_quantize dim = 1)
 *   codes_r [cols][rows] + scale_r: rotated along rows  (hq_quantize dim = 0)
 * rows and cols must both be multiples of k.  For a bf16 source with rows and cols multiples
 * of 64 one kernel computes both rotations from a single read of each 256 x 256 tile per pass
 * (2 launches: both absmax partials, then both code tensors).  When the tensor has at most one
 * such tile per SM and the codes are INT8 or FP8, both passes run in one cooperative launch over
 * tiles kept in shared memory, with a grid barrier between the passes (the source is read from
 * HBM once; the barrier's counter is the workspace's last 4 bytes of the first partial array,
 * zeroed by the call, and its wait is bounded: HQ_ERR_TIMEOUT, no codes, if it expires).
 * Otherwise the four single-rotation passes run back to back in alternating directions so that
 * after the first one most source reads are served by L2.  workspace: >=
 * hq_quantize_dual_workspace_bytes() bytes.
 * Device-side errors as for hq_quantize, per rotation (a rotation whose absmax is not finite
 * writes no codes and a NaN scale; the other rotation is still written).
 * ---------------------------------------------------------------------------------------- */
HQ_API size_t hq_quantize_dual_workspace_bytes(void);
HQ_API hq_status hq_quantize_dual(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int k,
                                  hq_fmt fmt, void* codes_c, float* scale_c, void* codes_r,
                                  float* scale_r, void* workspace, size_t ws_bytes,
                                  hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * hq_linear_fwd_bwd -- the whole layer step: Y = X W^T, dX = dY W and dW = dY^T X, each GEMM
 * on operands rotated along its contraction dimension, every operand rotation computed once
 * (six rotations in five quantization calls + three GEMMs, 13 kernels).  Outputs equal those
 * of hq_linear_fwd, hq_linear_bwd_dx and hq_linear_bwd_dw bit for bit.
 *   X [M][K], W [N][K], dY [M][N] (dtype dt); Y [M][N], dX [M][K], dW [N][K] bf16.
 *   M, K, N: positive multiples of k.  workspace: >= hq_linear_fwd_bwd_workspace_bytes().
 * dY in both rotations (one two-rotation call, as hq_quantize_dual) runs on a per-device side
 * stream that the library creates on first use (with three events) and forks from / joins back
 * to `stream` with events.  When X and W are bf16 with both dimensions >= 2048 (and multiples
 * of 64) and k <= 128, each is quantized in both rotations by one two-rotation call on `stream`, followed by
 * the three GEMMs, the backward ones after dY's codes have landed.  Otherwise X and W along K
 * and the forward GEMM run on `stream` while the side stream also quantizes W along N and X
 * along M; the dX GEMM waits only for dY along N and W along N, X along M lands while it runs
 * and the dW GEMM waits for it.  Everything is complete when `stream` reaches the end of the
 * call.
 * ---------------------------------------------------------------------------------------- */
HQ_API size_t hq_linear_fwd_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N);
HQ_API hq_status hq_linear_fwd_bwd(const void* X, const void* W, const void* dY, hq_dtype dt,
                                   int64_t M, int64_t K, int64_t N, int k, hq_fmt fmt, void* Y,
                                   void* dX, void* dW, void* workspace, size_t ws_bytes,
                                   hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Randomized Hadamard variant: a sign diagonal D applied before the blocks, t = H_k D x
 * (the randomized Hadamard transform of the neighbouring methods listed beside the pages'
 * subject, e.g. QuIP#'s incoherence processing; the two source pages use plain H).  D is
 * given per rotated dimension as device arrays of one byte per position, bit 0 set = that
 * position is negated (an exact sign flip of the source before the same fp32 butterflies).
 * Both operands of a GEMM must use the same D along its contraction dimension; D^2 = I then
 * cancels in the product exactly like H.  The flags are the caller's random draws (the
 * library draws nothing).  A NULL vector is the plain rotation (all flags clear).
 *   neg arrays: 16-byte aligned (HQ_ERR_ALIGN), length = the rotated dimension (not checked).
 *
 * hq_quantize_rht      -- hq_quantize with flags `neg` over the rotated dimension (cols for
 *                         dim = 1, rows for dim = 0).
 * hq_quantize_dual_rht -- hq_quantize_dual with flags neg_c over the columns (for codes_c)
 *                         and neg_r over the rows (for codes_r).
 * hq_linear_fwd_bwd_rht -- hq_linear_fwd_bwd with one sign vector per contraction dimension:
 *                         neg_k [K] (X and W for the forward GEMM), neg_n [N] (dY and W for
 *                         dX), neg_m [M] (dY and X for dW).
 * Errors, workspaces and launches as for the plain calls.
 * ---------------------------------------------------------------------------------------- */
HQ_API hq_status hq_quantize_rht(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim,
                                 int k, hq_fmt fmt, const uint8_t* neg, void* codes, float* scale,
                                 void* workspace, size_t ws_bytes, hq_stream_t stream);
HQ_API hq_status hq_quantize_dual_rht(const void* src, hq_dtype dt, int64_t rows, int64_t cols,
                                      int k, hq_fmt fmt, const uint8_t* neg_c, const uint8_t* neg_r,
                                      void* codes_c, float* scale_c, void* codes_r, float* scale_r,
                                      void* workspace, size_t ws_bytes, hq_stream_t stream);
HQ_API hq_status hq_linear_fwd_bwd_rht(const void* X, const void* W, const void* dY, hq_dtype dt,
                                       int64_t M, int64_t K, int64_t N, int k, hq_fmt fmt,
                                       const uint8_t* neg_k, const uint8_t* neg_n,
                                       const uint8_t* neg_m, void* Y, void* dX, void* dW,
                                       void* workspace, size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Sharded quantization (quantized FSDP weight communication, "HALO" HQ-FSDP): each rank holds
 * a slice of a tensor and must quantize it with the tensor-wise scale of the WHOLE tensor,
 * then all-gather 1-byte codes instead of 2-byte bf16 values.  The two passes of hq_quantize
 * are split so that the absmax can be reduced across ranks in between (e.g. an NCCL
 * all-reduce MAX on the device scalar):
 *
 * hq_quantize_absmax -- pass 1 only: *absmax = max |y| of the rotation of src (device fp32
 *   scalar; +inf if a rotated value is not finite).  Slices along the non-rotated dimension,
 *   or along the rotated one in multiples of k, have whole blocks each: the maximum of their
 *   absmax values is the whole tensor's.  workspace >= hq_quantize_workspace_bytes().
 * hq_quantize_codes -- pass 2 from a given absmax (device scalar, read only): codes and
 *   scale equal to hq_quantize of the whole tensor restricted to this slice, bit for bit.
 *   A non-finite absmax sets HQ_ERR_NONFINITE and writes no codes (scale NaN), an absmax of 0
 *   gives zero codes and scale 1.
 * neg: optional sign flags of the randomized variant (as hq_quantize_rht), NULL = plain.
 * Both calls enqueue on `stream`; argument errors as for hq_quantize.
 * ---------------------------------------------------------------------------------------- */
HQ_API hq_status hq_quantize_absmax(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim,
                                    int k, const uint8_t* neg, float* absmax, void* workspace,
                                    size_t ws_bytes, hq_stream_t stream);
HQ_API hq_status hq_quantize_codes(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim,
                                   int k, hq_fmt fmt, const uint8_t* neg, const float* absmax,
                                   void* codes, float* scale, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Training flow with saved codes ("HALO" Approach: the quantized rotated tensors are kept for
 * the backward pass instead of the bf16 activation, which halves the activation memory).
 *
 * hq_linear_fwd_save -- Y = X W^T like hq_linear_fwd, and in the same call X rotated along the
 * tokens M and quantized: xqt_codes [K][M] (1 byte per element, M innermost) and the device
 * scalar *xqt_scale, exactly the codes and scale hq_quantize(X, dim = 0) gives.  Keep them
 * for hq_linear_bwd; X itself is then not needed after the forward.
 *   X [M][K], W [N][K] (dtype dt); Y [M][N] bf16; M, K, N positive multiples of k.
 *   workspace: >= hq_linear_fwd_save_workspace_bytes(M, K, N) bytes (not preserved).
 * X is quantized in both rotations at once (as in hq_quantize_dual) on `stream` while W along
 * K runs on the library's per-device side stream (see hq_linear_fwd_bwd); all outputs are
 * complete when `stream` reaches the end of the call.
 *
 * hq_linear_bwd -- dX = dY W and dW = dY^T X from the saved codes: dY is quantized once in
 * both rotations (along N for dX, along M for dW, as in hq_quantize_dual) on `stream` while
 * W along N runs on the side stream, then the two GEMMs.  Outputs equal those of hq_linear_bwd_dx and hq_linear_bwd_dw (the
 * latter given the X the codes came from) bit for bit.
 *   dY [M][N], W [N][K] (dtype dt); xqt_codes [K][M] and xqt_scale from hq_linear_fwd_save
 *   with the same M, K, k and fmt (not checked: the library cannot tell codes apart);
 *   dX [M][K], dW [N][K] bf16.  workspace: >= hq_linear_bwd_workspace_bytes(M, K, N).
 * Errors: as hq_linear_fwd_bwd; a null xqt_codes or xqt_scale is HQ_ERR_ARG.
 * ---------------------------------------------------------------------------------------- */
HQ_API size_t hq_linear_fwd_save_workspace_bytes(int64_t M, int64_t K, int64_t N);
HQ_API hq_status hq_linear_fwd_save(const void* X, const void* W, hq_dtype dt, int64_t M,
                                    int64_t K, int64_t N, int k, hq_fmt fmt, void* Y,
                                    void* xqt_codes, float* xqt_scale, void* workspace,
                                    size_t ws_bytes, hq_stream_t stream);
HQ_API size_t hq_linear_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N);
HQ_API hq_status hq_linear_bwd(const void* dY, const void* W, const void* xqt_codes,
                               const float* xqt_scale, hq_dtype dt, int64_t M, int64_t K,
                               int64_t N, int k, hq_fmt fmt, void* dX, void* dW, void* workspace,
                               size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Backward placement that reuses the forward's codes ("HALO: Hadamard-Assisted Lower-Precision
 * Optimization for LLMs", Approach: quantized rotated tensors of the forward pass are reused,
 * and the output gradient gets a left-hand Hadamard; "Training Transformers with 4-bit
 * Integers", section 4: the backward GEMMs quantize only the output gradient and reuse the
 * forward's quantized activations and weights).
 *
 * With Wq = Q(W H) from the forward (rotated along K) and G = Q(H dY) (dY rotated along the
 * tokens M, quantized once), H symmetric and orthonormal:
 *   dW = G^T-contraction with the saved X codes (as hq_linear_bwd's dW, rotation along M);
 *   dX = dY W = H (H dY)(W H) H  ~  H [ fp32(sum_n G[n][m] Wq[n][j]) * fp32(s_g * s_w) ] H,
 * the GEMM reading both code tensors as stored (contraction outermost), then both rotations
 * undone on the fp32 output: along its columns (K) in k-blocks, then along its rows (M), each
 * as the library's rotation (butterflies, then x fp32(1/sqrt(k))), one bf16 rounding at the
 * end.  One quantization of dY and none of W in the backward: four rotations per layer step
 * instead of six.  Formats: HQ_INT8 and HQ_FP8_E4M3 only (the tensor cores read operands with
 * the contraction outermost only for 8-bit formats); others are HQ_ERR_ARG.
 *
 * hq_linear_fwd_keep -- hq_linear_fwd_save that also hands back W's codes along K:
 *   wq_codes [N][K] (1 byte per element) and the device scalar *wq_scale, exactly what
 *   hq_quantize(W, dim = 1) gives.  workspace: >= hq_linear_fwd_keep_workspace_bytes(M, K, N).
 *   Errors: as hq_linear_fwd_save; a null wq_codes or wq_scale is HQ_ERR_ARG.
 *
 * hq_linear_bwd_dx_reuse -- dX [M][K] bf16 from g_codes [N][M] (dY rotated along M, as
 *   hq_quantize(dY, dim = 0) writes them) with scale *g_scale, and wq_codes [N][K] with
 *   *wq_scale.  M and K multiples of k; N (the contraction) >= 1, at most HQ_MAX_K_INT8 for
 *   INT8.  workspace: >= hq_linear_bwd_dx_reuse_workspace_bytes(M, K, N) bytes (the fp32
 *   output before its de-rotation, 4 M K bytes; not preserved).  Three kernels on `stream`.
 *
 * hq_linear_bwd_reuse -- dX and dW of one layer from dY [M][N] (dtype dt), the saved
 *   xqt_codes [K][M] / *xqt_scale of hq_linear_fwd_save / _keep and the kept wq_codes [N][K] /
 *   *wq_scale: dY quantized once along M, the dX GEMM, then the dW GEMM on `stream` while the
 *   de-rotation of dX's rows runs on the library's side stream (see hq_linear_fwd_bwd); all
 *   outputs are complete when `stream` reaches the end of the call.  Shape rules as
 *   hq_linear_fwd_bwd.  workspace: >= hq_linear_bwd_reuse_workspace_bytes(M, K, N).  dW equals
 *   hq_linear_bwd's bit for bit, dX hq_linear_bwd_dx_reuse's.
 * ---------------------------------------------------------------------------------------- */
HQ_API size_t hq_linear_fwd_keep_workspace_bytes(int64_t M, int64_t K, int64_t N);
HQ_API hq_status hq_linear_fwd_keep(const void* X, const void* W, hq_dtype dt, int64_t M,
                                    int64_t K, int64_t N, int k, hq_fmt fmt, void* Y,
                                    void* xqt_codes, float* xqt_scale, void* wq_codes,
                                    float* wq_scale, void* workspace, size_t ws_bytes,
                                    hq_stream_t stream);
HQ_API size_t hq_linear_bwd_dx_reuse_workspace_bytes(int64_t M, int64_t K, int64_t N);
HQ_API hq_status hq_linear_bwd_dx_reuse(const void* g_codes, const float* g_scale,
                                        const void* wq_codes, const float* wq_scale, int64_t M,
                                        int64_t K, int64_t N, int k, hq_fmt fmt, void* dX,
                                        void* workspace, size_t ws_bytes, hq_stream_t stream);
HQ_API size_t hq_linear_bwd_reuse_workspace_bytes(int64_t M, int64_t K, int64_t N);
HQ_API hq_status hq_linear_bwd_reuse(const void* dY, hq_dtype dt, const void* xqt_codes,
                                     const float* xqt_scale, const void* wq_codes,
                                     const float* wq_scale, int64_t M, int64_t K, int64_t N,
                                     int k, hq_fmt fmt, void* dX, void* dW, void* workspace,
                                     size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * The next layer's rotation in this GEMM's epilogue ("Training Transformers with 4-bit
 * Integers", section 3.3: the Hadamard blocks come before quantization; "HALO: Hadamard-Assisted
 * Lower-Precision Optimization for LLMs", Approach).  When a GEMM's output is the next
 * GEMM's operand along its columns (a linear map with nothing nonlinear in between), the
 * producing GEMM can apply that rotation while its accumulators are in registers, and the
 * next operand is then only quantized.
 *
 * hq_gemm_rotout -- out [M][N] fp32 = blockdiag(H_k / sqrt(k)) along the columns of
 *   fp32(sum_l A[i][l] B[j][l]) * fp32(scale_a * scale_b).  A [M][K], B [N][K] codes (both
 *   contraction-innermost, as hq_gemm), device scales; N % k == 0.  Arithmetic as the
 *   library's rotation: butterflies h = 1 .. k/2 (index bit 0 first), then x fp32(1/sqrt(k)).
 *   Formats HQ_INT8 and HQ_FP8_E4M3 (others HQ_ERR_ARG).  Errors as hq_gemm.
 *
 * hq_quantize_prerotated -- tensor-wise codes of rotated values y [rows][cols] fp32 (no
 *   transform): a = max |y|, codes RNE(fp32(y * fp32(QMAX / a))), *scale = fp32(a / QMAX),
 *   exactly the steps hq_quantize takes after its rotation.  cols % 16 == 0.  Formats HQ_INT8
 *   and HQ_FP8_E4M3.  workspace: >= hq_quantize_prerotated_workspace_bytes() bytes.  A
 *   non-finite a sets HQ_ERR_NONFINITE in the status word and writes no codes.
 * ---------------------------------------------------------------------------------------- */
HQ_API hq_status hq_gemm_rotout(const void* A, const float* scale_a, const void* B,
                                const float* scale_b, int64_t M, int64_t N, int64_t K, int k,
                                hq_fmt fmt, float* out, hq_stream_t stream);
HQ_API size_t hq_quantize_prerotated_workspace_bytes(void);
HQ_API hq_status hq_quantize_prerotated(const float* y, int64_t rows, int64_t cols, hq_fmt fmt,
                                        void* codes, float* scale, void* workspace,
                                        size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * hq_quantize_noalloc -- hq_quantize for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call: it exists for integration only.  Some callers
 * receive nothing but their input and output buffers and may not allocate: plugin code run
 * inside another engine's execution step, code under a fixed device-memory budget, or code
 * on a latency-critical path where cudaMalloc (which can synchronise the device and can fail
 * when memory is fragmented) is not allowed.  Such a caller cannot provide the scratch that
 * hq_quantize takes as `workspace`.
 *
 * Same arguments, results and errors as hq_quantize, without the workspace.  Its scratch (the
 * per-CTA partial maxima of the absmax pass) lives in a fixed array inside the library:
 * HQ_NOALLOC_MAX_PARTIALS fp32 values (16 KiB), held on every GPU that loads the library until
 * the process exits.  The quantizer never launches more CTAs than that on current parts; a
 * launch that would need more partials than the array holds is refused with
 * HQ_ERR_WORKSPACE, and sizes beyond hq_quantize's own limits get the same errors as there.
 * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 *
 * The first call on a device looks up the array's device address (once per device, with
 * that device current); make that first call before any stream capture.  All calls share
 * the one array and it keeps the last call's contents (nothing in it needs clearing between
 * calls: each call writes every entry it later reads).  Calls whose kernels overlap on the
 * GPU race on the array: run them on one stream, or otherwise order them.
 * ---------------------------------------------------------------------------------------- */
#define HQ_NOALLOC_MAX_PARTIALS 4096
HQ_API hq_status hq_quantize_noalloc(const void* src, hq_dtype dt, int64_t rows, int64_t cols,
                                     int dim, int k, hq_fmt fmt, void* codes, float* scale,
                                     hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * hq_selftest_gemm_timeout -- test hook for the device-side failure path (no counterpart on
 * the pages).  Runs the single-CTA INT8 GEMM (raw accumulators) on caller buffers
 * A [M][K], B [N][K], out [M][N] int32 with its first pipeline stage deliberately left
 * un-armed: the MMA warp's bounded wait on it expires after about one second, the kernel
 * records HQ_ERR_TIMEOUT in the status word, every role stops, copies and MMAs in flight
 * are drained, tensor memory is freed and the kernel returns.  hq_get_error() then reports
 * HQ_ERR_TIMEOUT and the CUDA context stays usable.  out is unspecified.
 * Shapes as hq_gemm, each of M, N, K at most 4096.
 * ---------------------------------------------------------------------------------------- */
HQ_API hq_status hq_selftest_gemm_timeout(const void* A, const void* B, void* out, int64_t M,
                                          int64_t N, int64_t K, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * hq_mma_peak -- dense tensor-core throughput probe (no counterpart on the pages; it measures
 * the roofline denominator of the GEMMs on the device at hand).
 *
 * Runs one CTA pair per TPC (2 * floor(SMs / 2) CTAs), each pair issuing n_blocks x 4
 * back-to-back tcgen05.mma.cta_group::2 instructions (M = 256, N = 256, K = 32: 4,194,304
 * operations each) of kind::i8 (fmt HQ_INT8) or kind::f8f6f4 with e4m3 operands
 * (HQ_FP8_E4M3) on operand tiles resident in shared memory, accumulating in tensor memory:
 * no global-memory traffic.  The caller times the launch (CUDA events on `stream`); the
 * operation count is pairs * n_blocks * 4 * 4,194,304, with pairs from *pairs_out (may be
 * NULL).  1 <= n_blocks <= 2^24 (at most a few seconds); other formats give HQ_ERR_ARG.
 * ---------------------------------------------------------------------------------------- */
HQ_API hq_status hq_mma_peak(hq_fmt fmt, int64_t n_blocks, int* pairs_out, hq_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Status.
 * ---------------------------------------------------------------------------------------- */
/* Synchronises `stream`, then returns and clears the current device's status word (HQ_OK,
 * HQ_ERR_NONFINITE or HQ_ERR_TIMEOUT), or HQ_ERR_CUDA if the stream reported an error. */
HQ_API hq_status hq_get_error(hq_stream_t stream);
/* The cudaError_t of the most recent HQ_ERR_CUDA on this thread (0 if none). */
HQ_API int hq_last_cuda_error(void);
HQ_API const char* hq_status_string(hq_status status);
/* 10000 * major + 100 * minor + patch. */
HQ_API int hq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H_ */
