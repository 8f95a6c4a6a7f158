/* A plain C99 consumer of the library's C ABI: compiles against include/hq.h alone (no CUDA
 * headers), links libhq.so and exercises the calls that need no GPU: the version, status
 * strings, workspace queries and argument errors returned before any launch. */
#include <stdio.h>
#include <stdint.h>
#include <string.h>

#include "hq.h"

static int fails = 0;
#define CHECK(cond) do { if (!(cond)) { printf("FAIL %s:%d %s\n", __FILE__, __LINE__, #cond); ++fails; } } while (0)

int main(void) {
  CHECK(hq_version() > 0);
  CHECK(strcmp(hq_status_string(HQ_OK), "ok") == 0);
  CHECK(strlen(hq_status_string(HQ_ERR_ALIGN)) > 0);
  CHECK(hq_quantize_workspace_bytes() > 0);
  CHECK(hq_linear_fwd_bwd_workspace_bytes(4096, 4096, 11008) > (size_t)4096 * 11008);
  CHECK(hq_gemm_workspace_bytes(4096, 11008, 4096) == 0);
  /* one size covers every layer-level call of a shape, in every code format */
  CHECK(hq_workspace_bytes(4096, 4096, 11008, HQ_INT8) >= hq_linear_fwd_bwd_workspace_bytes(4096, 4096, 11008));
  CHECK(hq_workspace_bytes(4096, 4096, 11008, HQ_INT8) >= hq_linear_workspace_bytes(4096, 4096, 11008));
  CHECK(hq_workspace_bytes(4096, 4096, 11008, HQ_FP4_E2M1) == hq_workspace_bytes(4096, 4096, 11008, HQ_INT8));
  CHECK(hq_workspace_bytes(4096, 4096, 11008, (hq_fmt)9) == 0);
  /* the tensor-core probe rejects formats other than INT8 / FP8 before any launch */
  CHECK(hq_mma_peak(HQ_FP6_E2M3, 16, NULL, NULL) == HQ_ERR_ARG);
  CHECK(hq_mma_peak(HQ_INT8, 0, NULL, NULL) == HQ_ERR_ARG);
  float scale = 0.0f;
  /* null source: rejected before anything is launched */
  CHECK(hq_quantize(NULL, HQ_BF16, 256, 256, 1, 64, HQ_INT8, (void*)0x10000, &scale, (void*)0x10000,
                    hq_quantize_workspace_bytes(), NULL) == HQ_ERR_ARG);
  /* k outside {16, ..., 256} */
  CHECK(hq_quantize((void*)0x10000, HQ_BF16, 256, 256, 1, 48, HQ_INT8, (void*)0x10000, (float*)0x10000,
                    (void*)0x10000, hq_quantize_workspace_bytes(), NULL) == HQ_ERR_ARG);
  /* the reuse GEMM takes 8-bit formats only */
  CHECK(hq_linear_bwd_dx_reuse((void*)0x10000, (float*)0x10000, (void*)0x10000, (float*)0x10000, 256, 256, 256,
                               64, HQ_FP4_E2M1, (void*)0x10000, (void*)0x10000, 1u << 20, NULL) == HQ_ERR_ARG);
  printf("%s\n", fails ? "c consumer: FAILED" : "c consumer: ok");
  return fails ? 1 : 0;
}
