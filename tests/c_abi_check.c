/* A plain C99 caller of libgptq: the header compiles as C, the library links, and
 * the calls that need no device answer as include/gptq.h says (status strings,
 * workspace sizes, argument errors returned before anything is launched). */
#include <stdio.h>
#include <string.h>

#include "gptq.h"

static int failures = 0;

static void expect(int ok, const char* what) {
  if (!ok) {
    printf("FAIL %s\n", what);
    ++failures;
  }
}

int main(void) {
  gptq_config cfg = {4, 128, 0, GPTQ_ORDER_NATURAL, 0.01f, 128};
  gptq_config bad = {5, 128, 0, GPTQ_ORDER_NATURAL, 0.01f, 128};
  size_t a = gptq_workspace_size(GPTQ_OP_PREPARE, 0, 768, &cfg);
  size_t q = gptq_workspace_size(GPTQ_OP_QUANTIZE, 3072, 768, &cfg);
  int64_t n = 0;

  expect(strcmp(gptq_status_string(GPTQ_OK), "GPTQ_OK") == 0, "status string OK");
  expect(strcmp(gptq_status_string(GPTQ_ERR_NOT_PD), "GPTQ_ERR_NOT_PD") == 0,
         "status string NOT_PD");
  expect(a > (size_t)2 * 768 * 768 * 4 && a % 256 == 0, "prepare workspace");
  expect(q >= (size_t)3072 * 768 * 5 && q % 256 == 0, "quantize workspace");
  expect(gptq_workspace_size(GPTQ_OP_PREPARE, 0, 768, &bad) == 0, "bad bits -> 0 bytes");
  expect(gptq_workspace_size(GPTQ_OP_QUANTIZE, 10, 0, &cfg) == 0, "cols 0 -> 0 bytes");
  expect(gptq_pack(NULL, 4, 8, 4, NULL, NULL) == GPTQ_ERR_INVALID_ARG, "pack null pointers");
  expect(gptq_pack(NULL, 4, 8, 5, NULL, NULL) == GPTQ_ERR_INVALID_ARG, "pack bits 5");
  expect(gptq_hessian_accumulate(NULL, &n, NULL, GPTQ_F16, 8, 8, 8, NULL, NULL) ==
             GPTQ_ERR_INVALID_ARG, "hessian null H");
  expect(gptq_prepare(NULL, 8, &cfg, NULL, NULL, NULL, 0, NULL, NULL) == GPTQ_ERR_INVALID_ARG,
         "prepare null pointers");
  expect(gptq_selftest_timeout(GPTQ_SELFTEST_MBARRIER, NULL, NULL) == GPTQ_ERR_INVALID_ARG,
         "selftest null status");
  expect(gptq_launch_count() == 0, "nothing launched");
  expect(strcmp(gptq_last_error(), "") == 0, "no CUDA error recorded");
  if (failures == 0) printf("c abi ok\n");
  return failures == 0 ? 0 : 1;
}
