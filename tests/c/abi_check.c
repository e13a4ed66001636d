/* Plain-C client of librelkl.so: include/relkl.h compiles as C11 and every
 * check here runs without a GPU (validation happens before any CUDA call).
 * Prints "ok <n>" after n passed checks, or "FAIL <what>" and exits 1.      */
#include <stdio.h>
#include <string.h>

#include "relkl.h"

static int n_ok = 0;
#define CHECK(cond, what)                       \
  do {                                          \
    if (!(cond)) {                              \
      printf("FAIL %s\n", what);                \
      return 1;                                 \
    }                                           \
    ++n_ok;                                     \
  } while (0)

static relkl_desc desc(int B, int H, int N, int d, int dtype) {
  relkl_desc x;
  memset(&x, 0, sizeof x);
  x.B = B; x.H = H; x.N = N; x.d = d;
  x.stride[0] = (int64_t)H * N * d; x.stride[1] = (int64_t)N * d; x.stride[2] = d; x.stride[3] = 1;
  x.dtype = dtype; x.causal = 1; x.scale = 0.0f; x.reserved = 0;
  return x;
}

int main(void) {
  CHECK(relkl_workspace_bytes() == 256, "workspace size");
  CHECK(strcmp(relkl_status_string(RELKL_OK), "RELKL_OK") == 0, "status string OK");
  CHECK(strncmp(relkl_status_string(RELKL_ERR_TIMEOUT), "RELKL_ERR_TIMEOUT", 17) == 0,
        "status string TIMEOUT");

  relkl_desc tc = desc(1, 2, 256, 128, RELKL_BF16);
  relkl_desc simt = desc(1, 2, 256, 96, RELKL_FP32);
  relkl_desc bad = desc(1, 2, 256, 0, RELKL_BF16);
  CHECK(relkl_path_for(&tc) == 1, "tensor-core path for bf16 d=128");
  CHECK(relkl_path_for(&simt) == 2, "CUDA-core path for fp32 d=96");
  CHECK(relkl_path_for(&bad) == 0, "no path for d=0");

  /* null inputs and a missing workspace are refused before any launch */
  float* f = (float*)(size_t)4096;
  CHECK(relkl_fwd(&tc, NULL, NULL, f, f, NULL, 0, NULL) != RELKL_OK, "fwd with null inputs");
  CHECK(relkl_fwd(&bad, f, f, f, f, NULL, 0, NULL) == RELKL_ERR_INVALID, "fwd with d=0");

  relkl_rope rope = {1e4, 0.125, 0.0, 1, 0};
  CHECK(relkl_rope_bwd(1, 2, 8, 7, f, &rope, RELKL_BF16, f, NULL) == RELKL_ERR_INVALID,
        "rope_bwd with odd d");
  CHECK(relkl_rope_bwd(0, 2, 8, 64, NULL, &rope, RELKL_BF16, NULL, NULL) == RELKL_OK,
        "rope_bwd with no tokens is a no-op");
  CHECK(relkl_weight_grad(0, 64, 64, f, f, f, f, 256, NULL) == RELKL_ERR_INVALID,
        "weight_grad rows=0");

  /* the bf16 copy of dX_s: n = 0 is a no-op, overlapping ranges are refused */
  CHECK(relkl_cast_bf16(NULL, NULL, 0, NULL) == RELKL_OK, "cast of nothing");
  CHECK(relkl_cast_bf16(f, f, 16, NULL) == RELKL_ERR_INVALID, "cast onto its own source");
  CHECK(relkl_cast_bf16(f, f, -1, NULL) == RELKL_ERR_INVALID, "cast with n < 0");

  /* the backward kernel a launch would pick (host only) */
  relkl_desc big = desc(1, 32, 32768, 128, RELKL_BF16);
  relkl_desc d64 = desc(1, 2, 256, 64, RELKL_BF16);
  CHECK(relkl_bwd_kernel_for(1, &big, 148) == 3, "paired backward at 32K");
  CHECK(relkl_bwd_kernel_for(1, &tc, 148) == 2, "one-block backward at 2 row blocks");
  CHECK(relkl_bwd_kernel_for(1, &d64, 148) == 4, "paired d=64 backward");
  CHECK(relkl_bwd_kernel_for(1, &simt, 148) == 1, "CUDA-core backward");
  CHECK(relkl_bwd_kernel_for(1, &tc, 0) == 0, "no SMs");

  uint64_t old = relkl_set_wait_timeout_ns(123456789ull);
  CHECK(relkl_set_wait_timeout_ns(old) == 123456789ull, "timeout round trip");
  printf("ok %d\n", n_ok);
  return 0;
}
