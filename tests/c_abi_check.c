/* A plain C99 consumer of the library: include/mate.h compiles as C, libmate.so links without any C++ or
 * Python, and host-side validation answers as the header states.  Makes no CUDA call (no device needed). */
#include <stdio.h>
#include <string.h>

#include "mate.h"

static int fail(int code, const char* what) {
  fprintf(stderr, "c_abi_check: %s\n", what);
  return code;
}

int main(void) {
  mate_config c;
  memset(&c, 0, sizeof c);
  c.B = 1; c.T = 16; c.H = 32; c.W = 32; c.d = 1024;
  c.nh = 16; c.P = 64; c.N = 128; c.Q = 256; c.R = 256;
  c.th = 8; c.tp = 128; c.wt = 4; c.wh = 8; c.ww = 8; c.st = 2; c.sh = 4; c.sw = 4;
  c.dtype = MATE_BF16;
  c.mamba_extras = 0;
  if (mate_check_config(&c) != MATE_OK) return fail(1, "valid bf16 config rejected");
  size_t ws = mate_workspace_bytes(&c);
  if (ws == 0) return fail(2, "no workspace size for a valid config");
  c.mamba_extras = 1;
  if (mate_workspace_bytes(&c) <= ws) return fail(3, "the Mamba2 extras need more workspace");
  c.mamba_extras = 2;
  if (mate_check_config(&c) != MATE_ERR_ARG) return fail(4, "mamba_extras outside 0..1 accepted");
  c.mamba_extras = 0;
  c.T = 15;
  if (mate_check_config(&c) != MATE_ERR_SHAPE) return fail(5, "window not dividing the grid accepted");
  c.T = 16;
  mate_weights w;
  memset(&w, 0, sizeof w);
  if (mate_forward(NULL, &w, 0, NULL, &c, NULL, 0, NULL) != MATE_ERR_ARG) return fail(6, "null forward accepted");
  if (ssd_scan_bidir_pd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, &c, NULL, 0, NULL) !=
      MATE_ERR_ARG)
    return fail(7, "null per-direction scan accepted");
  if (mate_ssd_pd_workspace_bytes(&c, 256) <= mate_ssd_workspace_bytes(&c, 256))
    return fail(8, "per-direction scan workspace not larger");
  if (strcmp(mate_status_str(MATE_ERR_WORKSPACE), "workspace too small") != 0) return fail(9, "status string");
  if (mate_selftest_wait_timeout(0, NULL) != MATE_ERR_ARG) return fail(11, "zero poll limit accepted");
  for (int k = 0; k <= MATE_K_SELFTEST; ++k)
    if (mate_kernel_name(k) == NULL || strcmp(mate_kernel_name(k), "unknown") == 0) return fail(10, "kernel name");
  printf("ok %zu\n", ws);
  return 0;
}
