/* A plain C99 consumer of include/samba.h, built and run by the CPU test suite.
 * It uses only the host-side part of the ABI (no device is needed): version and
 * status strings, workspace queries of the 2048-wide block, and argument
 * validation that returns before anything touches the device. */
#include <stdio.h>
#include <string.h>

#include "samba.h"

static int fail(const char* what) {
  fprintf(stderr, "consumer: %s\n", what);
  return 1;
}

int main(void) {
  samba_block_config cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.d_model = 2048;
  cfg.d_inner = 4096;
  cfg.d_state = 16;
  cfg.d_conv = 4;
  cfg.dt_rank = 128;
  cfg.n_q = 32;
  cfg.n_kv = 4;
  cfg.head_dim = 64;
  cfg.window = 2048;
  cfg.d_ff = 8192;
  cfg.rope_base = 10000.0f;
  cfg.norm_eps = 1e-5f;
  cfg.dtype = SAMBA_BF16;

  if (!strstr(samba_version(), "sm_100a")) return fail("version");
  if (strcmp(samba_status_string(SAMBA_ERR_UNSUPPORTED), "SAMBA_ERR_UNSUPPORTED") != 0) return fail("status string");

  const size_t ws1 = samba_block_workspace_size(&cfg, 1, 4096);
  const size_t ws2 = samba_block_workspace_size(&cfg, 1, 8192);
  if (ws1 == 0 || ws2 <= ws1) return fail("block workspace grows with L");
  if (samba_step_workspace_size(&cfg, 32) == 0) return fail("step workspace");

  cfg.d_state = 8; /* not handled by these kernels */
  if (samba_block_workspace_size(&cfg, 1, 4096) != 0) return fail("d_state 8 must give no workspace");
  cfg.d_state = 16;

  /* NULL inputs are rejected before any launch */
  samba_status s = samba_selective_scan(NULL, NULL, NULL, 1, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 64,
                                        32, 16, SAMBA_BF16, NULL, 0, NULL);
  if (s != SAMBA_ERR_INVALID_ARG) return fail("scan with NULL inputs");
  samba_block_weights w;
  memset(&w, 0, sizeof(w));
  s = samba_block_fwd(&cfg, &w, NULL, NULL, NULL, NULL, 1, 64, NULL, 0, NULL);
  if (s != SAMBA_ERR_INVALID_ARG) return fail("block with no weights");

  printf("consumer ok: %s, block workspace %zu bytes at L=4096\n", samba_version(), ws1);
  return 0;
}
