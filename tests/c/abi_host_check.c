/* A plain C99 caller of libvdn's host-side entry points: the header compiles
 * as C, and parameter set-up, workspace sizing, the launch count and argument
 * validation behave as documented, with no GPU involved (every call here
 * returns before any CUDA work).  Prints one line per check; exit status 0
 * when all hold. */
#include <stdio.h>
#include <string.h>

#include "vdn.h"

static int failures = 0;

static void check(int cond, const char *what) {
  printf("%s %s\n", cond ? "ok  " : "FAIL", what);
  if (!cond) ++failures;
}

int main(void) {
  check(vdn_abi_version() == VDN_ABI_VERSION, "abi version");
  check(strcmp(vdn_status_string(VDN_OK), "VDN_OK") == 0, "status string");

  vdn_params p;
  memset(&p, 0, sizeof p);
  check(vdn_params_init(&p, 1, 24, 75, 1536, 128, 512, VDN_BF16) == VDN_OK, "params init");
  check(p.chunk == 5 && p.window_radius == 1 && p.D_out == 24 * 128, "params defaults");

  size_t ws = 0;
  check(vdn_workspace_bytes(&p, &ws) == VDN_OK && ws > 0, "workspace size");
  check(vdn_workspace_bytes(NULL, &ws) == VDN_ERR_INVALID_ARG, "workspace: NULL params");

  int n = 0;
  check(vdn_forward_launches(&p, &n) == VDN_OK && n == 7, "launches: 768p frame scan");
  p.flags = VDN_FLAG_SCAN_CHUNKS;
  check(vdn_forward_launches(&p, &n) == VDN_OK && n == 8, "launches: chunk route");
  p.flags = VDN_FLAG_SCAN_CHUNKS | VDN_FLAG_SCAN_FRAMES;
  check(vdn_forward_launches(&p, &n) == VDN_ERR_INVALID_ARG, "scan flags exclusive");
  p.flags = 0;

  /* validation before any launch: NULL inputs, a misaligned pointer, a short
   * workspace; no device memory is touched */
  static unsigned char buf[256] __attribute__((aligned(256)));
  check(vdn_hybrid_attn_fwd(&p, NULL, buf, buf, (const float *)buf, NULL, buf, buf, buf, buf,
                            buf, buf, buf, sizeof buf, NULL) == VDN_ERR_INVALID_ARG,
        "forward: NULL q");
  check(vdn_hybrid_attn_fwd(&p, buf + 1, buf, buf, (const float *)buf, NULL, buf, buf, buf,
                            buf, buf, buf, buf, sizeof buf, NULL) == VDN_ERR_ALIGNMENT,
        "forward: misaligned q");
  check(vdn_hybrid_attn_fwd(&p, buf, buf, buf, (const float *)buf, NULL, buf, buf, buf, buf,
                            buf, buf, buf, sizeof buf, NULL) == VDN_ERR_WORKSPACE,
        "forward: workspace too small");
  p.T = 0;
  check(vdn_workspace_bytes(&p, &ws) == VDN_ERR_SHAPE, "T = 0 rejected");
  return failures == 0 ? 0 : 1;
}
