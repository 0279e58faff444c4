/* A plain C caller of libbranch_attn: compiles against branch_attn.h, links
 * the shared library, and makes only calls that need no GPU (sizes, version,
 * argument validation).  Prints "ok" and exits 0 when every expectation
 * holds; otherwise names the first failed one and exits 1. */
#include <stdio.h>
#include <string.h>

#include "branch_attn.h"

static int failed(const char *what) {
  printf("FAILED: %s (last error: %s)\n", what, ba_last_error());
  return 1;
}

int main(void) {
  /* the tiny TTT batch: sequences of 96 and 160 tokens, a depth-3 branch at
   * every position, 4 q / 2 kv heads, d = 64; the index pointers are never
   * dereferenced by these calls */
  static int32_t cu[3], anchor[256], depth[256];
  ba_problem p;
  memset(&p, 0, sizeof(p));
  p.n_seqs = 2;
  p.n_main = 256;
  p.n_branches = 256;
  p.n_branch_tokens = 768;
  p.hq = 4;
  p.hkv = 2;
  p.head_dim = 64;
  p.scale = 0.125f;
  p.mask = BA_MASK_TTT_CAUSAL;
  p.zigzag_C = 1;
  p.cu_seqlens = cu;
  p.branch_anchor = anchor;
  p.branch_depth = depth;

  if (strstr(ba_version(), "sm_100a") == NULL) return failed("version names sm_100a");

  size_t plan_b = 0, fwd_b = 1, bwd_b = 0;
  if (ba_workspace_size(&p, &plan_b, &fwd_b, &bwd_b) != BA_OK) return failed("workspace size");
  if (plan_b == 0 || fwd_b != 0 || bwd_b == 0) return failed("workspace sizes for C = 1");

  ba_plan_layout L;
  if (ba_plan_layout_query(&p, &L) != BA_OK) return failed("layout query");
  if (L.total_bytes != plan_b || L.n_qtiles_main != 2 || L.n_qtiles_branch != 6)
    return failed("layout of the tiny batch");

  size_t staging = 0;
  if (ba_step_host_workspace_size(&p, &staging) != BA_OK || staging < plan_b + bwd_b)
    return failed("host-step staging size");

  ba_problem bad = p;
  bad.head_dim = 96;
  if (ba_workspace_size(&bad, &plan_b, &fwd_b, &bwd_b) != BA_ERR_UNSUPPORTED)
    return failed("head_dim 96 is unsupported");
  bad = p;
  bad.hq = 6;
  bad.hkv = 4;
  if (ba_workspace_size(&bad, &plan_b, &fwd_b, &bwd_b) != BA_ERR_INVALID_ARG)
    return failed("hq not a multiple of hkv");
  if (strlen(ba_last_error()) == 0) return failed("an error message is set");

  /* rejected before any launch: NULL workspace, too small a workspace */
  if (ba_plan(&p, NULL, plan_b, NULL) != BA_ERR_INVALID_ARG) return failed("NULL plan workspace");
  if (ba_plan(&p, (void *)0x100000, plan_b - 1, NULL) != BA_ERR_WORKSPACE_TOO_SMALL)
    return failed("small plan workspace");
  if (ba_wait_check(NULL, 0, NULL) != BA_ERR_INVALID_ARG) return failed("wait check without a plan");
  if (lse_merge(0, 4, 64, 1, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != BA_OK)
    return failed("empty merge is a no-op");
  if (ba_set_kernel_family(2) != BA_ERR_INVALID_ARG) return failed("unknown kernel family");

  printf("ok\n");
  return 0;
}
