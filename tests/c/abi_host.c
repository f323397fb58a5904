/* Host-only use of the C ABI from a C99 program: problem checks, padding, workspace and
 * weight sizes, the expert-parallel sizes, and argument errors returned before any CUDA
 * call. Exits 0 when every check holds, else prints the failing line. Built and run by
 * tests/test_c_header.py. */
#include <stdio.h>
#include <string.h>

#include "moe_b200.h"

static int failures = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      printf("FAILED line %d: %s\n", __LINE__, #cond);           \
      ++failures;                                                \
    }                                                            \
  } while (0)

int main(void) {
  moe_problem_t p;
  memset(&p, 0, sizeof(p));
  p.num_tokens = 4096;
  p.hidden = 2048;
  p.num_routed = 256;
  p.num_shared = 0;
  p.intermediate = 512;
  p.topk = 8;
  p.renormalize = 1;
  p.activation = MOE_ACT_SWIGLU;
  p.wdtype = MOE_DTYPE_BF16;
  p.block_m = 0;
  p.flags = MOE_FLAG_PDL;
  CHECK(moe_check_problem(&p) == MOE_OK);
  CHECK(strcmp(moe_status_string(MOE_ERR_WORKSPACE_TOO_SMALL), "MOE_ERR_WORKSPACE_TOO_SMALL") == 0);

  /* padding: gated to 16, relu2 and every 8-bit format to 128 */
  CHECK(moe_padded_intermediate(200, MOE_ACT_SWIGLU, MOE_DTYPE_BF16) == 208);
  CHECK(moe_padded_intermediate(200, MOE_ACT_RELU2, MOE_DTYPE_BF16) == 256);
  CHECK(moe_padded_intermediate(200, MOE_ACT_SWIGLU, MOE_DTYPE_MXFP8) == 256);
  CHECK(moe_padded_intermediate(0, MOE_ACT_SWIGLU, MOE_DTYPE_BF16) == -1);

  /* workspace: layout and size agree; regions do not run past the end */
  moe_workspace_layout_t lay;
  CHECK(moe_workspace_layout(&p, &lay) == MOE_OK);
  CHECK(lay.total_bytes == moe_workspace_size(&p));
  CHECK(lay.block_m == 16);
  CHECK(lay.y + (size_t)lay.max_rows * 2048 * 4 <= lay.total_bytes);

  /* prepared weights (bf16 tiles of 128 x 64): 256 experts x 8 x 32 tiles of 16 KB for w13 */
  CHECK(moe_prepared_weights_bytes(&p, 0) == (size_t)256 * 8 * 32 * 16384);
  CHECK(moe_prepared_weights_bytes(&p, 2) == 0);

  /* expert parallelism over 8 ranks: 32 experts each */
  CHECK(moe_ep_max_send_rows(&p, 8) == (4096 * 8 + 8 * 15 + 15) / 16 * 16);
  CHECK(moe_ep_workspace_size(&p, 8) > 0);
  CHECK(moe_ep_max_send_rows(&p, 3) == -1);

  /* argument errors come back before any CUDA call */
  CHECK(moe_forward(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG);
  moe_problem_t bad = p;
  bad.hidden = 100;
  CHECK(moe_check_problem(&bad) == MOE_ERR_UNSUPPORTED);
  bad = p;
  bad.topk = 300;
  CHECK(moe_check_problem(&bad) == MOE_ERR_INVALID_ARG);
  bad = p;
  bad.wdtype = MOE_DTYPE_MXFP8;
  bad.block_m = 128;
  CHECK(moe_check_problem(&bad) == MOE_ERR_UNSUPPORTED);

  /* T == 0 is valid and enqueues nothing */
  moe_problem_t empty = p;
  empty.num_tokens = 0;
  CHECK(moe_forward(&empty, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == MOE_OK);

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
