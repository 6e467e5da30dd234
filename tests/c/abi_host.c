/* A plain C99 client of include/moe.h, compiled with gcc against the header
 * and linked with libmoe. Without arguments it runs the host-only calls
 * (record layout, workspace sizes, argument checks, routing views over a
 * workspace, status strings); with the argument "gpu" it also creates a
 * context on device 0, reads its status word and destroys it. Prints "ok"
 * and exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe.h"

#define CHECK(c)                                                        \
  do {                                                                  \
    if (!(c)) {                                                         \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                         \
    }                                                                   \
  } while (0)

static unsigned char ws_raw[(1 << 20) + 256];

int main(int argc, char** argv) {
  const int use_gpu = argc > 1 && strcmp(argv[1], "gpu") == 0;
  moe_layer_cfg cfg = {2048, 768, 512, 10, 1, 2, 32, 1, 1, 0, 0, 0};
  moe_expert_layout lay;
  moe_routing r;
  moe_ctx* ctx = NULL;
  size_t ws, sws;
  int s;
  /* a workspace starts on a 256-byte boundary */
  unsigned char* ws_host = ws_raw + (256 - (uintptr_t)ws_raw % 256) % 256;

  /* record layout: sections on 256-byte boundaries, 2.5 bits per weight */
  CHECK(moe_expert_layout_get(&cfg, &lay) == MOE_OK);
  CHECK(lay.gu_codes % 256 == 0 && lay.dn_codes % 256 == 0);
  CHECK(lay.gu_scales % 256 == 0 && lay.dn_scales % 256 == 0);
  CHECK(lay.bytes == 1474560u);
  cfg.bits = 3;
  CHECK(moe_expert_layout_get(&cfg, &lay) == MOE_OK);
  CHECK(lay.bytes == 2064384u);
  cfg.bits = 4;
  CHECK(moe_expert_layout_get(&cfg, &lay) != MOE_OK);
  CHECK(moe_workspace_bytes(&cfg, 1) == 0);
  cfg.bits = 2;

  /* workspace sizes grow with T and with the number of stacked layers */
  ws = moe_workspace_bytes(&cfg, 1);
  CHECK(ws > 0 && ws % 256 == 0);
  CHECK(moe_workspace_bytes(&cfg, 8192) > ws);
  sws = moe_stack_workspace_bytes(&cfg, 48, 1);
  CHECK(sws > moe_stack_workspace_bytes(&cfg, 1, 1));

  /* routing views are plain pointer arithmetic inside the workspace */
  CHECK(ws <= sizeof ws_raw - 256);
  CHECK(moe_layer_routing(&cfg, 1, ws_host, ws, &r) == MOE_OK);
  CHECK(r.T == 1 && r.k == 10 && r.E == 512);
  CHECK((unsigned char*)r.logits >= ws_host && (unsigned char*)r.logits < ws_host + ws);
  CHECK((unsigned char*)r.grouping.n_uniq >= ws_host && (unsigned char*)r.grouping.n_uniq < ws_host + ws);
  CHECK(moe_layer_routing(&cfg, 1, ws_host, 16, &r) == MOE_ENOSPACE);

  /* argument checks on the host */
  CHECK(moe_check_device_status(NULL, NULL) == MOE_EINVAL);
  CHECK(moe_layer_forward(NULL, &cfg, NULL, 1, NULL, NULL, NULL, 1, NULL, lay.bytes, NULL, NULL, 0, NULL,
                          NULL) == MOE_EINVAL);
  for (s = 0; s <= MOE_ENOSPACE; ++s) CHECK(moe_status_string(s) != NULL && moe_status_string(s)[0] != '\0');

  if (use_gpu) {
    CHECK(moe_ctx_create(0, &ctx) == MOE_OK);
    CHECK(moe_check_device_status(ctx, NULL) == MOE_OK);
    CHECK(moe_last_device_error_detail(ctx) == 0);
    moe_ctx_destroy(ctx);
  }
  printf("ok\n");
  return 0;
}
