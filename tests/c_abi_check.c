/* A plain C99 consumer of the librssm C ABI: the header compiles as C and the
 * library links and answers the calls that need no GPU (sizes, validation,
 * argument errors). */
#include <stdio.h>
#include <string.h>

#include "rssm.h"

int main(void) {
  rssm_layer_desc d;
  memset(&d, 0, sizeof d);
  d.kind = RSSM_MAMBA2;
  d.batch = 4;
  d.nheads = 8;
  d.ngroups = 2;
  d.headdim = 64;
  d.dstate = 128;
  d.window = 16;
  d.max_draft = 4;
  d.in_dtype = RSSM_BF16;
  d.read_fmt = RSSM_READ_FP32;
  d.auto_flush = 1;
  d.out_scale = 1.0f;
  size_t ck = 0, buf = 0, rc = 0, meta = 0;
  rssm_layout lay;
  if (rssm_workspace_size(&d, &ck, &buf, &rc, &meta, &lay) != RSSM_OK) return 1;
  if (ck != (size_t)4 * 8 * 64 * 128 * 4 || rc != 0 || lay.cap != 20) return 2;
  d.branching = 1;
  size_t ck2 = 0;
  if (rssm_workspace_size(&d, &ck2, &buf, &rc, &meta, &lay) != RSSM_OK || ck2 != 2 * ck) return 3;
  d.window = 0;
  if (rssm_workspace_size(&d, &ck, &buf, &rc, &meta, &lay) != RSSM_ERR_INVALID_ARG) return 4;
  if (rssm_last_error_string()[0] == '\0') return 5;
  d.window = 16;
  d.kind = RSSM_KDA;
  d.headdim = d.dstate = 128;
  d.read_fmt = RSSM_READ_NVFP4;
  if (rssm_workspace_size(&d, &ck, &buf, &rc, &meta, &lay) != RSSM_OK || rc == 0) return 6;
  d.headdim = 64;
  if (rssm_workspace_size(&d, &ck, &buf, &rc, &meta, &lay) != RSSM_ERR_UNSUPPORTED) return 11;
  d.headdim = 128;
  if (rssm_branch(NULL, NULL, NULL) != RSSM_ERR_INVALID_ARG) return 7;
  if (rssm_decode_step(NULL, NULL, NULL, NULL) != RSSM_ERR_INVALID_ARG) return 8;
  size_t n = 0;
  if (rssm_state_bytes(NULL, &n) != RSSM_ERR_INVALID_ARG) return 9;
  if (rssm_get_lengths(NULL, NULL, NULL, NULL) != RSSM_ERR_INVALID_ARG) return 10;
  printf("c abi ok\n");
  return 0;
}
