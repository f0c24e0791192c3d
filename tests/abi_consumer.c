/* A plain C consumer of include/lidx.h.  It must compile as strict C11 and as
 * C++, link against liblidx.so, and find the library's compiled struct
 * layouts, ABI version and host-only calls equal to what the header states.
 * Runs without a GPU: nothing here touches a device. */
#include <stdio.h>
#include <string.h>

#include "lidx.h"

int main(void) {
  const size_t sizes[7] = {sizeof(lidx_kv), sizeof(lidx_score_args), sizeof(lidx_topk_args),
                           sizeof(lidx_attn_args), sizeof(lidx_eval_args), sizeof(lidx_decode_args),
                           sizeof(lidx_append_args)};
  int bad = 0;
  int i;
  lidx_topk_args t;
  lidx_score_args s;
  lidx_decode_args d;
  size_t n = 1;

  if (lidx_abi_version() != LIDX_ABI_VERSION) {
    printf("abi version %d, header %d\n", lidx_abi_version(), LIDX_ABI_VERSION);
    bad = 1;
  }
  for (i = 0; i < 7; i++) {
    if (lidx_struct_size(i) != sizes[i]) {
      printf("struct %d: library %zu, header %zu\n", i, lidx_struct_size(i), sizes[i]);
      bad = 1;
    }
  }
  if (strcmp(lidx_status_string(LIDX_OK), "ok") != 0) bad = 1;
  if (lidx_workspace_size(LIDX_OP_TOPK, NULL, &n) != LIDX_ERR_INVALID_ARG) bad = 1;
  memset(&t, 0, sizeof t); /* B = 0: rejected before any device call */
  if (lidx_workspace_size(LIDX_OP_TOPK, &t, &n) != LIDX_ERR_INVALID_ARG) bad = 1;
  memset(&s, 0, sizeof s);
  if (lidx_index_score(&s, NULL) != LIDX_ERR_INVALID_ARG) bad = 1;
  memset(&d, 0, sizeof d);
  if (lidx_workspace_size(LIDX_OP_DECODE, &d, &n) != LIDX_ERR_INVALID_ARG) bad = 1;
  printf(bad ? "FAIL\n" : "OK\n");
  return bad;
}
