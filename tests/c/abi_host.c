/* A plain C99 program against include/tp_block.h and libtp_block.so: the host-only
 * entry points (status strings, workspace sizing, argument checks that reject
 * before any CUDA call). Prints one "name value" line per result. */
#include <stdio.h>
#include <string.h>

#include "tp_block.h"

int main(void) {
  tp_dims d;
  memset(&d, 0, sizeof d);
  d.dim = 4096;
  d.n_heads = 32;
  d.n_kv_heads = 32;
  d.head_dim = 128;
  d.ffn_dim = 11008;
  d.vocab = 32000;
  d.max_batch = 1;
  d.max_seq = 1024;
  d.norm_eps = 1e-5f;
  d.rope_theta = 1e4f;
  size_t ws = 0, rank_ws = 0;
  printf("version %s\n", tp_version());
  printf("status_ok %s\n", tp_status_string(TP_OK));
  printf("block_ws_rc %d\n", tp_block_workspace_bytes(&d, 4, TP_PART_1D, 1, &ws));
  printf("block_ws %zu\n", ws);
  printf("rank_ws_rc %d\n", tp_block_rank_workspace_bytes(&d, 4, 1, 1, 2, &rank_ws));
  printf("rank_ws %zu\n", rank_ws);
  printf("bad_slices_rc %d\n", tp_block_workspace_bytes(&d, 3, TP_PART_1D, 1, &ws));
  tp_block* h = NULL;
  printf("create_no_ws_rc %d\n", tp_block_create(&d, 4, TP_PART_1D, 1, NULL, NULL, 0, &h));
  printf("quantize_bad_n_rc %d\n", tp_quantize_q8(NULL, NULL, NULL, 33, NULL));
  return 0;
}
