/* A plain C11 consumer of include/csa2.h: calls every host-checked error path
 * of the ABI that needs no GPU and prints one "name status" line per call.
 * Built and run by tests/test_c_consumer.py. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "csa2.h"

#define SHOW(name, expr) printf("%s %d\n", name, (int)(expr))

int main(void) {
  csa2_kv_view kv;
  memset(&kv, 0, sizeof kv);
  csa2_group_desc g;
  memset(&g, 0, sizeof g);
  csa2_cp_shard bad = {0, 2, 100}, ok = {0, 2, 128};
  void *p16 = (void *)(uintptr_t)256, *p8 = (void *)(uintptr_t)264;

  SHOW("quantize_ch", csa2_quantize_fp4(NULL, 4, 24, NULL, NULL, NULL));
  SHOW("quantize_null", csa2_quantize_fp4(NULL, 4, 512, NULL, NULL, NULL));
  SHOW("quantize_empty", csa2_quantize_fp4(NULL, 0, 512, NULL, NULL, NULL));
  SHOW("quantize_align", csa2_quantize_fp4((const uint16_t *)p8, 4, 512, (uint8_t *)p16,
                                           (uint8_t *)p16, NULL));
  SHOW("dequantize_null", csa2_dequantize_fp4(NULL, NULL, 4, 512, NULL, NULL));
  SHOW("index_full_kv", csa2_index_full(NULL, NULL, NULL, 512, 2048, NULL, NULL, NULL, NULL,
                                        NULL, 0, NULL));
  SHOW("index_full_codes", csa2_index_full(&kv, NULL, NULL, 512, 2048, NULL, NULL, NULL, NULL,
                                           NULL, 0, NULL));
  SHOW("reindex_kv", csa2_index_reindex(NULL, NULL, NULL, NULL, NULL, 2048, 512, NULL, NULL,
                                        NULL, 0, NULL));
  SHOW("attn_kv", csa2_sparse_attn_decode(NULL, NULL, NULL, NULL, 512, NULL, NULL, 0.04f, NULL,
                                          NULL, 0, NULL));
  SHOW("group_null", csa2_layer_group(NULL, NULL, 0, NULL));
  SHOW("group_empty", csa2_layer_group(&g, NULL, 0, NULL));
  SHOW("group_ws_size", (int)csa2_group_workspace_size(&g));
  SHOW("append_kv", csa2_cache_append(NULL, NULL, NULL, 0, NULL, NULL, NULL, NULL, NULL, 0,
                                      NULL));
  SHOW("cp_ws_bad", (int)csa2_cp_workspace_size(&bad, 1, 1, 512));
  SHOW("cp_rows_bad", csa2_cp_local_rows(&bad, NULL, 1, NULL, NULL, 0, NULL));
  SHOW("cp_filter_unit", csa2_cp_filter(&ok, 3, (const int32_t *)p16, (const int32_t *)p16, 1,
                                        1, (int32_t *)p16, (int32_t *)p16, 1, NULL, NULL, p16,
                                        256, NULL));
  SHOW("cp_partial_floats", (int)csa2_cp_partial_floats(1, 2));
  printf("status_string %s\n", csa2_status_string(CSA2_ERR_TIMEOUT));
  printf("constants %d %d %d %d %d %d %d %d %d\n", CSA2_D, CSA2_H, CSA2_HI, CSA2_DI, CSA2_BLK,
         CSA2_W, CSA2_MAX_TOPK, CSA2_MAX_POOL, CSA2_CP_MAX_WORLD);
  return 0;
}
