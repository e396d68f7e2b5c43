/* Plain C99 user of include/deltakv.h: plans the 128k batch-8 decode layer
 * (host-only, no GPU needed) and prints the status, the cache and workspace
 * sizes and the reference-plane capacity.  Built and run by test_abi_c.py. */
#include <stdio.h>

#include "deltakv.h"

int main(void) {
  deltakv_config c = {0};
  c.layers = 1;
  c.batch = 8;
  c.kv_heads = 8;
  c.q_heads = 32;
  c.d_h = 128;
  c.max_T = 131072;
  c.stride_s = 16;
  c.k = 4;
  c.d_c = 32;
  c.hidden = 256;
  c.dtype = DELTAKV_BF16;
  c.act = DELTAKV_ACT_GELU_ERF;
  deltakv_plan_t p = NULL;
  size_t cache_bytes = 0, ws_bytes = 0;
  deltakv_cache_layout L = {0};
  deltakv_status s = deltakv_plan(&c, &p, &cache_bytes, &ws_bytes);
  if (s == DELTAKV_OK) s = deltakv_get_cache_layout(p, &L);
  printf("%d %zu %zu %lld %lld\n", (int)s, cache_bytes, ws_bytes, (long long)L.n_ref_cap, (long long)L.n_code_cap);
  /* a query-head count that is not a multiple of the kv-heads is refused */
  c.q_heads = 30;
  deltakv_plan_t bad = NULL;
  printf("%d %s\n", (int)deltakv_plan(&c, &bad, NULL, NULL), bad == NULL ? "null" : "set");
  deltakv_plan_destroy(p);
  return 0;
}
