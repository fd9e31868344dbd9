/* A plain C99 caller of the C ABI (no C++, no CUDA headers): queries the workspace size of
 * the tiny configuration, a rejected parameter set and the status strings.  No GPU call. */
#include <stdio.h>

#include "abattn.h"

int main(void) {
  ab_params p = {1, 2, 1024, 64, 128, 4, 8, 1, 0, 0};
  size_t n = 0;
  ab_status r = ab_workspace_bytes(&p, &n);
  ab_params bad = p;
  bad.d = 96;
  size_t m = 0;
  ab_status rb = ab_workspace_bytes(&bad, &m);
  /* a head slice: heads [2, 4) of an 8-head layer needs the workspace of its own 2 heads */
  ab_params slice = p;
  slice.head0 = 2;
  slice.heads_total = 8;
  size_t ns = 0;
  ab_status rs = ab_workspace_bytes(&slice, &ns);
  printf("%d %zu %d %s|%s %d\n", (int)r, n, (int)rb, ab_status_string(AB_OK),
         ab_status_string(AB_ERR_UNSUPPORTED), ab_version());
  return r == AB_OK && rb == AB_ERR_UNSUPPORTED && rs == AB_OK && ns == n ? 0 : 1;
}
