/* A plain C11 consumer of include/linattn.h: it compiles against the header,
 * links liblinattn.so and calls entry points whose answers need no device
 * (argument checks, empty problems, status strings). Prints one line per check;
 * the test compares them. */
#include <stdio.h>
#include <string.h>

#include "linattn.h"

static la_params params(int N, int D) {
  la_params p;
  memset(&p, 0, sizeof(p));
  p.B = 1;
  p.H = 2;
  p.N = N;
  p.D = D;
  p.dtype = LA_BF16;
  p.mode = LA_BIDIRECTIONAL;
  p.rope_theta = 10000.0;
  p.eps = 1e-6f;
  return p;
}

int main(void) {
  size_t bytes = 0;
  la_params bad = params(64, 48);
  la_params empty = params(0, 64);
  printf("workspace_size_bad_D %d\n", (int)lin_attn_workspace_size(&bad, &bytes));
  printf("forward_empty %d\n", (int)lin_attn_forward(&empty, NULL, NULL, NULL, NULL, NULL,
                                                     NULL, 0, NULL));
  printf("cross_no_keys %d\n", (int)lin_attn_cross_workspace_size(&empty, 0, &bytes));
  printf("tconv_empty %d\n", (int)lin_attn_temporal_conv(1, 0, 4, 8, LA_BF16, NULL, NULL, NULL,
                                                         NULL, NULL, NULL, NULL));
  printf("tconv_bad_C %d\n", (int)lin_attn_temporal_conv(1, 2, 4, 12, LA_BF16, NULL, NULL, NULL,
                                                         NULL, NULL, NULL, NULL));
  printf("status_ok %s\n", lin_attn_status_string(LA_OK));
  printf("status_limit %d\n", (int)LA_WORKSPACE_CONTROL_BYTES);
  return 0;
}
