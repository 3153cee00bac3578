/* Plain C99 user of the C ABI: compiles against include/knapspec.h alone,
 * links libknapspec.so, and exercises the host-only calls (no GPU needed):
 * version, weight quantisation, grid size, workspace size and an argument
 * error with its message.  Prints one line per check; exits non-zero on the
 * first failure. */
#include <stdio.h>
#include <string.h>

#include "knapspec.h"

#define CHECK(cond, what)                         \
  do {                                            \
    if (!(cond)) {                                \
      printf("FAIL %s\n", what);                  \
      return 1;                                   \
    }                                             \
    printf("ok %s\n", what);                      \
  } while (0)

int main(void) {
  const char* v = ks_version();
  CHECK(v != NULL && strstr(v, "sm_100a") != NULL, "version");

  /* a tiny 4-layer model: Attn latency 4, MLP latency 3, 28 bins */
  double t[8] = {4, 3, 4, 3, 4, 3, 4, 3};
  int32_t w[8];
  CHECK(ks_quantize_weights(t, 8, 28, w) == KS_OK, "quantize");
  CHECK(w[0] == 4 && w[1] == 3 && w[6] == 4 && w[7] == 3, "quantized weights");

  ks_params p;
  memset(&p, 0, sizeof p);
  p.gamma_max = 8;
  p.n_bins = 28;
  int32_t C = 0;
  CHECK(ks_solve_cells(8, NULL, t, &p, &C) == KS_OK && C == 29, "grid size");

  ks_model_desc m;
  memset(&m, 0, sizeof m);
  m.n_layers = 4;
  m.d_model = 256;
  m.n_q_heads = 4;
  m.n_kv_heads = 4;
  m.head_dim = 64;
  m.ffn = 688;
  m.rms_eps = 1e-6f;
  m.rope_base = 1e4;
  m.wdtype = KS_F32;
  size_t bytes = 0;
  CHECK(ks_workspace_size(&m, C, 4, &bytes) == KS_OK && bytes > 0, "workspace size");

  m.head_dim = 96;
  CHECK(ks_workspace_size(&m, C, 4, &bytes) == KS_ERR_UNSUPPORTED, "unsupported head_dim");
  CHECK(strstr(ks_last_error(), "head_dim") != NULL, "error message");
  CHECK(strcmp(ks_status_string(KS_ERR_TIMEOUT), "device wait timed out") == 0, "status string");
  return 0;
}
