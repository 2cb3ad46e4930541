/* A plain C99 client of the library: includes the public header, links libdsv4v.so and calls
 * the entry points that need no GPU (sizing, layout, status strings, host-side validation).
 * Built and run by tests/test_abi_host.py; exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "dsv4v.h"

static int failures = 0;

static void check(int ok, const char* what) {
  if (!ok) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  dsv4v_config cfg = {1024, 16, 2816, 2, 4096, 32, 1e-6f, 10000.0f, DSV4V_BF16};
  int32_t grid[2] = {28, 28};
  int32_t cu[2] = {0, 784};
  dsv4v_batch batch = {1, grid, grid, cu, cu};
  int32_t types[16];
  int64_t len = -1;

  check(dsv4v_aligner_tokens(&cfg, &batch) == 196, "aligner tokens of a 28x28 grid");
  check(dsv4v_workspace_size(&cfg, &batch) > 0, "forward workspace size");
  check(dsv4v_backward_workspace_size(&cfg, &batch) > dsv4v_workspace_size(&cfg, &batch),
        "backward workspace holds the forward layout and more");
  check(dsv4v_bridge_workspace_size(1) == 1024, "bridge workspace of one position");
  check(dsv4v_image_layout(3, 5, 2, NULL, 0, &len) == DSV4V_OK && len == 10, "layout length");
  check(dsv4v_image_layout(3, 5, 2, types, 16, NULL) == DSV4V_OK, "layout written");
  check(types[0] == DSV4V_TOKEN_START && types[4] == DSV4V_TOKEN_NEWLINE && types[9] == DSV4V_TOKEN_END &&
            types[1] == DSV4V_TOKEN_IMAGE,
        "layout contents");
  /* graph replay switch and release: host state only, no GPU needed */
  dsv4v_set_graph_replay(0);
  dsv4v_release_graphs();
  dsv4v_set_graph_replay(1);
  check(strcmp(dsv4v_status_string(DSV4V_OK), "ok") == 0, "status string");
  check(dsv4v_status_string(DSV4V_ERR_LAYOUT) != NULL, "layout status string");

  /* rejected on the host, before any CUDA call */
  cfg.n_heads = 7;
  check(dsv4v_workspace_size(&cfg, &batch) == 0, "vision_dim not divisible by n_heads");
  cfg.n_heads = 16;
  cu[1] = 783;
  check(dsv4v_aligner_tokens(&cfg, &batch) == -1, "offsets that do not match the grid");
  cu[1] = 784;
  cfg.dtype = DSV4V_F32;
  check(dsv4v_backward_workspace_size(&cfg, &batch) == 0, "backward is bf16 only");

  if (failures == 0) printf("c abi ok\n");
  return failures == 0 ? 0 : 1;
}
