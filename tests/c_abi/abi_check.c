/* Compiled as plain C99 by tests/test_abi.py and linked against libtasq.so: the boundary must be
 * a C ABI (no C++ or torch types). It calls only entry points that fail on the host before any
 * device work, so it runs without a GPU. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "tasq.h"

static int expect(tasq_status got, tasq_status want, const char* what) {
  if (got != want) {
    fprintf(stderr, "%s: status %d, expected %d (%s)\n", what, (int)got, (int)want, tasq_last_error());
    return 1;
  }
  return 0;
}

int main(void) {
  int bad = 0;
  tasq_ctx* ctx = (tasq_ctx*)0x1;
  tasq_layer_desc layer;
  memset(&layer, 0, sizeof(layer));
  layer.N = 64;
  layer.K = 12; /* not a multiple of 8 */
  bad |= expect(tasq_linear_create(&ctx, &layer, 1, 1, 64, 16, TASQ_OUT_F16, NULL), TASQ_ERR_INVALID_ARG,
                "create with K % 8 != 0");
  bad |= (ctx != NULL);
  bad |= expect(tasq_linear_forward(NULL, NULL, 0, 0, 0, 0, NULL, 0, NULL), TASQ_ERR_INVALID_ARG, "forward(NULL)");
  bad |= expect(tasq_set_schedule(NULL, NULL, NULL), TASQ_ERR_INVALID_ARG, "set_schedule(NULL)");
  bad |= expect(tasq_linear_destroy(NULL), TASQ_OK, "destroy(NULL)");
  bad |= expect(tasq_linear_forward_noalloc(NULL, 1, 8, 8, NULL, NULL, 8, 9, 64, NULL, 8, TASQ_OUT_F16, NULL, NULL),
                TASQ_ERR_INVALID_ARG, "noalloc with bits 9");
  bad |= (TASQ_MAX_KP != 16384) || (TASQ_GROUP_MAX != 4) || (TASQ_DMPQ_MAX_LAYERS != 32);
  printf(bad ? "FAIL\n" : "OK\n");
  return bad;
}
