/*
 * Host-only checks of libzcmoe.so from plain C (built and run by tests/test_abi_c.py):
 * the header compiles as C99, the library links from C, and the entry points
 * refuse bad arguments with the documented codes before touching a device.
 * Exit status 0 when every check holds; otherwise the failing check's line.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "zcmoe.h"

static int failures = 0;

#define CHECK(cond)                                        \
  do {                                                     \
    if (!(cond)) {                                         \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                          \
    }                                                      \
  } while (0)

static zcmoe_config good_config(void) {
  zcmoe_config c;
  memset(&c, 0, sizeof c);
  c.d = 256;
  c.n_ffn = 16;
  c.n_zero = 8;
  c.inter = 128;
  c.top_k = 4;
  c.max_tokens = 64;
  c.dtype = ZCMOE_BF16;
  c.routed_scale = 1.0f;
  return c;
}

int main(void) {
  zcmoe_config c = good_config();
  zcmoe_weights w;
  zcmoe_t h = (zcmoe_t)0;
  zcmoe_t fake = (zcmoe_t)(uintptr_t)0x1000;
  zcmoe_gains g = {0.0f, 0.02f, 0.0f, 1.0f, 2.0f};
  float bias[24] = {0};
  int64_t counts[24] = {0}, tokens = 0;
  float eta = 1.0f;
  w.w_router = w.w_gate = w.w_up = w.w_down = (const void *)(uintptr_t)0x100;

  /* create: NULL arguments and bad shapes are refused, *out stays NULL */
  CHECK(zcmoe_create(NULL, &w, &h) == ZCMOE_EINVAL);
  CHECK(zcmoe_create(&c, NULL, &h) == ZCMOE_EINVAL);
  CHECK(zcmoe_create(&c, &w, NULL) == ZCMOE_EINVAL);
  c.d = 100;
  CHECK(zcmoe_create(&c, &w, &h) == ZCMOE_EINVAL && h == NULL);
  c = good_config();
  c.top_k = 33;
  CHECK(zcmoe_create(&c, &w, &h) == ZCMOE_EINVAL && h == NULL);
  c = good_config();
  c.n_zero = 1020;
  CHECK(zcmoe_create(&c, &w, &h) == ZCMOE_EINVAL && h == NULL);
  c = good_config();
  c.dtype = ZCMOE_FP8; /* needs d a multiple of 512 */
  CHECK(zcmoe_create(&c, &w, &h) == ZCMOE_EINVAL && h == NULL);
  c = good_config();
  w.w_gate = (const void *)(uintptr_t)0x108; /* not 16-byte aligned */
  CHECK(zcmoe_create(&c, &w, &h) == ZCMOE_EINVAL && h == NULL);
  w.w_gate = (const void *)(uintptr_t)0x100;
  CHECK(zcmoe_create_ep(&c, &w, 2, 2, 0, &h) == ZCMOE_EINVAL && h == NULL);
  CHECK(strlen(zcmoe_last_error()) > 0);

  /* a handle that was never created is refused by every entry point */
  CHECK(zcmoe_forward(fake, NULL, 1, NULL, 0, NULL) == ZCMOE_EINVAL);
  CHECK(zcmoe_update_bias(fake, &g, 0) == ZCMOE_EINVAL);
  CHECK(zcmoe_read_counts(fake, NULL, 0) == ZCMOE_EINVAL);
  CHECK(zcmoe_write_counts(fake, NULL, 0) == ZCMOE_EINVAL);
  CHECK(zcmoe_get_state(fake, bias, counts, &tokens, &eta) == ZCMOE_EINVAL);
  CHECK(zcmoe_set_bias(fake, bias) == ZCMOE_EINVAL);
  CHECK(zcmoe_get_controller(fake, bias, bias, bias, &eta, counts, &tokens) == ZCMOE_EINVAL);
  CHECK(zcmoe_set_controller(fake, bias, bias, bias, &eta, counts, &tokens) == ZCMOE_EINVAL);
  CHECK(zcmoe_check(fake) == ZCMOE_EINVAL);
  CHECK(zcmoe_backward(fake, NULL, NULL, 1, NULL, NULL, NULL, NULL, NULL, 0) == ZCMOE_EINVAL);
  CHECK(zcmoe_forward_host(fake, NULL, 1, NULL, 0) == ZCMOE_EINVAL);
  CHECK(zcmoe_destroy(fake) == ZCMOE_EINVAL);
  CHECK(zcmoe_destroy(NULL) == ZCMOE_OK);

  if (failures) return 1;
  printf("abi_check: all host-side checks hold\n");
  return 0;
}
