/* A plain C client of the library's C ABI (no Python, no torch): the host-only
 * entry points and the argument checks that return before any device work.
 * Built and run by tests/test_c_abi.py; needs no GPU. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "kvsculpt.h"

#define CHECK(cond)                                         \
  do {                                                      \
    if (!(cond)) {                                          \
      fprintf(stderr, "FAIL line %d: %s\n", __LINE__, #cond); \
      return 1;                                             \
    }                                                       \
  } while (0)

int main(void) {
  CHECK(strstr(kvs_version(), "sm_100a") != NULL);

  /* a host-described batch: 3 problems, d = 128, n_q = 40, z = 30, k = 7, 5, 9 */
  static int64_t q_off[4] = {0, 40, 80, 120}, z_off[4] = {0, 30, 60, 90};
  static int64_t c_off[4] = {0, 7, 12, 21};
  kvs_batch b;
  b.B = 3;
  b.d = 128;
  b.q_off = q_off; /* never dereferenced on the host paths below */
  b.z_off = z_off;
  b.c_off = c_off;
  b.q_off_h = q_off;
  b.z_off_h = z_off;
  b.c_off_h = c_off;
  kvs_schedule s = {40, 5, 10, 20, 1, 1e-3f, 1.f, 1.f, 1e-4f, 0.5f};
  const size_t ws = kvs_workspace_bytes(&b, &s);
  CHECK(ws > 0 && ws % 256 == 0);
  CHECK(kvs_lbfgs_state_bytes(&b, 10) >= (size_t)21 * 128 * 4 * 22);

  /* invalid batches */
  kvs_batch bad = b;
  bad.d = 96;
  CHECK(kvs_workspace_bytes(&bad, &s) == 0);
  bad = b;
  bad.B = 0;
  CHECK(kvs_workspace_bytes(&bad, &s) == 0);
  static int64_t c_bad[4] = {0, 7, 5, 21}; /* decreasing offsets */
  bad = b;
  bad.c_off_h = c_bad;
  CHECK(kvs_workspace_bytes(&bad, &s) == 0);

  /* argument errors come back before any device work */
  void *fake = (void *)(uintptr_t)(1u << 20);
  CHECK(kvs_loss_grad(&b, NULL, fake, fake, fake, fake, 1.f, 1.f, fake, NULL, NULL, fake, ws,
                      NULL) == KVS_EINVAL);
  CHECK(kvs_loss_grad(&b, fake, fake, fake, fake, fake, 1.f, 1.f, fake, NULL, NULL, fake, ws - 256,
                      NULL) == KVS_EWORKSPACE);
  CHECK(kvs_adam_step(&b, fake, fake, fake, fake, 0, 1e-2f, 0.9f, 0.999f, 1e-8f, NULL) ==
        KVS_EINVAL);

  /* the host-only budget allocation: k_b proportional to sqrt(mse), clamped, exact sum */
  float mse[3] = {1.f, 4.f, 0.f};
  int32_t kmax[3] = {100, 100, 100}, k[3] = {0, 0, 0};
  CHECK(kvs_pilot_allocate(3, mse, 60, 5, kmax, 0.5f, k) == KVS_OK);
  CHECK(k[0] + k[1] + k[2] == 60);
  CHECK(k[2] == 5);                 /* zero signal: the floor */
  CHECK(k[1] > k[0] && k[0] >= 5);  /* sqrt(4) = 2 x sqrt(1) before rounding */
  CHECK(kvs_pilot_allocate(3, mse, 10, 5, kmax, 0.5f, k) == KVS_EINVAL); /* below 3 x k_min */
  printf("c abi ok: ws %zu bytes, k = %d %d %d\n", ws, k[0], k[1], k[2]);
  return 0;
}
