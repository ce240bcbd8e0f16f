/* A plain C99 consumer of the library's C ABI: it includes the public headers, links
 * libpisa_b200.so and calls the host-only entry points (no GPU needed).  Exit status 0 when every
 * check holds; otherwise the number of the first failed check. */
#define _POSIX_C_SOURCE 200112L
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "pisa.h"
#include "pisa_testing.h"

#define CHECK(n, cond)                                   \
  do {                                                   \
    if (!(cond)) {                                       \
      fprintf(stderr, "check %d failed: %s\n", n, #cond); \
      return n;                                          \
    }                                                    \
  } while (0)

static int aligned_in(const void* p, const char* base, size_t bytes) {
  const char* c = (const char*)p;
  return c >= base && c < base + bytes && ((uintptr_t)c % 256u) == 0;
}

int main(void) {
  pisa_shape sh;
  pisa_stats st;
  void* buf = NULL;
  size_t bytes;
  int32_t perm[25];
  int32_t i, seen[25] = {0};

  CHECK(1, pisa_abi_version() == 7);
  CHECK(2, pisa_num_blocks(75600, 128) == 591);
  CHECK(3, pisa_num_blocks(0, 64) == -1);

  sh.batch = 1; sh.heads = 2; sh.seq_len = 1000; sh.head_dim = 128; sh.block = 64;
  sh.dtype = PISA_BF16; sh.softmax_scale = 1.0f;
  bytes = pisa_stats_bytes(&sh, 0);
  CHECK(4, bytes > 0);
  CHECK(5, posix_memalign(&buf, 256, bytes) == 0);
  CHECK(6, pisa_stats_carve(&sh, buf, bytes - 1, 0, &st) == PISA_ERR_INVALID_ARG);
  CHECK(7, pisa_stats_carve(&sh, buf, bytes, 0, &st) == PISA_OK);
  CHECK(8, aligned_in(st.qbar, (const char*)buf, bytes) && aligned_in(st.kbar, (const char*)buf, bytes) &&
               aligned_in(st.vsum, (const char*)buf, bytes) && aligned_in(st.hbar, (const char*)buf, bytes) &&
               aligned_in(st.M, (const char*)buf, bytes) && aligned_in(st.v_op, (const char*)buf, bytes));
  CHECK(9, st.H == NULL && st.q8 == NULL && st.qscale == NULL);
  free(buf);
  CHECK(10, pisa_workspace_bytes(&sh) >= 256);

  /* axis order "hwt" of a 2 x 3 x 4 grid plus one extra token: position (h, w, t) holds stored
   * token t*12 + h*4 + w; the extra token stays last */
  CHECK(11, pisa_axis_permutation(2, 3, 4, 1, "hwt", perm, 24) == PISA_ERR_INVALID_ARG);
  CHECK(12, pisa_axis_permutation(2, 3, 4, 1, "hwx", perm, 25) == PISA_ERR_INVALID_ARG);
  CHECK(13, pisa_axis_permutation(2, 3, 4, 1, "hwt", perm, 25) == PISA_OK);
  CHECK(14, perm[0] == 0 && perm[1] == 12 && perm[2] == 1 && perm[23] == 23 && perm[24] == 24);
  for (i = 0; i < 25; ++i) {
    CHECK(15, perm[i] >= 0 && perm[i] < 25 && !seen[perm[i]]);
    seen[perm[i]] = 1;
  }
  CHECK(16, pisa_status_string(PISA_OK) != NULL && pisa_status_string(PISA_ERR_DEVICE_TIMEOUT) != NULL);
  printf("c consumer ok: abi %d, stats %zu bytes\n", (int)pisa_abi_version(), bytes);
  return 0;
}
