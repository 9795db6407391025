/* A plain C99 user of the library's C ABI (host-only calls and host-side
 * argument validation): no CUDA or PyTorch headers, linked against libsata.so.
 * Exit status 0 and "ok" on success, else the number of the failed check. */
#include <stdio.h>

#include "sata.h"

int main(void) {
  /* basis sizes m = C(dK+P-1, P-1) */
  if (sata_basis_size(64, 4) != 47905) return 1;
  if (sata_basis_size(8, 4) != 165) return 2;
  if (sata_basis_size(64, 5) != 814385) return 3;
  if (sata_basis_size(0, 4) != -1) return 4;
  /* M_2 for dK = 3 in lexicographic order */
  int32_t t[12];
  const int32_t want[12] = {0, 0, 0, 1, 0, 2, 1, 1, 1, 2, 2, 2};
  if (sata_index_table(3, 2, t, 12) != 6) return 5;
  for (int i = 0; i < 12; ++i)
    if (t[i] != want[i]) return 6;
  if (sata_index_table(3, 2, t, 11) != -1) return 7; /* capacity too small */
  /* invalid calls return a status before anything is launched */
  if (sata_prefill(NULL, NULL, NULL, NULL, NULL, 1, 1, 8, 8, 8, 4, SATA_F32, NULL) !=
      SATA_ERR_INVALID_ARG)
    return 8;
  if (sata_decode_step(NULL, NULL, NULL, NULL, NULL, 1, 1, 8, 8, 4, SATA_BF16, NULL) !=
      SATA_ERR_INVALID_ARG)
    return 9;
  if (sata_status_string(SATA_ERR_UNSUPPORTED) == NULL) return 10;
  /* the test hook keeps and returns its setting (host only) */
  if (sata_test_set_wait_limit(1000) != 0) return 11;
  if (sata_test_set_wait_limit(0) != 1000) return 12;
  printf("ok\n");
  return 0;
}
