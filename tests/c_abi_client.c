/* A plain C client of the library's boundary: it includes only coll.h,
 * links libmvrcoll.so, and calls the entry points that answer on the host
 * (sizes, form queries, error strings, argument checks that fail before any
 * launch).  It touches no device memory and needs no GPU.  Prints "ok" and
 * exits 0 when every answer is the documented one. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "coll.h"

static int failures = 0;

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "%s:%d: failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                \
    }                                                            \
  } while (0)

int main(void) {
  /* fake, never dereferenced device addresses: every call below fails its
   * argument checks (or only computes sizes) before it could launch */
  const uintptr_t base = (uintptr_t)1 << 40;
  const void* send[9];
  void* recv[9];
  for (int r = 0; r < 9; ++r) {
    send[r] = (const void*)(base + (uintptr_t)r * 0x100000);
    recv[r] = (void*)(base + 0x10000000 + (uintptr_t)r * 0x100000);
  }

  CHECK(coll_version() > 0);
  CHECK(strlen(coll_strerror(COLL_OK)) > 0);
  CHECK(strlen(coll_strerror(COLL_ERR_WORKSPACE)) > 0);

  /* packet sizes: LL doubles the bytes in 8-byte lines, LL128 carries 120 of every 128 */
  CHECK(coll_packed_bytes(8, COLL_PROTO_LL) == 16);
  CHECK(coll_packed_bytes(120, COLL_PROTO_LL128) == 128);
  CHECK(coll_packed_bytes(121, COLL_PROTO_LL128) == 256);

  /* workspace sizes and the form each algorithm resolves to */
  CHECK(coll_all_reduce_workspace_size(8, 1000, COLL_BF16, COLL_ALGO_TWOSHOT) == 0);
  CHECK(coll_all_reduce_workspace_size(8, 1000, COLL_BF16, COLL_ALGO_RING) >= 256 + 4000);
  CHECK(coll_all_reduce_form(8, 1000, COLL_BF16, COLL_ALGO_AUTO, 1) == COLL_ALGO_TWOSHOT);
  CHECK(coll_all_reduce_form(8, 1000, COLL_BF16, COLL_ALGO_RING, 1) == COLL_ALGO_RING_LANE);
  CHECK(coll_all_reduce_form(8, 1 << 20, COLL_BF16, COLL_ALGO_RING, 1) == COLL_ALGO_RING_CTA);
  CHECK(coll_all_reduce_form(8, 1000, COLL_BF16, COLL_ALGO_RING_WIRE, 1) == COLL_ALGO_RING_WIRE);
  CHECK(coll_all_reduce_form(8, 1000, COLL_BF16, COLL_ALGO_RING_WIRE, 0) == COLL_ERR_UNSUPPORTED);
  CHECK(coll_ll_pack_ranks(NULL, NULL, 4, 16, COLL_PROTO_LL, 1, NULL) == COLL_ERR_INVALID_ARG);
  CHECK(coll_ll_unpack_ranks(NULL, NULL, 4, 16, COLL_PROTO_LL128, 1, NULL, NULL) == COLL_ERR_INVALID_ARG);
  CHECK(coll_all_reduce_form(8, 1000, COLL_BF16, COLL_ALGO_RING, 0) == COLL_ALGO_RING_STEPS);
  CHECK(coll_all_reduce_form(9, 1000, COLL_BF16, COLL_ALGO_RING, 1) == COLL_ALGO_RING_STEPS);
  CHECK(coll_moe_route_workspace_size(8, 4096, 8, 256) > 0);
  CHECK(coll_moe_route_workspace_size(8, 4096, 8, 250) == 0);

  /* argument checks that fail on the host */
  CHECK(coll_all_reduce(send, recv, 0, 16, COLL_BF16, COLL_SUM, COLL_ALGO_TWOSHOT, NULL, 0, NULL) ==
        COLL_ERR_INVALID_ARG);
  CHECK(coll_all_reduce(send, recv, 4, 16, COLL_BF16, COLL_SUM, COLL_ALGO_RING, NULL, 0, NULL) ==
        COLL_ERR_WORKSPACE);
  CHECK(coll_all_reduce(send, recv, 9, 16, COLL_BF16, COLL_SUM, COLL_ALGO_RING_CTA, NULL, 0, NULL) ==
        COLL_ERR_UNSUPPORTED);
  CHECK(coll_broadcast(recv, 4, 16, COLL_BF16, 4, NULL) == COLL_ERR_INVALID_ARG);
  CHECK(coll_ll_pack(send[0], recv[0], 64, COLL_PROTO_LL, 0, NULL) == COLL_ERR_INVALID_ARG);
  /* every output of an all-reduce the same buffer */
  void* same[4] = {recv[0], recv[0], recv[0], recv[0]};
  CHECK(coll_all_reduce(send, same, 4, 16, COLL_BF16, COLL_SUM, COLL_ALGO_TWOSHOT, NULL, 0, NULL) ==
        COLL_ERR_ALIAS);
  /* zero elements: nothing to do */
  CHECK(coll_all_reduce(send, recv, 4, 0, COLL_BF16, COLL_SUM, COLL_ALGO_TWOSHOT, NULL, 0, NULL) == COLL_OK);

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
