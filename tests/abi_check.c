/* A plain C99 program against include/tilemix.h: the library's host entry
 * points and the synchronous argument checks of its device entry points,
 * called with no Python and no C++ in between.  Prints "ok" and exits 0, or
 * names the first check that failed and exits 1.  Touches no GPU: every
 * device call here is rejected before anything is enqueued. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "tilemix.h"

#define CHECK(cond)                                            \
  do {                                                         \
    if (!(cond)) {                                             \
      printf("failed: %s (line %d)\n", #cond, __LINE__);       \
      return 1;                                                \
    }                                                          \
  } while (0)

int main(void) {
  CHECK(tilemix_version() == TILEMIX_VERSION);
  CHECK(strcmp(tilemix_status_string(TILEMIX_OK), "ok") == 0);

  /* grouping factor: the smallest g with ceil(ceil(L / 64) / g) <= 64 */
  int g = 0;
  CHECK(tilemix_auto_g(4096, &g) == TILEMIX_OK && g == 1);
  CHECK(tilemix_auto_g(4097, &g) == TILEMIX_OK && g == 2);
  CHECK(tilemix_auto_g(-1, &g) == TILEMIX_ERR_INVALID_ARG);

  /* a ragged batch with an empty sequence: 300, 0, 64 tokens */
  const int32_t cu[4] = {0, 300, 300, 364};
  int32_t cq[4], ck[4];
  CHECK(tilemix_tile_offsets(cu, 3, cq, ck) == TILEMIX_OK);
  CHECK(cq[1] == 3 && cq[2] == 3 && cq[3] == 4);
  CHECK(ck[1] == 5 && ck[2] == 5 && ck[3] == 6);

  /* routing words: all FP16 at 0%, every legal group INT8 at 100% */
  const int32_t gs[3] = {1, 1, 1};
  uint64_t words[4 * 2];
  int64_t legal[3], int8[3];
  CHECK(tilemix_build_routing(TILEMIX_SPTRANS, 0, 0, cu, 3, 2, gs, 1, words, legal, int8) ==
        TILEMIX_OK);
  for (int i = 0; i < 8; ++i) CHECK(words[i] == 0);
  CHECK(tilemix_build_routing(TILEMIX_BAND, 100, 0, cu, 3, 2, gs, 1, words, legal, int8) ==
        TILEMIX_OK);
  /* sequence 0 (300 tokens, causal): rows of 128 reach key tiles 1, 3, 4 */
  CHECK(words[0] == 0x3 && words[2] == 0xF && words[4] == 0x1F);
  CHECK(words[1] == words[0]); /* the same word for each KV head */
  CHECK(legal[0] == 2 + 4 + 5 && int8[0] == legal[0] && legal[1] == 0);

  /* runs of the host-buffer call: two runs of about half the tokens each */
  int32_t starts[3];
  int nruns = 0;
  CHECK(tilemix_host_runs(cu, 3, 2, starts, &nruns) == TILEMIX_OK);
  CHECK(nruns == 2 && starts[0] == 0 && starts[1] == 1 && starts[2] == 3);

  /* device entry points reject bad arguments before touching the GPU */
  tilemix_prefill_args a;
  memset(&a, 0, sizeof(a));
  a.d = 96;
  a.hq = a.hk = 1;
  CHECK(tilemix_prefill_fwd(&a, NULL) == TILEMIX_ERR_UNSUPPORTED);
  a.d = 128;
  a.hq = 3;
  a.hk = 2;
  CHECK(tilemix_prefill_fwd(&a, NULL) == TILEMIX_ERR_INVALID_ARG);
  CHECK(tilemix_prefill_fwd(NULL, NULL) == TILEMIX_ERR_INVALID_ARG);
  CHECK(tilemix_prefill_host(NULL, NULL) == TILEMIX_ERR_INVALID_ARG);
  size_t bytes = 0;
  CHECK(tilemix_workspace_size(NULL, &bytes) == TILEMIX_ERR_INVALID_ARG);

  printf("ok\n");
  return 0;
}
