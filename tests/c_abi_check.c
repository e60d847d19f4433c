/* The C ABI used from plain C (no Python, no GPU): version and status
 * strings, the host-only views of the tile schedules, the workspace query, and
 * argument errors caught on the host before any device work.  Built and run by
 * tests/test_c_abi.py. */
#include <stdio.h>
#include <string.h>

#include "magi_bca.h"

static int fails = 0;

static void check(int cond, const char* what) {
  if (!cond) {
    printf("FAIL: %s\n", what);
    ++fails;
  }
}

int main(void) {
  printf("%s\n", magi_bca_version());
  check(strcmp(magi_bca_status_string(MAGI_BCA_OK), "ok") == 0, "status string of MAGI_BCA_OK");
  check(strlen(magi_bca_status_string(MAGI_BCA_DEVICE_TIMEOUT)) > 0, "status string of MAGI_BCA_DEVICE_TIMEOUT");

  /* training layout: 4 chunks of 1024 tokens, 16 query heads, 4 kv heads, head_dim 128 */
  int32_t offs[5] = {0, 1024, 2048, 3072, 4096};
  magi_bca_dims d;
  memset(&d, 0, sizeof d);
  d.batch = 1;
  d.seqlen_q = 4096;
  d.seqlen_kv = 4096;
  d.heads_q = 16;
  d.heads_kv = 4;
  d.head_dim = 128;
  d.n_q_chunks = 4;
  d.n_kv_chunks = 4;
  d.softmax_scale = 0.f;
  d.rms_eps = 1e-6f;

  /* forward: 32 query tiles x 16 heads, two sub-tiles per unit */
  static int32_t units[256 * 12];
  const int64_t n = magi_bca_fwd_schedule(offs, offs, &d, NULL, 0);
  check(n == 256, "forward schedule: 256 units");
  check(magi_bca_fwd_schedule(offs, offs, &d, units, 256) == n, "forward schedule: count when written");
  long long pairs = 0;
  for (int64_t i = 0; i < n && i < 256; ++i) {
    const int32_t* u = units + 12 * i;
    const int subs = u[4] >= 0 ? 2 : 1;
    pairs += (long long)subs * (u[7] - u[8]);
  }
  /* the 8 query tiles of chunk c see 8 (c + 1) kv tiles, for each of the 16 heads */
  check(pairs == 16LL * 8 * (8 + 16 + 24 + 32), "forward schedule: every visible tile pair once");

  check(magi_bca_bwd_schedule(offs, offs, &d, 148, NULL, 0) > 0, "backward schedule");
  d.deterministic = 1;
  check(magi_bca_bwd_schedule(offs, offs, &d, 148, NULL, 0) == 4 * 32,
        "deterministic backward schedule: one unit per (kv head, kv tile)");
  d.deterministic = 0;
  check(magi_bca_bwd_workspace_size(&d) > 0, "workspace size");

  /* argument errors, all caught on the host */
  check(magi_bca_fwd(NULL, NULL, NULL, offs, offs, NULL, NULL, NULL, NULL, &d, NULL) == MAGI_BCA_INVALID_ARG,
        "null tensor pointers");
  int32_t empty_chunk[5] = {0, 1024, 1024, 3072, 4096};
  check(magi_bca_fwd_schedule(empty_chunk, empty_chunk, &d, NULL, 0) == MAGI_BCA_BAD_OFFSETS, "empty chunk");
  d.head_dim = 96;
  check(magi_bca_fwd_schedule(offs, offs, &d, NULL, 0) == MAGI_BCA_UNSUPPORTED, "head_dim 96");
  d.head_dim = 128;
  d.deterministic = 2;
  check(magi_bca_bwd_schedule(offs, offs, &d, 148, NULL, 0) == MAGI_BCA_INVALID_ARG, "deterministic = 2");
  d.deterministic = 0;
  check(magi_bca_bwd_workspace_size(NULL) == 0, "workspace size of a null dims struct");

  if (fails) {
    printf("C ABI check: %d failure(s)\n", fails);
    return 1;
  }
  printf("C ABI check: ok\n");
  return 0;
}
