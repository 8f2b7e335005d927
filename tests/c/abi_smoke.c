/* A plain C caller of the library's ABI (no Python, no GPU needed):
 * host-only planning, argument validation and status strings. */
#include <stdio.h>
#include <string.h>

#include "flce.h"

static int fail(const char* what) {
  fprintf(stderr, "FAIL: %s\n", what);
  return 1;
}

int main(void) {
  if (flce_version() != FLCE_VERSION) return fail("version");
  flce_options opt;
  flce_options_init(&opt);
  flce_stats st;
  /* Llama-3-8B lm_head: 4096 tokens x 4096 hidden x 128256 vocabulary, bf16 */
  if (flce_plan(4096, 4096, 128256, FLCE_BF16, 1, &opt, &st) != FLCE_OK) return fail("plan");
  if (st.n_chunks < 2 || st.chunk_rows % 128 != 0) return fail("chunking");
  if (st.workspace_bytes >= st.materialized_logits_bytes) return fail("workspace bound");
  printf("chunk_rows=%lld n_chunks=%lld workspace=%lld logits=%lld\n", (long long)st.chunk_rows,
         (long long)st.n_chunks, (long long)st.workspace_bytes, (long long)st.materialized_logits_bytes);
  /* validation happens on the host, before any device work */
  flce_tensor X, W, t, loss;
  memset(&X, 0, sizeof(X));
  memset(&W, 0, sizeof(W));
  memset(&t, 0, sizeof(t));
  memset(&loss, 0, sizeof(loss));
  if (flce_fwd_bwd(NULL, &W, &t, -100, FLCE_MEAN, &loss, NULL, NULL, NULL) != FLCE_ERR_INVALID_ARG)
    return fail("null X");
  X.dtype = FLCE_BF16;
  W.dtype = FLCE_F32;
  if (flce_fwd_bwd(&X, &W, &t, -100, FLCE_MEAN, &loss, NULL, NULL, NULL) != FLCE_ERR_UNSUPPORTED_DTYPE)
    return fail("dtype mix");
  if (strcmp(flce_status_string(FLCE_OK), "ok") != 0) return fail("status string");
  if (flce_workspace_bytes(4096, 4096, 128256, FLCE_BF16, &opt) != (size_t)st.workspace_bytes)
    return fail("workspace bytes");
  /* two-phase planning: one chunk holding the whole batch, in a caller workspace */
  flce_options keep;
  flce_options_init(&keep);
  keep.flags = FLCE_FLAG_KEEP_LOGITS;
  flce_stats kst;
  if (flce_plan(4096, 4096, 128256, FLCE_BF16, 1, &keep, &kst) != FLCE_OK) return fail("keep plan");
  if (kst.n_chunks != 1 || kst.chunk_rows != 4096) return fail("keep chunking");
  if (kst.workspace_bytes < kst.materialized_logits_bytes) return fail("keep workspace holds the store");
  if (flce_plan(40000, 4096, 128256, FLCE_BF16, 1, &keep, &kst) != FLCE_ERR_INVALID_ARG)
    return fail("keep limit");
  printf("ok\n");
  return 0;
}
