/*
 * A plain C caller of libsca (include/sca.h), host-side calls only, so it
 * runs without a GPU: it lays out the 480p long session (12 cached 480p
 * segments and the current one; a 480p segment is 31 latent frames of
 * 15 x 26 tokens, a 128-token head and four 32-token action tails whose
 * windows split the frames 8/8/8/7), builds the mask metadata, reads the
 * counts and the schedule back, then makes two calls that must fail
 * validation and prints their error codes and messages.
 *
 * Output, one line each:
 *   counts <A> <n_queries> <n_cache_keys> <n_q_tiles> <n_kv_tiles> <nnz> <n_full> <n_partial>
 *   schedule <row_ptr[n_q_tiles]> <first kv_tile> <first flag>
 *   bad_segment <code> <message>
 *   bad_window <code> <message>
 */
#include <stdio.h>

#include "sca.h"

int main(void) {
  int32_t len[4] = {32, 32, 32, 32};
  int32_t begin[4] = {0, 8, 16, 24};
  int32_t end[4] = {8, 16, 24, 31};
  sca_segment seg = {31, 15 * 26, 128, 4, len, begin, end};
  sca_segment cached[12];
  for (int i = 0; i < 12; ++i) cached[i] = seg;

  sca_metadata* md = NULL;
  if (sca_metadata_create(&md) != SCA_OK) return 1;
  int rc = sca_build_segment_mask_metadata(md, cached, 12, &seg, 1, SCA_TEXTQ_OWN_TAIL);
  if (rc != SCA_OK) {
    printf("build failed %d %s\n", rc, sca_last_error());
    return 1;
  }
  int64_t a = 0, nq = 0, nc = 0, nnz = 0, nf = 0, np = 0;
  int32_t nqt = 0, nkt = 0;
  if (sca_metadata_get_counts(md, &a, &nq, &nc, &nqt, &nkt, &nnz, &nf, &np) != SCA_OK) return 1;
  printf("counts %lld %lld %lld %d %d %lld %lld %lld\n", (long long)a, (long long)nq,
         (long long)nc, nqt, nkt, (long long)nnz, (long long)nf, (long long)np);

  const int32_t* row_ptr = NULL;
  const int32_t* kv_tile = NULL;
  const uint8_t* flag = NULL;
  if (sca_metadata_get_schedule(md, &row_ptr, &kv_tile, &flag) != SCA_OK) return 1;
  printf("schedule %d %d %d\n", row_ptr[nqt], kv_tile[0], (int)flag[0]);

  sca_segment bad = seg;
  bad.num_frames = 0;
  rc = sca_build_segment_mask_metadata(md, NULL, 0, &bad, 1, SCA_TEXTQ_OWN_TAIL);
  printf("bad_segment %d %s\n", rc, sca_last_error());

  int32_t bad_end[4] = {8, 16, 24, 32}; /* past the last frame */
  bad = seg;
  bad.action_end = bad_end;
  rc = sca_build_segment_mask_metadata(md, NULL, 0, &bad, 1, SCA_TEXTQ_OWN_TAIL);
  printf("bad_window %d %s\n", rc, sca_last_error());

  sca_metadata_destroy(md);
  return 0;
}
