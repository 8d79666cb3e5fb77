/* Plain-C user of the library's host entry points (no GPU needed): builds a
 * BigBird layout and a caller CSR layout, reads their views and checks the
 * documented error codes.  Prints "ok" and returns 0 when every check holds.
 * Compiled as C11 against include/bsa.h and linked with libbsa.so by
 * tests/test_c_abi.py. */
#include <stdio.h>
#include <string.h>

#include "bsa.h"

#define CHECK(cond)                                                \
  do {                                                             \
    if (!(cond)) {                                                 \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main(void) {
  bsa_layout* lay = NULL;
  /* 2 heads, 8 blocks of 64: window 1, global block 0, one random block */
  CHECK(bsa_layout_build(2, 512, 64, 1, 1, 1, 0, NULL, &lay) == BSA_OK && lay != NULL);
  const int32_t* rp = NULL;
  const int32_t* ci = NULL;
  int64_t nnz = 0;
  int nb = 0, H = 0;
  CHECK(bsa_layout_csr(lay, &rp, &ci, &nnz, &nb, &H) == BSA_OK);
  CHECK(nb == 8 && H == 2 && rp[0] == 0 && rp[H * nb] == nnz);
  /* the global block attends every key block; every row holds block 0 */
  CHECK(rp[1] - rp[0] == 8);
  for (int r = 0; r < H * nb; ++r) {
    CHECK(rp[r + 1] > rp[r] && ci[rp[r]] == 0);
    for (int32_t x = rp[r] + 1; x < rp[r + 1]; ++x) CHECK(ci[x] > ci[x - 1] && ci[x] < nb);
  }
  const int32_t* g = NULL;
  int ng = -1;
  CHECK(bsa_layout_globals(lay, &g, &ng) == BSA_OK && ng == 1 && g[0] == 0);
  const int32_t* pair_q = NULL;
  int n_pairs = 0;
  CHECK(bsa_layout_tiles(lay, &pair_q, &n_pairs, NULL, NULL, NULL) == BSA_OK && n_pairs > 0);
  CHECK(bsa_layout_key_tiles(lay, NULL, &n_pairs, NULL, NULL, NULL) == BSA_OK && n_pairs > 0);
  size_t ws = 0, bws = 0;
  CHECK(bsa_workspace_bytes(lay, 2, &ws) == BSA_OK && ws > 0 && ws % 256 == 0);
  CHECK(bsa_backward_workspace_bytes(lay, 2, &bws) == BSA_OK && bws >= 2 * 4 * 2 * 512);

  /* the same rows given back as a caller's CSR */
  bsa_layout* lay2 = NULL;
  CHECK(bsa_layout_from_csr(2, 512, 64, rp, ci, &lay2) == BSA_OK);
  const int32_t* rp2 = NULL;
  const int32_t* ci2 = NULL;
  int64_t nnz2 = 0;
  CHECK(bsa_layout_csr(lay2, &rp2, &ci2, &nnz2, NULL, NULL) == BSA_OK && nnz2 == nnz);
  CHECK(memcmp(rp, rp2, sizeof(int32_t) * (size_t)(H * nb + 1)) == 0);
  CHECK(memcmp(ci, ci2, sizeof(int32_t) * (size_t)nnz) == 0);

  /* a token-level layout: window 70 tokens, global tokens 3 and 300 (blocks 0 and 4) */
  bsa_layout* tok = NULL;
  const int32_t gtok[2] = {300, 3};
  CHECK(bsa_layout_build_tokens(2, 512, 70, 2, 1, 7, gtok, &tok) == BSA_OK && tok != NULL);
  int tw = -1;
  const uint64_t* gbits = NULL;
  CHECK(bsa_layout_token_masks(tok, &tw, &gbits) == BSA_OK && tw == 70);
  CHECK(gbits[0] == (1ull << 3) && gbits[4] == (1ull << (300 - 256)) && gbits[1] == 0);
  CHECK(bsa_layout_globals(tok, &g, &ng) == BSA_OK && ng == 2 && g[0] == 0 && g[1] == 4);
  {
    /* its block CSR is the block layout with window ceil(70 / 64) = 2 blocks and those two blocks global */
    bsa_layout* blk = NULL;
    const int32_t gb[2] = {0, 4};
    CHECK(bsa_layout_build(2, 512, 64, 2, 2, 1, 7, gb, &blk) == BSA_OK);
    const int32_t *trp = NULL, *tci = NULL, *brp = NULL, *bci = NULL;
    int64_t tn = 0, bn = 0;
    CHECK(bsa_layout_csr(tok, &trp, &tci, &tn, NULL, NULL) == BSA_OK);
    CHECK(bsa_layout_csr(blk, &brp, &bci, &bn, NULL, NULL) == BSA_OK && tn == bn);
    CHECK(memcmp(trp, brp, sizeof(int32_t) * (size_t)(H * nb + 1)) == 0);
    CHECK(memcmp(tci, bci, sizeof(int32_t) * (size_t)tn) == 0);
    bsa_layout_free(blk);
  }
  CHECK(bsa_layout_token_masks(lay, &tw, &gbits) == BSA_ERR_UNSUPPORTED);
  bsa_layout* tbad = NULL;
  CHECK(bsa_layout_build_tokens(2, 500, 70, 0, 0, 0, NULL, &tbad) == BSA_ERR_INVALID_ARG && tbad == NULL);
  {
    const int32_t out_of_range[1] = {512};
    CHECK(bsa_layout_build_tokens(2, 512, 70, 1, 0, 0, out_of_range, &tbad) == BSA_ERR_INVALID_ARG);
  }
  size_t ws128 = 0;
  CHECK(bsa_forward_workspace_bytes(lay, 2, 128, &ws128) == BSA_OK && ws128 >= ws);
  CHECK(bsa_forward_workspace_bytes(lay, 2, 96, &ws128) == BSA_ERR_UNSUPPORTED);
  CHECK(bsa_out_projection(NULL, NULL, NULL, 1, 1, 64, 64, NULL, NULL) == BSA_ERR_INVALID_ARG);
  CHECK(bsa_qkv_projection(NULL, NULL, NULL, 1, 64, 1, NULL, NULL, NULL, NULL) == BSA_ERR_INVALID_ARG);
  bsa_layout_free(tok);

  /* documented errors, before anything touches a GPU */
  bsa_layout* bad = (bsa_layout*)1;
  CHECK(bsa_layout_build(2, 512, 96, 1, 1, 1, 0, NULL, &bad) == BSA_ERR_UNSUPPORTED && bad == NULL);
  CHECK(bsa_layout_build(0, 512, 64, 1, 1, 1, 0, NULL, &bad) == BSA_ERR_INVALID_ARG);
  CHECK(bsa_layout_build(2, 500, 64, 1, 1, 1, 0, NULL, &bad) == BSA_ERR_INVALID_ARG);
  CHECK(bsa_layout_build(2, 512, 64, 1, 1, 1, 0, NULL, NULL) == BSA_ERR_INVALID_ARG);
  CHECK(bsa_forward(NULL, NULL, NULL, 1, 2, 512, 64, lay, NULL, 0.f, NULL, NULL, NULL, 0, NULL) ==
        BSA_ERR_INVALID_ARG);
  CHECK(bsa_backward(NULL, NULL, NULL, NULL, NULL, NULL, 1, 2, 512, 64, lay, NULL, 0.f, NULL, NULL, NULL,
                     NULL, 0, NULL) == BSA_ERR_INVALID_ARG);
  CHECK(strlen(bsa_strerror(BSA_ERR_DEVICE_TIMEOUT)) > 0);

  bsa_layout_free(lay2);
  bsa_layout_free(lay);
  bsa_layout_free(NULL);
  puts("ok");
  return 0;
}
