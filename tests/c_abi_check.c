/* A C caller of libra_b200.so: the boundary used with nothing but include/ra.h,
 * a C compiler and the shared library (no Python, no CUDA headers).
 *
 * Every call below returns before any CUDA work: status strings, the
 * workspace and plan queries, and argument validation, which the library
 * does synchronously on the host.  Built and run by tests/test_abi.py;
 * prints "ok <checks>" and exits 0, or names the first failed check and
 * exits 1. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ra.h"

static int checks = 0;

#define CHECK(cond)                                                  \
  do {                                                               \
    ++checks;                                                        \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
      return 1;                                                      \
    }                                                                \
  } while (0)

int main(void) {
  /* an aligned, non-null address that validation never dereferences */
  void* const P = (void*)(uintptr_t)(1u << 20);
  const size_t none = (size_t)-1;

  CHECK(strcmp(ra_status_string(RA_OK), "RA_OK") == 0);
  CHECK(strcmp(ra_status_string(RA_ERR_TIMEOUT), "RA_ERR_TIMEOUT") == 0);
  CHECK(strcmp(ra_status_string((ra_status)99), "RA_ERR_UNKNOWN") == 0);
  CHECK(strstr(ra_version(), "sm_100a") != NULL);

  /* workspace: none for bf16 inputs on the default path; bf16 copies of
   * Q, K, V for fp32 inputs; invalid shapes give (size_t)-1 */
  CHECK(ra_ring_attention_workspace(1, 24000, 32, 128, 4, 4, RA_PART_ZIGZAG, RA_BF16, RA_F32, NULL) == 0);
  CHECK(ra_ring_attention_workspace(1, 24000, 32, 128, 4, 4, RA_PART_ZIGZAG, RA_F32, RA_F32, NULL) >=
        (size_t)24000 * (32 + 8 + 8) * 128 * 2);
  CHECK(ra_ring_attention_workspace(1, 4095, 8, 128, 4, 1, RA_PART_ZIGZAG, RA_BF16, RA_F32, NULL) == none);
  CHECK(ra_ring_attention_backward_workspace(1, 24000, 32, 128, 4, 4, RA_PART_ZIGZAG, RA_BF16) >=
        (size_t)2 * 24000 * 32 * 4);
  CHECK(ra_ring_attention_backward_workspace(1, 4095, 8, 128, 4, 1, RA_PART_ZIGZAG, RA_BF16) == none);
  CHECK(ra_noalloc_scratch_bytes() == ((size_t)64 << 20));
  CHECK(ra_decode_splits(1, 1, 10, 8, 3, 128, 0) == -1); /* Hq not a multiple of Hkv */
  /* 5 chunks asked of 1,000 keys: 200 keys rounded up to 256, so 4 chunks */
  CHECK(ra_decode_splits(2, 3, 1000, 8, 2, 128, 5) == 4);
  CHECK(ra_decode_workspace(2, 3, 1000, 8, 2, 128, 5) >= (size_t)4 * 2 * 3 * 8 * 129 * 4);

  /* validation, before any launch */
  CHECK(ra_ring_attention(P, P, P, RA_BF16, 1, 4100, 8, 128, 4, 1, RA_PART_ZIGZAG, 1, P, RA_F32, (float*)P, P,
                          (size_t)1 << 40, NULL, NULL) == RA_ERR_INVALID_ARG); /* S % 2n != 0 */
  CHECK(ra_ring_attention(P, P, P, RA_BF16, 1, 4096, 8, 96, 4, 1, RA_PART_ZIGZAG, 1, P, RA_F32, (float*)P, P,
                          (size_t)1 << 40, NULL, NULL) == RA_ERR_UNSUPPORTED); /* D = 96 */
  CHECK(ra_ring_attention_noalloc(NULL, P, P, RA_BF16, 1, 4096, 8, 128, 4, 1, RA_PART_ZIGZAG, 1, P, RA_F32,
                                  (float*)P, NULL, NULL) == RA_ERR_INVALID_ARG);
  CHECK(ra_block_attn(P, P, P, RA_BF16, 1, 1024, 4, 4, 0, 4, 2, 128, 1, RA_PART_ZIGZAG, (float*)P, (float*)P,
                      NULL) == RA_ERR_INVALID_ARG); /* q_block out of range */
  CHECK(ra_block_attn_merge(P, P, P, RA_F32, 1, 1024, 4, 0, 0, 4, 2, 128, 1, RA_PART_ZIGZAG, (float*)P,
                            (float*)P, NULL) == RA_ERR_UNSUPPORTED); /* fp32 block inputs */
  CHECK(ra_merge_partial((float*)P, (float*)P, (const float*)P, (const float*)P, 0, 128, NULL) == RA_OK);
  CHECK(ra_merge_partial((float*)P, (float*)P, (const float*)P, (const float*)P, -1, 128, NULL) ==
        RA_ERR_INVALID_ARG);
  CHECK(ra_zigzag_permute(P, P, 1, 96, 2, 8, 2, 3, 0, NULL) == RA_ERR_INVALID_ARG); /* in place */
  CHECK(ra_decode_attention(P, P, P, RA_BF16, 1, 5000, 4096, 8, 2, 128, 1, 0, P, RA_F32, (float*)P, P,
                            (size_t)1 << 40, NULL) == RA_ERR_INVALID_ARG); /* Tq > Skv */
  CHECK(ra_ring_attention_backward(P, P, P, RA_BF16, P, RA_F32, (const float*)P, P, 1, 4096, 8, 128, 4, 1,
                                   RA_PART_ZIGZAG, 2, (float*)P, (float*)P, (float*)P, NULL, 0, NULL,
                                   NULL) == RA_ERR_WORKSPACE); /* the backward always needs its workspace */
  {
    ra_options o;
    memset(&o, 0, sizeof(o));
    o.order = 9; /* no such order */
    CHECK(ra_ring_attention(P, P, P, RA_BF16, 1, 4096, 8, 128, 4, 1, RA_PART_ZIGZAG, 1, P, RA_F32, (float*)P, P,
                            (size_t)1 << 40, &o, NULL) == RA_ERR_INVALID_ARG);
  }
  printf("ok %d\n", checks);
  return 0;
}
