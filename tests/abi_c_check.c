/* abi_c_check.c -- the C ABI of include/attn.h used from plain C99.
 *
 * Host-side entry points and argument errors only: every device entry point
 * is called with arguments that fail validation before any device work, so
 * the program runs the same with or without a GPU.  Expected values follow
 * from the mask definitions (causal: key j allowed for query i iff
 * j <= i + Nkv - Nq; frames: query frame f sees key frames {0, f-1, f}).
 * Exit status 0 and "ok" on success.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "attn.h"

static int fails = 0;
#define EXPECT(c)                                                   \
  do {                                                              \
    if (!(c)) {                                                     \
      fprintf(stderr, "%s:%d: failed: %s\n", __FILE__, __LINE__, #c); \
      ++fails;                                                      \
    }                                                               \
  } while (0)

int main(void) {
  void* fake = (void*)0x10000; /* never dereferenced: each call below fails validation first */
  char buf[256];
  const char* v = attn_version();
  EXPECT(v != NULL && strlen(v) > 0);

  /* Frame map: 24 frames of 1040 tokens; 69 live (query frame, key frame)
     pairs, each a 65 x 65 square of 16 x 16 blocks. */
  {
    const int nf = 24, fl = 1040, nb = nf * fl / 16;
    uint8_t* map = (uint8_t*)malloc((size_t)nb * nb);
    long live = 0;
    int i;
    EXPECT(map != NULL);
    EXPECT(attn_frame_block_map(nf, fl, map) == ATTN_OK);
    for (i = 0; i < nb * nb; ++i) live += map[i];
    EXPECT(live == 69L * (fl / 16) * (fl / 16));
    EXPECT(map[0] == 1);                                /* frame 0 sees itself */
    EXPECT(map[(size_t)(5 * 65) * nb + 4 * 65] == 1);    /* frame 5 sees frame 4 */
    EXPECT(map[(size_t)(5 * 65) * nb + 3 * 65] == 0);    /* but not frame 3 */
    EXPECT(map[(size_t)(5 * 65) * nb + 6 * 65] == 0);    /* nor frame 6 */
    EXPECT(attn_frame_block_map(2, 100, map) == ATTN_ERR_SHAPE); /* 100 is not a multiple of 16 */
    free(map);
  }

  /* Tile classes, causal 256 x 256 on 128 x 128 tiles: diagonal partial,
     below it full, above it empty. */
  {
    uint8_t cls[4] = {9, 9, 9, 9};
    EXPECT(attn_classify(ATTN_MASK_CAUSAL, NULL, 256, 256, 128, 128, cls) == ATTN_OK);
    EXPECT(cls[0] == 2 && cls[1] == 0 && cls[2] == 1 && cls[3] == 2);
    EXPECT(attn_classify(ATTN_MASK_BLOCK, NULL, 256, 256, 128, 128, cls) == ATTN_ERR_MASK);
  }

  /* Causal plan of 1024 x 1024: 8 Q tiles, Q tile t visits t + 1 KV tiles. */
  {
    int nq = -1, nk = -1, t;
    int32_t qt[8][4], kt[36][3];
    EXPECT(attn_plan(ATTN_MASK_CAUSAL, NULL, 1024, 1024, NULL, 0, NULL, 0, &nq, &nk) == ATTN_OK);
    EXPECT(nq == 8 && nk == 36);
    EXPECT(attn_plan(ATTN_MASK_CAUSAL, NULL, 1024, 1024, &qt[0][0], 8, &kt[0][0], 36, &nq, &nk) == ATTN_OK);
    for (t = 0; t < 8; ++t) EXPECT(qt[t][0] == 128 * t && qt[t][1] == 128 && qt[t][3] == t + 1);
    EXPECT(attn_plan(ATTN_MASK_CAUSAL, NULL, 1024, 1024, &qt[0][0], 7, &kt[0][0], 36, &nq, &nk) ==
           ATTN_ERR_SHAPE); /* capacity too small */
  }

  /* Argument errors carry a status and a message; nothing aborts. */
  EXPECT(attn_fwd(NULL, fake, fake, fake, NULL, 1, 2, 2, 16, 16, 64, 0.125f, ATTN_MASK_NONE, NULL, ATTN_BF16,
                  NULL) == ATTN_ERR_NULL);
  EXPECT(attn_last_error_detail(buf, (int)sizeof buf) == ATTN_OK && strlen(buf) > 0);
  EXPECT(attn_fwd(fake, fake, fake, fake, NULL, 1, 3, 2, 16, 16, 64, 0.125f, ATTN_MASK_NONE, NULL, ATTN_BF16,
                  NULL) == ATTN_ERR_SHAPE); /* Hq not a multiple of Hkv */
  EXPECT(attn_fwd(fake, fake, fake, fake, NULL, 1, 2, 2, 16, 16, 96, 0.125f, ATTN_MASK_NONE, NULL, ATTN_BF16,
                  NULL) == ATTN_ERR_UNSUPPORTED); /* d = 96 */
  EXPECT(attn_fwd(fake, fake, fake, fake, NULL, 1, 2, 2, 16, 16, 64, 0.125f, ATTN_MASK_BLOCK, NULL, ATTN_BF16,
                  NULL) == ATTN_ERR_MASK); /* BLOCK without a map */
  EXPECT(attn_decode(fake, fake, fake, (const int32_t*)fake, fake, NULL, 1, 12, 4, 64, 128, 0.1f, NULL) ==
         ATTN_ERR_UNSUPPORTED); /* 3 query heads per KV head */
  EXPECT(attn_decode_multi(fake, fake, fake, (const int32_t*)fake, fake, NULL, 1, 5, 8, 2, 64, 128, 0.1f, NULL) ==
         ATTN_ERR_UNSUPPORTED); /* (Hq/Hkv) * Sq = 20 > 16 */
  EXPECT(attn_bwd(fake, fake, fake, fake, (const float*)fake, fake, fake, fake, fake, 1, 2, 2, 16, 16, 64, 0.125f,
                  9, NULL, NULL) == ATTN_ERR_MASK);
  EXPECT(attn_key_stats(fake, (float*)fake, (float*)fake, 1, 0, 2, 64, NULL) == ATTN_ERR_SHAPE);
  EXPECT(attn_shutdown() == ATTN_OK);

  if (fails) return 1;
  printf("ok\n");
  return 0;
}
