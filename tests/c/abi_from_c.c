/* The C ABI used from plain C99 (no C++, no torch): the header compiles as C, every
 * entry point links, and the argument checks answer without a GPU.  Built and run by
 * tests/test_abi.py. */
#include <stdio.h>
#include <string.h>

#include "entattn.h"

#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__);    \
            return 1;                                                      \
        }                                                                  \
    } while (0)

int main(void) {
    /* a 16-byte aligned non-null stand-in, never dereferenced on argument errors */
    void *fake = (void *)(size_t)(1u << 20);
    float *ffake = (float *)fake;
    uint8_t *bfake = (uint8_t *)fake;
    CHECK(ent_attn_block_size() == 128);
    CHECK(ent_attn_fwd_workspace_size(1, 1, 128, 64, ENT_BF16) >= 256);
    CHECK(ent_attn_bwd_workspace_size(1, 1, 128, 64, ENT_BF16) >= 256 + 128 * 4);
    /* alpha outside (1, 2] */
    CHECK(ent_attn_fwd(fake, fake, fake, 1, 1, 128, 64, ENT_BF16, 2.5f, 1, fake, ffake, bfake,
                       NULL, fake, 256, NULL) == ENT_EINVAL);
    CHECK(strlen(ent_attn_last_error()) > 0);
    /* a head dimension the library does not implement */
    CHECK(ent_attn_bwd(fake, fake, fake, NULL, fake, ffake, bfake, 1, 1, 128, 96, ENT_BF16, 1.5f,
                       1, fake, fake, fake, fake, (size_t)1 << 30, NULL) == ENT_EUNSUPPORTED);
    /* the otilde pair wants its otilde pointer */
    CHECK(ent_attn_fwd_otilde(fake, fake, fake, 1, 1, 128, 64, ENT_BF16, 1.5f, 1, fake, ffake,
                              bfake, NULL, NULL, fake, 256, NULL) == ENT_EINVAL);
    CHECK(ent_attn_bwd_otilde(fake, fake, fake, NULL, fake, ffake, bfake, 1, 1, 128, 64, ENT_BF16,
                              1.5f, 1, fake, fake, fake, fake, (size_t)1 << 30, NULL) == ENT_EINVAL);
    CHECK(ent_attn_bwd_noalloc(fake, fake, fake, NULL, fake, ffake, bfake, 1, 1, 128, 64, ENT_BF16,
                               0.5f, 1, fake, fake, fake, NULL) == ENT_EINVAL);
    /* row-wise entmax */
    CHECK(ent_entmax_rows_max_n() == 16384);
    CHECK(ent_entmax_rows_fwd(fake, 2, 8, ENT_F32, 1.5f, 7, fake, ffake, NULL, NULL) == ENT_EINVAL);
    CHECK(ent_entmax_rows_bwd(fake, ffake, fake, 2, 99999, ENT_F32, 1.5f, fake, NULL) ==
          ENT_EUNSUPPORTED);
    CHECK(ent_attn_read_status(NULL, NULL, NULL) == ENT_EINVAL);
    /* no device here: the no-alloc status reader reports an error, never OK */
    CHECK(ent_attn_noalloc_read_status(NULL, NULL) != ENT_OK);
    printf("abi from C ok\n");
    return 0;
}
