/*
 * A C99 consumer of libba: compiles against include/ba.h and
 * include/ba_graph.h with a C compiler, links the shared library and checks
 * the entry points that need no GPU (layout helpers, workspace queries,
 * status strings, argument checks that return before any CUDA call).
 * Prints "ok" and exits 0 when every check holds.
 */
#include <stdio.h>
#include <string.h>

#include "ba_graph.h"

static int failures = 0;

#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
            ++failures;                                                    \
        }                                                                  \
    } while (0)

int main(void)
{
    void* fake = (void*)(uintptr_t)(1u << 20);
    ba_fwd_graph* graph = (ba_fwd_graph*)fake;

    /* layout helpers: W = ceil(d / 32) words per token, code rows padded to 16 */
    CHECK(ba_words(1) == 1 && ba_words(32) == 1 && ba_words(33) == 2 && ba_words(128) == 4);
    CHECK(ba_vq_ld(1) == 16 && ba_vq_ld(577) == 592 && ba_vq_ld(16384) == 16384);

    /* workspace of the fused forward: staged key tiles, none for invalid sizes */
    CHECK(ba_attention_workspace_bytes(1, 1, 256, 64, BA_BIAS_NONE, 0, 0) > 0);
    CHECK(ba_attention_workspace_bytes(0, 1, 256, 64, BA_BIAS_NONE, 0, 0) == -1);
    CHECK(ba_attention_workspace_bytes(1, 1, 9, 64, BA_BIAS_RELPOS2D_CLS, 3, 3) == -1);
    CHECK(ba_attention_bwd_workspace_bytes(1, 1, 10) > 0);
    CHECK(ba_prepass_launches(577, 64, BA_BF16) == 1);

    /* argument checks that return before the CUDA runtime is touched */
    CHECK(ba_pack_qk(NULL, BA_BF16, 1, 1, 8, 64, NULL, NULL, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_attention_fwd(fake, fake, fake, fake, fake, fake, BA_BIAS_NONE, NULL, 0, 0, 0,
                           1, 1, 8, 0, fake, 0, fake, BA_BF16, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_fwd_graph_create(fake, fake, fake, BA_BF16, 1, 1, 8, 64, fake, fake, fake, fake, fake, fake,
                              BA_BIAS_NONE, NULL, 0, 0, 0, fake, 0, fake, BA_BF16, BA_QK_AUTO, NULL)
          == BA_ERR_INVALID_ARG);
    CHECK(ba_fwd_graph_launch(NULL, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_fwd_graph_kernels(NULL) == -1);
    CHECK(ba_fwd_graph_destroy(NULL) == BA_OK);
    (void)graph;

    /* every status has a name */
    CHECK(strcmp(ba_status_string(BA_OK), "") != 0);
    CHECK(strcmp(ba_status_string(BA_ERR_DEVICE_STATUS), "") != 0);

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
