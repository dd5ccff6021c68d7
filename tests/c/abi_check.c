/*
 * Compiled and run by the boundary tests: include/moe_b200.h used from plain
 * C11, linked against the library, host-side calls only (queries and calls
 * that validation rejects before any launch, so no GPU is needed).
 * Exit status 0 when every check holds; otherwise the number of the failed check.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe_b200.h"

#define CHECK(n, cond)                                  \
    do {                                                \
        if (!(cond)) {                                  \
            fprintf(stderr, "check %d failed\n", (n));  \
            return (n);                                 \
        }                                               \
    } while (0)

int main(void) {
    const char *v = moe_version();
    CHECK(1, v != NULL && strstr(v, "sm_100a") != NULL);

    /* empty calls succeed and launch nothing */
    CHECK(2, moe_route_topk(NULL, NULL, 0, 8, 2, NULL, NULL, NULL, NULL) == MOE_OK);
    CHECK(3, moe_last_error()[0] == '\0');

    /* rejected on the host with the documented status and a message */
    CHECK(4, moe_route_topk(NULL, NULL, -1, 8, 2, NULL, NULL, NULL, NULL) == MOE_ERR_INVALID_ARGUMENT);
    CHECK(5, moe_last_error()[0] != '\0');
    CHECK(6, moe_route_topk(NULL, NULL, 4, 8, 9, NULL, NULL, NULL, NULL) == MOE_ERR_UNSUPPORTED_SHAPE);
    CHECK(7, moe_matmul_id(NULL, NULL, NULL, NULL, 4, 32, 37, 2, 8, 0, NULL, 0, NULL) ==
                 MOE_ERR_UNSUPPORTED_SHAPE);

    /* workspace queries: positive for a valid shape, 0 for a rejected one */
    size_t ws = moe_ffn_workspace(4096, 4096, 1536, 8, 256, MOE_LAYOUT_SHARED_PER_TOKEN);
    CHECK(8, ws > (size_t)2 * 32768 * 1536 * 2);
    CHECK(9, moe_ffn_workspace(4096, 4096, 1536, 0, 256, 0) == 0);
    CHECK(10, moe_matmul_id_workspace(8, 1536, 4096, 8, 256, 0) > 0);
    CHECK(11, moe_expert_map_workspace(4, 2, 2000) == 0);
    CHECK(12, moe_ffn_shared_workspace(64, 64, 32, 48, 2, 4) > moe_ffn_workspace(64, 64, 32, 2, 4, 0));

    /* a workspace that is too small is refused before any launch */
    uint8_t fake[256] __attribute__((aligned(256)));
    CHECK(13, moe_expert_map((const int32_t *)(uintptr_t)0x10000, 4, 2, 8, (int32_t *)fake,
                             (int32_t *)fake, (int32_t *)fake, (int32_t *)fake, fake, 16,
                             NULL) == MOE_ERR_WORKSPACE_TOO_SMALL);
    printf("abi ok\n");
    return 0;
}
