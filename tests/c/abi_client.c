/* A plain C99 client of libqlinear.so: the header compiles as C, the library links, and the calls
 * that need no GPU behave as the header states (argument errors are returned before any launch). */
#include <stdio.h>
#include <string.h>

#include "qlinear.h"

#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
            return 1;                                                 \
        }                                                             \
    } while (0)

int main(void) {
    void* const fake = (void*)(size_t)0x10000000u;   /* never dereferenced: rejected before any launch */
    char buf[64];
    CHECK(qlinear_version() == 100);
    CHECK(strcmp(qlinear_status_string(QL_ERR_WORKSPACE), "QL_ERR_WORKSPACE") == 0);
    CHECK(qlinear_workspace_size(16, 100, 256, 64) == (size_t)-1);
    CHECK(qlinear8_workspace_size(16, 100, 256, 64) == (size_t)-1);
    CHECK(qlinear_forward(fake, (const uint32_t*)fake, fake, fake, fake, 16, 256, 256, 32, NULL, 0, 0) ==
          QL_ERR_UNSUPPORTED);
    CHECK(qlinear8_forward(NULL, (const uint32_t*)fake, fake, fake, fake, 16, 256, 256, 64, NULL, 0, 0) ==
          QL_ERR_INVALID_ARG);
    CHECK(qlinear_swiglu_forward(fake, NULL, fake, fake, (const uint32_t*)fake, fake, fake, fake, QL_BF16, 16, 256,
                                 256, 64, fake, 1u << 20, 0) == QL_ERR_INVALID_ARG);
    CHECK(qlinear_reduce_partials(NULL, 2, 64, fake, QL_BF16, 0) == QL_ERR_INVALID_ARG);
    CHECK(qlinear_last_dispatch(NULL, 8) == QL_ERR_INVALID_ARG);
    CHECK(qlinear_last_dispatch(buf, sizeof buf) == QL_OK);
    printf("c abi client ok\n");
    return 0;
}
