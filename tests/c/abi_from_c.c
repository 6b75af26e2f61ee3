/* A plain C99 client of include/pa.h: the header compiles as C, the library
 * links without C++ or torch, and argument errors come back before anything
 * touches a GPU (this program runs on machines without one). */
#include <stdio.h>
#include <string.h>

#include "pa.h"

#define CHECK(cond)                                                    \
    do {                                                               \
        if (!(cond)) {                                                 \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__,     \
                    __LINE__, #cond);                                  \
            return 1;                                                  \
        }                                                              \
    } while (0)

int main(void) {
    CHECK(pa_abi_version() == PA_ABI_VERSION);
    CHECK(strcmp(pa_status_string(PA_OK), "ok") == 0);
    CHECK(strcmp(pa_status_string(PA_ERR_WORKSPACE), "workspace too small") == 0);

    pa_shape shape = {1, 1024, 8, 2, 64, 128, 1, 0};
    pa_budget budget = {PA_BUDGET_DYNAMIC, 0.95f, 0, 1, 0.0f};
    CHECK(pa_workspace_size(&shape, &budget) > 0);

    /* argument errors are reported synchronously, with a message */
    pa_strides st = {1024 * 8 * 64, 8 * 64, 64};
    CHECK(pa_pool_heads(&shape, NULL, st, NULL, st, NULL, NULL, NULL) == PA_ERR_INVALID_ARG);
    CHECK(strlen(pa_last_error()) > 0);
    pa_shape bad = shape;
    bad.head_dim = 96;
    CHECK(pa_prefill(&bad, &budget, NULL, st, NULL, st, NULL, st, NULL, st, NULL, NULL, 0, NULL) !=
          PA_OK);
    bad = shape;
    bad.seqlen = 1000;
    CHECK(pa_prefill(&bad, &budget, NULL, st, NULL, st, NULL, st, NULL, st, NULL, NULL, 0, NULL) !=
          PA_OK);
    printf("ok\n");
    return 0;
}
