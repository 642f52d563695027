/* A plain C99 consumer of libgnf4: includes only the public header, links the
 * shared library, and exercises the calls that need no GPU (version, shape
 * refusals, an empty call, workspace sizes, the engagement counters).
 * Exits 0 when every check holds; otherwise prints the failed check and exits 1. */
#include <stdio.h>
#include <string.h>

#include "gnf4.h"

static int failures = 0;

#define CHECK(cond)                                              \
    do {                                                         \
        if (!(cond)) {                                           \
            fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
            ++failures;                                          \
        }                                                        \
    } while (0)

int main(void) {
    const char *v = gnf4_version();
    CHECK(v != NULL && strstr(v, "sm_100a") != NULL);

    gnf4_call_stats s;
    CHECK(gnf4_call_stats_get(NULL, &s, 1) == GNF4_OK);

    /* E = 0 is refused before any pointer or device is looked at */
    int32_t dummy = 0;
    CHECK(gnf4_grouped_gemm_nf4(NULL, NULL, NULL, &dummy, NULL, 0, 64, 64, 8, NULL, NULL) ==
          GNF4_ERR_UNSUPPORTED_SHAPE);
    CHECK(strlen(gnf4_last_error()) > 0);
    /* exactly one of offsets and counts */
    CHECK(gnf4_grouped_gemm_mxfp4(NULL, NULL, NULL, NULL, NULL, 4, 64, 64, 8, NULL, NULL) == GNF4_ERR_INVALID_ARG);
    /* M = 0: nothing to enqueue */
    CHECK(gnf4_grouped_gemm_nf4(NULL, NULL, NULL, &dummy, NULL, 4, 64, 64, 0, NULL, NULL) == GNF4_OK);

    CHECK(gnf4_call_stats_get("gnf4_grouped_gemm_nf4", &s, 0) == GNF4_OK);
    CHECK(s.calls == 2 && s.refused == 1 && s.engaged == 0 && s.rows == 0);
    CHECK(gnf4_call_stats_get("gnf4_grouped_gemm_mxfp4", &s, 0) == GNF4_OK);
    CHECK(s.calls == 1 && s.refused == 1);
    CHECK(gnf4_call_stats_get("not_an_entry_point", &s, 0) == GNF4_ERR_INVALID_ARG);
    CHECK(gnf4_call_stats_get(NULL, &s, 1) == GNF4_OK && s.calls == 3);
    CHECK(gnf4_call_stats_get(NULL, &s, 0) == GNF4_OK && s.calls == 0);

    int n = 0;
    while (gnf4_call_stats_name(n) != NULL) ++n;
    CHECK(n > 20);
    CHECK(strncmp(gnf4_call_stats_name(0), "gnf4_", 5) == 0);

    /* workspace sizes are pure host arithmetic */
    CHECK(gnf4_route_workspace_bytes(0, 2, 8) == 0);
    CHECK(gnf4_route_workspace_bytes(4096, 8, 384) > 0);
    CHECK(gnf4_grouped_gemm_mxfp4_workspace_bytes(1, 128) == 2 * 128 + 2 * 16);
    CHECK(gnf4_grouped_gemm_mxfp4_workspace_bytes(8, 96) == 0);
    CHECK(gnf4_grouped_gemm_mxfp4_native_max_rows() == 96);

    if (failures == 0) printf("c consumer ok (%d counted entry points)\n", n);
    return failures == 0 ? 0 : 1;
}
