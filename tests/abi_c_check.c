/* A plain C99 caller of the library: include/moe.h must compile as C, and the
 * entry points must link and reject bad arguments before touching a GPU (the
 * calls below all fail in argument checking, so no device is needed).
 * Built and run by tests/test_abi_from_c.py. */
#include <stdio.h>

#include "../include/moe.h"

static int fails = 0;

static void expect(int got, int want, const char* what) {
    if (got != want) {
        fprintf(stderr, "%s: got %d (%s), want %d\n", what, got, moe_status_string(got), want);
        ++fails;
    }
}

int main(void) {
    moe_config cfg = {64, 4096, 192, 8, 1536, 2.826f, 0u};
    const size_t ws = moe_workspace_size(&cfg);
    if (ws == 0) {
        fprintf(stderr, "workspace size 0 for the Hy3 decode shape\n");
        ++fails;
    }
    moe_config bad = cfg;
    bad.d = 100;
    if (moe_workspace_size(&bad) != 0) {
        fprintf(stderr, "unsupported d accepted\n");
        ++fails;
    }
    bad = cfg;
    bad.flags = MOE_FLAG_STREAM_PATH | MOE_FLAG_GEMM_PATH;
    if (moe_workspace_size(&bad) != 0) {
        fprintf(stderr, "both path flags accepted\n");
        ++fails;
    }
    /* NULL inputs are argument errors, reported before any launch */
    expect(moe_forward(&cfg, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, ws, NULL),
           MOE_ERR_INVALID_ARG, "moe_forward(NULL...)");
    expect(moe_route(NULL, NULL, NULL, NULL, NULL, NULL, NULL, ws, NULL), MOE_ERR_INVALID_ARG,
           "moe_route(NULL cfg)");
    expect(moe_combine(&bad, NULL, NULL, NULL, NULL, NULL, ws, NULL), MOE_ERR_INVALID_ARG,
           "moe_combine(bad flags)");
    if (moe_status_string(MOE_ERR_TIMEOUT) == NULL) ++fails;
    if (fails == 0) printf("ok\n");
    return fails ? 1 : 0;
}
