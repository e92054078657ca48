/* Test program (C99): the host-side calls of the library, no GPU needed.
 * Prints one line per check and exits non-zero on the first failure. */
#include <stdio.h>
#include <string.h>

#include "dq.h"

static int fail(const char *what, int got) {
    printf("FAIL %s (%d)\n", what, got);
    return 1;
}

int main(void) {
    dq_format f;
    size_t bytes = 0;
    int64_t rows[2] = {4096, 1024}, cols[2] = {4096, 4096};
    if (strstr(dq_version(), "sm_100a") == NULL) return fail("version", 0);
    if (dq_format_preset("mxfp4", 32, &f) != DQ_OK) return fail("preset mxfp4", -1);
    if (f.codes != DQ_CODES_E2M1 || f.group != 32 || f.group_scale != DQ_SCALE_E8M0 ||
        f.outer_scale != DQ_SCALE_E8M0)
        return fail("mxfp4 fields", f.codes);
    if (dq_format_preset("no-such-format", 32, &f) != DQ_ERR_FORMAT) return fail("unknown preset", 0);
    if (dq_format_preset("int4_bf16", 64, &f) != DQ_OK) return fail("preset int4_bf16", -1);
    if (dq_workspace_size(2, rows, cols, &f, &bytes) != DQ_OK || bytes == 0)
        return fail("workspace size", (int)bytes);
    if (dq_code_bytes(&f, 3, 128) != 3 * 64) return fail("code bytes", (int)dq_code_bytes(&f, 3, 128));
    cols[0] = 100;                                        /* not a multiple of G */
    if (dq_workspace_size(1, rows, cols, &f, &bytes) != DQ_ERR_SHAPE) return fail("shape check", 0);
    if (dq_quantize(NULL, DQ_DT_BF16, 4, 64, &f, NULL, NULL, 1.0f, NULL, NULL, NULL) != DQ_ERR_ARG)
        return fail("null input", 0);
    if (strlen(dq_strerror(DQ_ERR_TIMEOUT)) == 0) return fail("strerror", 0);
    {
        /* graph API: argument errors come back before any CUDA call */
        dq_matrix m;
        dq_graph g = (dq_graph)&m;
        memset(&m, 0, sizeof(m));
        m.rows = 4;
        m.cols = 64;
        if (dq_graph_solve_batched(1, &m, DQ_DT_BF16, &f, 3, NULL, 0, NULL) != DQ_ERR_ARG)
            return fail("graph: no out", 0);
        if (dq_graph_solve_batched(1, &m, DQ_DT_BF16, &f, 3, NULL, 0, &g) != DQ_ERR_ARG || g != NULL)
            return fail("graph: no W", 0);
        if (dq_graph_launch(NULL, NULL) != DQ_ERR_ARG) return fail("graph: launch NULL", 0);
        if (dq_graph_launches(NULL) != 0) return fail("graph: launches NULL", 0);
        if (dq_graph_destroy(NULL) != DQ_OK) return fail("graph: destroy NULL", 0);
    }
    printf("ok %s\n", dq_version());
    return 0;
}
