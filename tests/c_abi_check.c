/* Compiled as C11 against include/ftk.h and linked with libftk.so by
 * tests/test_abi.py: the header is plain C and the host-side entry points
 * (no GPU needed) answer as documented. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include "ftk.h"

static int fail(const char *what)
{
    printf("FAIL %s\n", what);
    return 1;
}

int main(void)
{
    if (ftk_version() <= 0) return fail("version");
    if (!ftk_status_string(FTK_ERR_TOPK_RANGE) || !ftk_status_string(12345)) return fail("status strings");
    ftk_rows_options o;
    ftk_rows_options_init(&o);
    if (o.sorted != 0 || o.index_bits != 32 || o.out_stride != 0 || o.idx_fill != -1 || !isinf(o.val_fill) ||
        o.val_fill > 0)
        return fail("rows options defaults");
    ftk_config c = {0};
    const size_t n = ftk_select_workspace_size(4096, 131072, 2048, &c);
    if (n == 0 || n != ftk_select_workspace_size(4096, 131072, 2048, NULL)) return fail("workspace size");
    if (ftk_select_workspace_size(0, 10, 5, NULL) != 0) return fail("workspace size of T = 0");
    /* host-side argument errors return before any device work */
    if (ftk_topk_rows(FTK_BF16, NULL, 4, 100, 104, 8, (int32_t *)0x10000, NULL, NULL, NULL) !=
        FTK_ERR_INVALID_ARG)
        return fail("topk_rows NULL x");
    if (ftk_select(FTK_F8E4M3, (void *)0x10000, (void *)0x10000, NULL, (float *)0x10000, (int32_t *)0x10000,
                   (int32_t *)0x10000, 16, 1000, 0, (int32_t *)0x10000, NULL, (void *)0x10000, n, NULL,
                   NULL) != FTK_ERR_TOPK_RANGE)
        return fail("select topk 0");
    printf("OK\n");
    return 0;
}
