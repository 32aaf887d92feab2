/* A plain C99 client of libfca_b200.so: the boundary needs no C++ and no
 * torch.  Calls only entry points that stop at their host-side checks, so it
 * runs without a GPU.  Prints one line the test compares. */
#include <stdio.h>
#include "fca.h"

int main(void)
{
    fca_plan_opts o;
    fca_plan_t plan = NULL;
    int32_t word = -1;
    fca_plan_opts_default(&o);
    /* null tables: refused before any device work, no plan handed out */
    fca_status s_plan = fca_plan(NULL, 4, NULL, 2, 16, 8, 4, 1, 64, &o, &plan, NULL);
    /* head_dim 96 is not built */
    fca_status s_dim = fca_plan((const int32_t *)16, 4, (const int32_t *)16, 2, 16, 8, 4, 1, 96, &o, &plan, NULL);
    fca_status s_upd = fca_plan_update(NULL, NULL, 4, NULL, 2, NULL);
    fca_status s_self = fca_selftest_wait_timeout(NULL, NULL);
    fca_status s_destroy = fca_plan_destroy(NULL);
    printf("%s|%s|%d|%d|%d|%d|%d|%d|%d|%d|%d\n", fca_version(), fca_status_string(FCA_ERR_BAD_BLOCK_ID),
           (int)s_plan, (int)s_dim, plan == NULL, (int)s_upd, (int)s_self, (int)s_destroy,
           o.min_group_size, o.min_saved_blocks, (int)word);
    return 0;
}
