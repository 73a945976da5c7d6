/* A plain C client of libmoda.so: compiles against include/moda.h as C99
 * (no C++), links, and calls only entry points that validate arguments
 * without a GPU. Built and run by tests/test_abi.py. */
#include <stdio.h>

#include "moda.h"

int main(void) {
    int bad = 0;
    if (moda_abi_version() != MODA_ABI_VERSION) bad |= 1;
    /* a NULL query is rejected before any device work */
    if (moda_fwd(NULL, NULL, NULL, NULL, NULL, 1, 8, 4, 2, 64, 2, MODA_BF16, 0.125f, NULL, NULL, NULL) !=
        MODA_ERR_INVALID_VALUE)
        bad |= 2;
    /* sizes of the workspace and of the host entry's staging buffer */
    if (moda_bwd_workspace_bytes(1, 8, 4, 2, 64, 2, MODA_F32) != 256) bad |= 4;
    if (moda_fwd_host_staging_bytes(1, 8, 3, 2, 64, 2, MODA_BF16) != 0) bad |= 8;
    long long off = 0, st[4] = {0, 0, 0, 0};
    if (moda_depth_slot_layout(2, 5, 2, 4, 3, 1, &off, st) != MODA_OK || off != 8 || st[0] != 120 || st[1] != 24 ||
        st[2] != 4 || st[3] != 1)
        bad |= 16;
    printf("%s %d\n", moda_status_string(MODA_ERR_WORKSPACE), bad);
    return bad;
}
