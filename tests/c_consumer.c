/* A plain C99 user of the libmoe boundary: includes the header, links the
 * library and makes the calls that need no GPU (version, status strings,
 * capacity and buffer-size queries, host-side argument validation). */
#include <stdio.h>

#include "libmoe.h"

int main(void) {
    printf("abi %d\n", moe_abi_version());
    printf("status %s\n", moe_status_string(MOE_ERR_SHAPE));
    printf("capacity %lld\n", (long long)moe_capacity(1.25, 8192, 2, 8));
    printf("max_rows %lld %lld\n", (long long)moe_permute_max_rows(8192, 2, 8, 1.25, 0),
           (long long)moe_permute_max_rows(4096, 8, 256, 0.0, 8));
    printf("ws %d\n", moe_permute_workspace_bytes(8192, 2, 8, 0) > 0);
    /* rejected on the host before any launch: k > E, then T = 0 (nothing to do) */
    printf("k>E %d\n", (int)moe_route_topk(NULL, 16, 8, 9, 0, NULL, NULL, NULL));
    printf("T=0 %d\n", (int)moe_route_topk(NULL, 0, 8, 2, 0, NULL, NULL, NULL));
    return 0;
}
