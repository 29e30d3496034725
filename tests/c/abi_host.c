/*
 * Plain C (C99) user of the mixer library's C ABI: includes only
 * include/bimamba.h, links libbimamba.so, and calls the entry points that
 * need no device (version, error strings, workspace sizing, launch plans,
 * and argument checks that fail before anything is launched).  Prints
 * "abi ok" and exits 0 when every answer is the documented one.
 */
#include <stdio.h>
#include <string.h>

#include "bimamba.h"

static int fails = 0;
#define CHECK(cond)                                                     \
    do {                                                                \
        if (!(cond)) {                                                  \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            ++fails;                                                    \
        }                                                               \
    } while (0)

int main(void)
{
    CHECK((bimamba_version() >> 16) == 1);
    CHECK(strcmp(bimamba_strerror(BIMAMBA_OK), "unknown status") != 0);
    CHECK(strcmp(bimamba_strerror(99), "unknown status") == 0);

    /* the benchmarked layer takes the tensor-core path */
    bimamba_dims d = {8, 4096, 64, 64, 128, 1, 4, BIMAMBA_BF16};
    int plan[4] = {-1, -1, -1, -1};
    CHECK(bimamba_launch_plan(&d, plan) == BIMAMBA_OK);
    CHECK(plan[0] == 1 && plan[1] >= 1 && plan[2] >= 1 && plan[3] >= 0);
    CHECK(bimamba_workspace_bytes(&d) > 0);

    /* fp32 takes the sequential path and needs no workspace */
    bimamba_dims f = {1, 256, 4, 32, 16, 1, 4, BIMAMBA_F32};
    CHECK(bimamba_launch_plan(&f, plan) == BIMAMBA_OK && plan[0] == 0);
    CHECK(bimamba_workspace_bytes(&f) == 0);

    /* invalid and unsupported shapes are reported, nothing is launched */
    bimamba_dims bad = d;
    bad.heads = 0;
    CHECK(bimamba_workspace_bytes(&bad) == 0);
    CHECK(bimamba_launch_plan(&bad, plan) == BIMAMBA_ERR_INVALID);
    CHECK(bimamba_launch_plan(&d, NULL) == BIMAMBA_ERR_INVALID);
    bimamba_dims odd = d;
    odd.headdim = 12;
    CHECK(bimamba_launch_plan(&odd, plan) == BIMAMBA_ERR_UNSUPPORTED);
    CHECK(bimamba_ssd_fwd_rev(&bad, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) == BIMAMBA_ERR_INVALID);
    CHECK(bimamba_ssd_fwd_rev(&d, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) == BIMAMBA_ERR_INVALID);
    CHECK(bimamba_ssd_fwd_rev_untied(&d, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 7, 0, 0, 0) ==
          BIMAMBA_ERR_INVALID);
    CHECK(bimamba_shard_states(&f, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) == BIMAMBA_ERR_UNSUPPORTED);

    if (fails) return 1;
    printf("abi ok\n");
    return 0;
}
