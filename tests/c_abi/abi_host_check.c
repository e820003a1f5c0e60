/* A plain C program against include/zero_adam.h and libzero_adam.so: the
 * host-only entry points with the values the pages print, and argument
 * errors that are rejected before any device call.  Exit status 0 when
 * every check holds; the failing check is printed otherwise. */
#include <stdio.h>
#include <string.h>

#include "zero_adam.h"

static int failures = 0;

#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            ++failures;                                               \
        }                                                             \
    } while (0)

int main(void) {
    /* Owners of 11 parameters on 4 ranks: [0,2) [2,5) [5,8) [8,11). */
    uint64_t lo[4], hi[4];
    CHECK(zero_partition_bounds(11, 4, lo, hi) == ZERO_OK);
    const uint64_t want_lo[4] = {0, 2, 5, 8}, want_hi[4] = {2, 5, 8, 11};
    for (int r = 0; r < 4; ++r) CHECK(lo[r] == want_lo[r] && hi[r] == want_hi[r]);
    CHECK(zero_partition_bounds(11, 0, lo, hi) == ZERO_EINVAL);

    /* Per-rank state of 1.5e9 parameters on 4 ranks (16-byte recipe):
     * 24.00, 10.50, 8.25 and 6.00 GB, returned times R. */
    uint64_t out[4];
    CHECK(zero_state_bytes(1500000000ull, 4, 2, 2, 12, out) == ZERO_OK);
    CHECK(out[0] == 4ull * 24000000000ull && out[1] == 4ull * 10500000000ull);
    CHECK(out[2] == 4ull * 8250000000ull && out[3] == 4ull * 6000000000ull);
    /* ZeRO-3 of 1e9 parameters on 4 ranks with 4-byte gradients: 4.5e9 B. */
    CHECK(zero_state_bytes(1000000000ull, 4, 2, 4, 12, out) == ZERO_OK);
    CHECK(out[3] == 4ull * 4500000000ull);
    CHECK(zero_state_bytes(10, 4, 0, 2, 12, out) == ZERO_EINVAL);

    /* ZeRO-3 shards: 10 elements on 4 ranks are shards of 3; rank 3 holds [9, 10). */
    uint64_t s_lo, s_hi, shard;
    CHECK(zero3_shard_bounds(10, 4, 3, &s_lo, &s_hi, &shard) == ZERO_OK);
    CHECK(shard == 3 && s_lo == 9 && s_hi == 10);

    /* Parameter storage: shards of every tensor plus the gathered live one. */
    const uint64_t sizes[2] = {1000, 37};
    const uint32_t live[1] = {0};
    uint64_t st[3];
    CHECK(zero_parameter_storage(sizes, 2, 4, live, 1, st) == ZERO_OK);
    CHECK(st[0] == 250 + 10 && st[1] == 1000 && st[2] == 1260);

    /* Sizes, status text, and calls refused on the host. */
    CHECK(zero_ctrl_bytes() == sizeof(zero_ctrl) && zero_workspace_bytes() == ZERO_WORKSPACE_BYTES);
    CHECK(zero_status_string(ZERO_EINVAL) != NULL && strlen(zero_status_string(ZERO_EINVAL)) > 0);
    CHECK(zero_step_fused(NULL, NULL) == ZERO_EINVAL);
    zero_step_args a;
    memset(&a, 0, sizeof a);
    a.P = 1000;
    a.R = 0;
    CHECK(zero_step_fused(&a, NULL) == ZERO_EINVAL);
    CHECK(zero_scan_nonfinite(NULL, ZERO_F16, 10, NULL, NULL) == ZERO_EINVAL);

    if (failures == 0) printf("abi_host_check: all checks passed\n");
    return failures == 0 ? 0 : 1;
}
