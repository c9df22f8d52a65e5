/* A plain C consumer of librlscan: includes rlscan.h, links the shared
 * library and calls the host-only entry points (no GPU needed): the version,
 * the launch plan and workspace size of a few shapes, and argument checks
 * that fail before any CUDA call. */
#include <stdio.h>
#include "rlscan.h"

int main(void) {
    printf("version %d\n", rlscan_version());
    const int64_t shapes[][2] = {{4096, 128}, {16, 262144}, {3, 70000}};
    for (int i = 0; i < 3; ++i) {
        int64_t tile = 0, ntiles = 0;
        int threads = 0, lookback = 0;
        int rc = rlscan_plan(shapes[i][0], shapes[i][1], 1, &tile, &threads, &lookback, &ntiles);
        printf("plan %lld %lld rc=%d tile=%lld threads=%d lookback=%d ntiles=%lld ws=%zu\n",
               (long long)shapes[i][0], (long long)shapes[i][1], rc, (long long)tile, threads, lookback,
               (long long)ntiles, rlscan_workspace_bytes(shapes[i][0], shapes[i][1]));
    }
    /* NULL rewards: rejected on the host */
    int rc = rlscan_gae(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 4, 128, 0.99f, 0.95f, NULL, 0, NULL);
    printf("null rc=%d msg=%s\n", rc, rlscan_last_error());
    /* an empty batch is a no-op */
    printf("batch rc=%d\n", rlscan_batch(NULL, 0, NULL, 0, NULL));
    return 0;
}
