/* A C caller of the boundary (no Python): host-side entry points only -- window geometry, workspace
 * and saved-state sizes, status strings and argument validation that returns before any launch.
 * Prints one line per check; the test compares them with the header's contract. */
#include <stdint.h>
#include <stdio.h>

#include "vdn.h"

int main(void) {
    int lo = -1, hi = -1;
    /* window of frame 12 of a 31-frame clip, chunk 5, radius 1: chunks 1..3 -> frames 5..19 */
    vdn_status s = vdn_window_bounds(12, 31, 5, 1, &lo, &hi);
    printf("bounds %d %d %d\n", (int)s, lo, hi);
    s = vdn_window_bounds(0, 31, 0, 1, &lo, &hi);
    printf("bounds_bad_chunk %d\n", (int)s);

    vdn_shape sh = {1, 24, 31, 4032, 128, 3, VDN_DTYPE_BF16};
    size_t fwd = vdn_branch_workspace_size(&sh, VDN_RULE_VDN_SOLVE);
    size_t bwd = vdn_branch_backward_workspace_size(&sh, VDN_RULE_VDN_SOLVE);
    size_t sav = vdn_branch_saved_size(&sh);
    size_t soft = vdn_window_softmax_workspace_size(&sh);
    printf("sizes %d %d %d %d\n", fwd > 0 && fwd % 256 == 0, bwd > fwd, sav > 0, (int)soft);

    vdn_shape bad = sh;
    bad.d = 64;
    printf("unsupported %d\n", vdn_branch_workspace_size(&bad, VDN_RULE_VDN_SOLVE) == 0);

    /* a forward call with a NULL q fails validation before touching the device */
    char* base = (char*)(uintptr_t)(1ULL << 40);
    const size_t gap = 1ULL << 34;
    s = vdn_branch_forward(&sh, NULL, base + 1 * gap, base + 2 * gap, (const float*)(base + 3 * gap),
                           (const float*)(base + 4 * gap), base + 5 * gap, (const float*)(base + 6 * gap), NULL, NULL,
                           NULL, VDN_RULE_VDN_SOLVE, 1.0f, 5, 1, base + 7 * gap, fwd, base + 8 * gap, NULL);
    printf("null_q %d %s\n", (int)s, vdn_status_string(s));

    /* frame sharding of the 31-frame clip over 3 ranks in chunks of 5: 7 chunks -> 3, 2, 2 */
    int f0 = -1, f1 = -1, owner = -1;
    printf("frames");
    for (int r = 0; r < 3; ++r) {
        s = vdn_frame_range(31, 3, r, 5, &f0, &f1);
        printf(" %d:%d-%d", (int)s, f0, f1);
    }
    s = vdn_frame_owner(31, 3, 5, 30, &owner);
    printf(" owner %d %d\n", (int)s, owner);
    vdn_shape part = sh;
    part.F = 15;
    size_t maps = vdn_frames_map_bytes(&part, 31, 3, 0, 5);
    /* maps [B*H][2][nch][2][d][d] fp32, then one int32 exponent per map, padded to 16 bytes */
    size_t expect = (size_t)24 * 2 * 3 * 2 * 128 * 128 * 4 + (size_t)24 * 2 * 3 * 2 * 4;
    expect = (expect + 15) / 16 * 16;
    printf("map_bytes %d\n", maps == expect);
    return 0;
}
