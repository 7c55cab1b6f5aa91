/* Test driver: the host code of the C-ABI library (libgdn's validation, workspace
 * planning, split choice, error strings and event timer), built with
 * AddressSanitizer and UndefinedBehaviorSanitizer, driven through its entry points
 * with arguments that it must refuse before anything reaches the device, and
 * with sizes that it must plan.  No GPU is needed: every call here returns before
 * a kernel launch.  Exit status 0 when every call returned what it should; the
 * sanitizers abort on the first memory or undefined-behaviour error. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "gdn.h"

static int failures = 0;
#define EXPECT(call, want)                                                                    \
    do {                                                                                      \
        const gdn_status got_ = (call);                                                       \
        if (got_ != (want)) {                                                                 \
            ++failures;                                                                       \
            printf("line %d: %s -> %d, want %d (%s)\n", __LINE__, #call, (int)got_, (int)(want), \
                   gdn_last_error());                                                         \
        }                                                                                     \
    } while (0)

static gdn_desc desc(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int dtype, int gate) {
    gdn_desc d;
    memset(&d, 0, sizeof d);
    d.B = B; d.T = T; d.H = H; d.dk = dk; d.dv = dv; d.dtype = dtype; d.gate = gate; d.scale = 1.0f; d.hk = 0;
    return d;
}

#define P(i) ((void *)(uintptr_t)((1ULL << 40) + (uint64_t)(i) * (1ULL << 32)))
#define F(i) ((float *)P(i))

int main(void) {
    size_t n = 0;
    /* workspace planning over many shapes (packed bound, split scan, both paths) */
    const int64_t Ts[] = {0, 1, 63, 64, 65, 4096, 262144, 1 << 20};
    for (int dt = 0; dt < 2; ++dt)
        for (int gate = 0; gate < 2; ++gate)
            for (int i = 0; i < 8; ++i)
                for (int64_t B = 1; B <= 64; B *= 4) {
                    gdn_desc d = desc(B, Ts[i], 16, 128, 128, dt, gate);
                    EXPECT(gdn_chunk_workspace_size(&d, (int32_t)B, &n), GDN_OK);
                    EXPECT(gdn_chunk_workspace_size(&d, 1000, &n), GDN_OK);
                }
    gdn_desc d = desc(2, 130, 3, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    EXPECT(gdn_chunk_workspace_size(&d, 2, NULL), GDN_ERR_INVALID_ARG);
    EXPECT(gdn_chunk_workspace_size(NULL, 2, &n), GDN_ERR_INVALID_ARG);
    EXPECT(gdn_chunk_workspace_size(&d, -1, &n), GDN_ERR_INVALID_ARG);
    gdn_desc bad = d; bad.dk = 96;
    EXPECT(gdn_chunk_workspace_size(&bad, 2, &n), GDN_ERR_UNSUPPORTED);
    bad = d; bad.hk = 2;
    EXPECT(gdn_chunk_workspace_size(&bad, 2, &n), GDN_ERR_INVALID_ARG);
    bad = d; bad.B = 1LL << 40; bad.T = 1LL << 20;
    EXPECT(gdn_chunk_workspace_size(&bad, 2, &n), GDN_ERR_INVALID_ARG);

    /* gdn_chunk_fwd: every refusal happens before a launch */
    const size_t big = (size_t)1 << 40;
    EXPECT(gdn_chunk_fwd(NULL, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(5), NULL, NULL, P(7), big, NULL),
           GDN_ERR_INVALID_ARG);
    EXPECT(gdn_chunk_fwd(&d, NULL, P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(5), NULL, NULL, P(7), big, NULL),
           GDN_ERR_INVALID_ARG);
    EXPECT(gdn_chunk_fwd(&d, (char *)P(0) + 8, P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(5), NULL, NULL, P(7), big,
                         NULL),
           GDN_ERR_INVALID_ARG);
    EXPECT(gdn_chunk_fwd(&d, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(0), NULL, NULL, P(7), big, NULL),
           GDN_ERR_INVALID_ARG); /* out overlaps q */
    EXPECT(gdn_chunk_fwd(&d, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(5), NULL, NULL, NULL, big, NULL),
           GDN_ERR_WORKSPACE);
    EXPECT(gdn_chunk_fwd(&d, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(5), NULL, NULL, P(7), 16, NULL),
           GDN_ERR_WORKSPACE);
    EXPECT(gdn_chunk_fwd(&d, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(5), NULL, NULL, (char *)P(7) + 64,
                         big, NULL),
           GDN_ERR_WORKSPACE);
    EXPECT(gdn_chunk_fwd(&d, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 100, P(5), NULL, F(6), P(7), big, NULL),
           GDN_ERR_INVALID_ARG); /* stride not a multiple of 64 */
    EXPECT(gdn_chunk_fwd(&d, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 64, P(5), NULL, NULL, P(7), big, NULL),
           GDN_ERR_INVALID_ARG); /* snapshots missing */
    gdn_desc packed = desc(1, 300, 3, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    EXPECT(gdn_chunk_fwd(&packed, P(0), P(1), P(2), F(3), F(4), NULL, (int32_t *)P(8), 3, 64, P(5), NULL, F(6), P(7),
                         big, NULL),
           GDN_ERR_UNSUPPORTED); /* snapshots with packed sequences */
    gdn_desc empty = desc(0, 100, 3, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    EXPECT(gdn_chunk_fwd(&empty, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 0, 0, P(5), NULL, NULL, P(7), big, NULL),
           GDN_OK); /* no sequences: nothing to do */
    int32_t code = 0;
    EXPECT(gdn_chunk_status(NULL, NULL, &code), GDN_ERR_INVALID_ARG);
    EXPECT(gdn_chunk_status(P(7), NULL, NULL), GDN_ERR_INVALID_ARG);
    gdn_desc huge = desc(4, 40000, 16, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    EXPECT(gdn_chunk_fwd_static(&huge, P(0), P(1), P(2), F(3), F(4), NULL, NULL, 4, 0, P(5), F(6), NULL, NULL),
           GDN_ERR_WORKSPACE);

    /* decode, multi-token decode, state select, pre-rule work */
    gdn_desc dd = desc(4, 1, 2, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    EXPECT(gdn_decode_step(&dd, P(0), P(1), P(2), F(3), F(4), NULL, P(5), NULL), GDN_ERR_INVALID_ARG);
    EXPECT(gdn_decode_step(&dd, P(0), P(1), P(2), F(3), F(4), F(5), P(5), NULL), GDN_ERR_INVALID_ARG);
    gdn_desc dt2 = dd; dt2.T = 2;
    EXPECT(gdn_decode_step(&dt2, P(0), P(1), P(2), F(3), F(4), F(6), P(5), NULL), GDN_ERR_INVALID_ARG);
    gdn_desc dm = desc(4, 65, 2, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    EXPECT(gdn_decode_multi(&dm, P(0), P(1), P(2), F(3), F(4), NULL, F(6), 1, P(5), NULL, NULL), GDN_ERR_INVALID_ARG);
    dm.T = 4;
    EXPECT(gdn_decode_multi(&dm, P(0), P(1), P(2), F(3), F(4), NULL, F(6), 2, P(5), NULL, NULL), GDN_ERR_INVALID_ARG);
    EXPECT(gdn_state_select(&dm, NULL, (int32_t *)P(1), F(2), NULL), GDN_ERR_INVALID_ARG);
    EXPECT(gdn_state_select(&dm, F(1), (int32_t *)P(1), F(1), NULL), GDN_ERR_INVALID_ARG);
    gdn_desc dp = desc(1, 100, 4, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    dp.hk = 2;
    EXPECT(gdn_prerule(&dp, P(0), P(1), P(2), F(3), 5, F(4), F(5), NULL, 0, NULL, NULL, P(6), P(7), P(8), F(9), F(10),
                       NULL),
           GDN_ERR_UNSUPPORTED); /* convolution width 5 */
    EXPECT(gdn_prerule(&dp, P(0), P(1), P(2), F(3), 4, F(4), F(5), NULL, 0, NULL, NULL, P(0), P(7), P(8), F(9), F(10),
                       NULL),
           GDN_ERR_INVALID_ARG); /* q overlaps x */
    gdn_desc dpc = dp; dpc.gate = GDN_GATE_CHANNEL;
    EXPECT(gdn_prerule(&dpc, P(0), P(1), P(2), F(3), 4, F(4), F(5), NULL, 0, NULL, NULL, P(6), P(7), P(8), F(9),
                       F(10), NULL),
           GDN_ERR_UNSUPPORTED);
    gdn_desc dpd = desc(3, 1, 4, 128, 128, GDN_BF16, GDN_GATE_HEAD);
    EXPECT(gdn_decode_step_prerule(&dpd, P(0), P(1), P(2), F(3), 0, F(4), F(5), NULL, F(6), P(7), NULL),
           GDN_ERR_UNSUPPORTED);

    /* strings, last error, event timer without launches */
    for (int s = 0; s <= 7; ++s)
        if (!gdn_status_string((gdn_status)s) || !gdn_status_string((gdn_status)s)[0]) ++failures;
    if (!gdn_last_error()) ++failures;
    EXPECT(gdn_profile_enable(1), GDN_OK);
    gdn_kernel_time t[4];
    int32_t cnt = -1;
    EXPECT(gdn_profile_read(t, 4, &cnt), GDN_OK);
    if (cnt != 0) ++failures;
    EXPECT(gdn_profile_read(NULL, 4, &cnt), GDN_ERR_INVALID_ARG);
    EXPECT(gdn_profile_enable(0), GDN_OK);

    printf("library host sanitize run: %d failures\n", failures);
    return failures != 0;
}
