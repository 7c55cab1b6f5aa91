/* Test driver: runs the fp64 oracle (oracle/gdn_oracle.c, compiled into the same
 * executable with AddressSanitizer and UndefinedBehaviorSanitizer) over small
 * problems that reach every branch of it -- one gate per head and per key
 * channel, packed sequences including an empty one, a given and a zero initial
 * state, snapshots, the additive test mode, several threads -- and over bad
 * arguments.  Exit status 0 when every call behaved; the sanitizers abort on
 * the first memory or undefined-behaviour error. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

int oracle_gdn_forward(int64_t n_seqs, const int64_t *seq_start, const int64_t *seq_len, int64_t H, int64_t dk,
                       int64_t dv, const double *q, const double *k, const double *v, const double *g,
                       const double *beta, const double *h0, int per_channel, int additive, double scale,
                       int64_t snapshot_stride, int64_t n_snap_max, double *out, double *final_state,
                       double *snapshots, int n_threads);

static double urand(uint64_t *s) {
    *s = *s * 6364136223846793005ULL + 1442695040888963407ULL;
    return (double)(*s >> 11) / 9007199254740992.0;
}

static double *filled(size_t n, uint64_t *s, double lo, double hi) {
    double *a = (double *)malloc(sizeof(double) * (n ? n : 1));
    for (size_t i = 0; i < n; ++i) a[i] = lo + (hi - lo) * urand(s);
    return a;
}

int main(void) {
    const int64_t lens[3] = {5, 0, 70}, starts[3] = {0, 5, 5};
    const int64_t N = 3, T = 75, H = 2, dk = 8, dv = 6, stride = 16, n_snap = 70 / 16;
    uint64_t s = 12345;
    int failures = 0;
    for (int per_channel = 0; per_channel < 2; ++per_channel) {
        for (int variant = 0; variant < 3; ++variant) {
            double *q = filled((size_t)(T * H * dk), &s, -1, 1), *k = filled((size_t)(T * H * dk), &s, -1, 1);
            double *v = filled((size_t)(T * H * dv), &s, -1, 1);
            double *g = filled((size_t)(T * H * (per_channel ? dk : 1)), &s, -2, 0);
            double *beta = filled((size_t)(T * H), &s, 0, 1);
            double *h0 = variant == 1 ? NULL : filled((size_t)(N * H * dv * dk), &s, -0.1, 0.1);
            double *out = filled((size_t)(T * H * dv), &s, 0, 0);
            double *fin = filled((size_t)(N * H * dv * dk), &s, 0, 0);
            double *snaps = filled((size_t)(N * n_snap * H * dv * dk), &s, 0, 0);
            const int rc = oracle_gdn_forward(N, starts, lens, H, dk, dv, q, k, v, g, beta, h0, per_channel,
                                              variant == 2, 0.5, stride, n_snap, out, fin, snaps, 1 + variant);
            if (rc != 0) ++failures;
            for (int64_t i = 0; i < T * H * dv; ++i)
                if (!isfinite(out[i])) ++failures;
            free(q); free(k); free(v); free(g); free(beta); free(h0); free(out); free(fin); free(snaps);
        }
    }
    /* bad arguments are refused */
    double x = 0.0;
    if (oracle_gdn_forward(-1, starts, lens, H, dk, dv, &x, &x, &x, &x, &x, NULL, 0, 0, 1.0, 0, 0, &x, NULL, NULL, 1) !=
        -1)
        ++failures;
    if (oracle_gdn_forward(N, starts, lens, H, dk, dv, NULL, &x, &x, &x, &x, NULL, 0, 0, 1.0, 0, 0, &x, NULL, NULL, 1) !=
        -1)
        ++failures;
    printf("oracle sanitize run: %d failures\n", failures);
    return failures != 0;
}
