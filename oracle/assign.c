/*
 * PARK oracle: the K-means assign step in plain C, float64.
 *
 * TEST INFRASTRUCTURE ONLY (see park_oracle.py): it is the oracle's own code,
 * shares nothing with the CUDA library, and only tests, the smoke check and
 * the benchmark's CPU baseline call it.
 *
 * Definition (PARK, Figure 2 caption: the keys are clustered with K-means after
 * a query-derived transform; the queries with plain K-means): every row x_i is
 * assigned to argmin_k sum_j (x_ij - c_kj)^2, ties to the lowest k.  Rows and
 * centroids arrive already transformed (for the key side, multiplied by F with
 * M = F F^T), so this is the Euclidean distance.  The sum runs over j in
 * ascending order with one rounding per operation (build with
 * -ffp-contract=off and without fast-math, so no FMA or reassociation).  Rows
 * are split over OpenMP threads; the result does not depend on the thread
 * count.
 */
#include <stdint.h>

void oracle_assign(const double *X, const double *C, int64_t N, int64_t K, int64_t D, int64_t *labels) {
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < N; ++i) {
        const double *x = X + i * D;
        double best = 0.0;
        int64_t arg = -1;
        /* four centroids at a time (four independent sums, each in j order) */
        int64_t k = 0;
        for (; k + 4 <= K; k += 4) {
            const double *c0 = C + k * D, *c1 = c0 + D, *c2 = c1 + D, *c3 = c2 + D;
            double s[4] = {0.0, 0.0, 0.0, 0.0};
            for (int64_t j = 0; j < D; ++j) {
                const double d0 = x[j] - c0[j], d1 = x[j] - c1[j], d2 = x[j] - c2[j], d3 = x[j] - c3[j];
                s[0] = s[0] + d0 * d0;
                s[1] = s[1] + d1 * d1;
                s[2] = s[2] + d2 * d2;
                s[3] = s[3] + d3 * d3;
            }
            for (int u = 0; u < 4; ++u)
                if (arg < 0 || s[u] < best) { /* strict: the first of equal distances stays */
                    best = s[u];
                    arg = k + u;
                }
        }
        for (; k < K; ++k) {
            const double *c = C + k * D;
            double s = 0.0;
            for (int64_t j = 0; j < D; ++j) {
                const double d = x[j] - c[j];
                s = s + d * d;
            }
            if (arg < 0 || s < best) {
                best = s;
                arg = k;
            }
        }
        labels[i] = arg;
    }
}
