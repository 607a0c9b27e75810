/*
 * Scalar float64 brute force of Re-ttention's calibration and reshaped sparse
 * step, written independently of oracle/reference.py (plain loops, token-level
 * keep mask, no blocks) so that it can pin that module on tiny inputs.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests through oracle/brute.py; nothing on
 * the product path links or calls it.
 *
 * Definitions (Re-ttention OpenReview discussion, replies to W1 of the first
 * and third reviewers, Q2 and Q4): for query i of one head,
 *   s_ij = scale * sum_t q[i][t] k[j][t]
 *   Z_full = sum_j e^{s_ij - m},  Z_sp = sum_{j kept} e^{s_ij - m},  m = max_j s_ij
 *   rho_i = Z_sp / Z_full
 *   R_i   = sum_{j not kept} e^{s_ij - m} v_j / Z_full
 *   O_i   = sum_j e^{s_ij - m} v_j / Z_full
 * and the sparse step with a given rho_hat:
 *   O'_i = rho_hat_i * sum_{j kept} e^{s'_ij - m'} v'_j / sum_{j kept} e^{s'_ij - m'} + R_i
 *   (O'_i = R_i when row i keeps no key).
 * keep is row-major [L][L]: keep[i*L + j] != 0 iff key j is in query i's window.
 */
#include <math.h>
#include <stddef.h>

static double dot(const double* a, const double* b, int d) {
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += a[t] * b[t];
    return acc;
}

int brute_calibrate(int L, int d, const double* q, const double* k, const double* v,
                    const unsigned char* keep, double scale,
                    double* o, double* rho, double* r) {
    if (L <= 0 || d <= 0) return 1;
    for (int i = 0; i < L; ++i) {
        double m = -INFINITY;
        for (int j = 0; j < L; ++j) {
            double s = scale * dot(q + (size_t)i * d, k + (size_t)j * d, d);
            if (s > m) m = s;
        }
        double z_full = 0.0, z_sp = 0.0;
        for (int t = 0; t < d; ++t) { o[(size_t)i * d + t] = 0.0; r[(size_t)i * d + t] = 0.0; }
        for (int j = 0; j < L; ++j) {
            double e = exp(scale * dot(q + (size_t)i * d, k + (size_t)j * d, d) - m);
            int kept = keep[(size_t)i * L + j] != 0;
            z_full += e;
            if (kept) z_sp += e;
            for (int t = 0; t < d; ++t) {
                o[(size_t)i * d + t] += e * v[(size_t)j * d + t];
                if (!kept) r[(size_t)i * d + t] += e * v[(size_t)j * d + t];
            }
        }
        for (int t = 0; t < d; ++t) { o[(size_t)i * d + t] /= z_full; r[(size_t)i * d + t] /= z_full; }
        rho[i] = z_sp / z_full;
    }
    return 0;
}

int brute_sparse_step(int L, int d, const double* q, const double* k, const double* v,
                      const unsigned char* keep, double scale, const double* rho_hat,
                      const double* r, double* o) {
    if (L <= 0 || d <= 0) return 1;
    for (int i = 0; i < L; ++i) {
        double m = -INFINITY;
        int any = 0;
        for (int j = 0; j < L; ++j) {
            if (!keep[(size_t)i * L + j]) continue;
            double s = scale * dot(q + (size_t)i * d, k + (size_t)j * d, d);
            if (!any || s > m) m = s;
            any = 1;
        }
        for (int t = 0; t < d; ++t) o[(size_t)i * d + t] = r[(size_t)i * d + t];
        if (!any) continue;
        double z = 0.0;
        double acc[512];
        if (d > 512) return 2;
        for (int t = 0; t < d; ++t) acc[t] = 0.0;
        for (int j = 0; j < L; ++j) {
            if (!keep[(size_t)i * L + j]) continue;
            double e = exp(scale * dot(q + (size_t)i * d, k + (size_t)j * d, d) - m);
            z += e;
            for (int t = 0; t < d; ++t) acc[t] += e * v[(size_t)j * d + t];
        }
        for (int t = 0; t < d; ++t) o[(size_t)i * d + t] += rho_hat[i] * acc[t] / z;
    }
    return 0;
}
