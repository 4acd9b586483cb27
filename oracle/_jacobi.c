/*
 * One-sided (Hestenes) Jacobi SVD in float64 -- part of the CPU oracle
 * (test infrastructure only).
 *
 * The SVDQuant pages split the smoothed weight by its singular value
 * decomposition W = U S V^T and keep the k largest singular triplets
 * ("AI图像生成4-bit量化技术解析与应用", 2.2; "SVDQuant是什么？", 技术原理).  This
 * file computes that decomposition the plain way: columns of A are rotated in
 * pairs until every pair is orthogonal to working precision; then the column
 * norms are the singular values, the normalised columns are U and the
 * accumulated rotations are V.
 *
 * A is m x n, column-major (column j at A + j*m), n <= m.  On return A holds
 * U*S (unsorted), V (n x n, column-major) the accumulated rotations.
 * Convergence: every pair satisfies |a_p . a_q| <= tol * ||a_p|| ||a_q||.
 * Returns the number of sweeps used, or -1 if max_sweeps was reached first.
 */
#include <math.h>
#include <stddef.h>

static double dot(const double* x, const double* y, int m) {
    double s = 0.0;
    for (int i = 0; i < m; ++i) s += x[i] * y[i];
    return s;
}

int oracle_jacobi_svd(int m, int n, double* A, double* V, double tol, int max_sweeps) {
    for (int j = 0; j < n; ++j)
        for (int i = 0; i < n; ++i) V[(size_t)j * n + i] = (i == j) ? 1.0 : 0.0;

    for (int sweep = 1; sweep <= max_sweeps; ++sweep) {
        int rotated = 0;
        for (int p = 0; p < n - 1; ++p) {
            for (int q = p + 1; q < n; ++q) {
                double* ap = A + (size_t)p * m;
                double* aq = A + (size_t)q * m;
                double alpha = dot(ap, ap, m);
                double beta = dot(aq, aq, m);
                double gamma = dot(ap, aq, m);
                if (gamma == 0.0 || fabs(gamma) <= tol * sqrt(alpha * beta)) continue;
                rotated = 1;
                /* rotation that makes the pair orthogonal (smaller angle root) */
                double zeta = (beta - alpha) / (2.0 * gamma);
                double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                double c = 1.0 / sqrt(1.0 + t * t);
                double s = c * t;
                for (int i = 0; i < m; ++i) {
                    double x = ap[i], y = aq[i];
                    ap[i] = c * x - s * y;
                    aq[i] = s * x + c * y;
                }
                double* vp = V + (size_t)p * n;
                double* vq = V + (size_t)q * n;
                for (int i = 0; i < n; ++i) {
                    double x = vp[i], y = vq[i];
                    vp[i] = c * x - s * y;
                    vq[i] = s * x + c * y;
                }
            }
        }
        if (!rotated) return sweep;
    }
    return -1;
}
