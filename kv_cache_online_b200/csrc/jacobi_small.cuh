// One-sided (Hestenes) Jacobi on the columns of a small matrix held in one CTA's shared memory.
// Used for the SVD of the b x b residual factor R_R of the fold (iS-KV reading notes, Section 4.1:
// "QR + SVD of the small factor"). Written from the published method: Hestenes (1958), with the
// stable rotation of Rutishauser and the convergence test of Demmel and Veselic (1992).
#pragma once

#include "common.cuh"

namespace iskv {

// Rotation angle that makes columns with squared norms alpha, beta and inner product gamma
// orthogonal: returns (c, s) with x' = c x - s y, y' = s x + c y.
ISKV_DEV void jacobi_rotation(double alpha, double beta, double gamma, double &c, double &s) {
  const double zeta = (beta - alpha) / (2.0 * gamma);
  double t;
  if (fabs(zeta) > 1e100) {
    t = 0.5 / zeta;
  } else {
    t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
  }
  c = 1.0 / sqrt(1.0 + t * t);
  s = c * t;
}

// Round-robin ("circle") pairing: n even players, player 0 fixed, the rest rotate by `step`.
ISKV_DEV int circle_player(int i, int step, int n) {
  return i == 0 ? 0 : ((i - 1 + step) % (n - 1)) + 1;
}

// Orthogonalise the `ncols` columns of M (column-major, leading dimension ld, `rows` rows) in
// place. All threads of the CTA must call it. Returns the number of sweeps used, or -1 when the
// sweep cap was reached without convergence. Rotations are skipped when
// |gamma| <= tol * sqrt(alpha * beta).
ISKV_DEV int cta_jacobi_columns(float *M, int rows, int ncols, int ld, double tol, int max_sweeps) {
  __shared__ int rotated;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int ne = ncols + (ncols & 1);
  const int npairs = ne / 2;
  if (ne < 2) return 0;
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    if (threadIdx.x == 0) rotated = 0;
    __syncthreads();
    for (int step = 0; step < ne - 1; ++step) {
      for (int pr = warp; pr < npairs; pr += nwarps) {
        const int a = circle_player(pr, step, ne), b = circle_player(ne - 1 - pr, step, ne);
        if (a >= ncols || b >= ncols) continue;
        float *x = M + (size_t)a * ld, *y = M + (size_t)b * ld;
        double al = 0.0, be = 0.0, ga = 0.0;
        for (int i = lane; i < rows; i += 32) {
          const double xv = x[i], yv = y[i];
          al = fma(xv, xv, al);
          be = fma(yv, yv, be);
          ga = fma(xv, yv, ga);
        }
        al = warp_sum(al);
        be = warp_sum(be);
        ga = warp_sum(ga);
        if (ga != 0.0 && fabs(ga) > tol * sqrt(al * be)) {
          double c, s;
          jacobi_rotation(al, be, ga, c, s);
          const float cf = (float)c, sf = (float)s;
          for (int i = lane; i < rows; i += 32) {
            const float xv = x[i], yv = y[i];
            x[i] = cf * xv - sf * yv;
            y[i] = sf * xv + cf * yv;
          }
          if (lane == 0) rotated = 1;
        }
      }
      __syncthreads();
    }
    if (!rotated) return sweep + 1;
    __syncthreads();
  }
  return -1;
}

}  // namespace iskv
