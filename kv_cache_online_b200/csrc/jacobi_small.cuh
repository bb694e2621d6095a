// One-sided (Hestenes) Jacobi on the columns of a small matrix held in one CTA's shared memory.
// Used for the SVD of the b x b residual factor R_R of the fold (iS-KV reading notes, Section 4.1:
// "QR + SVD of the small factor"). Written from the published method: Hestenes (1958), with the
// rotation angle of Rutishauser and the convergence test of Demmel and Veselic (1992).
#pragma once

#include "common.cuh"

namespace iskv {

// Round-robin ("circle") pairing: n even players, player 0 fixed, the rest rotate by `step`.
// Requires 0 <= i < n and 0 <= step < n - 1 (so one conditional subtraction reduces mod n - 1).
ISKV_DEV int circle_player(int i, int step, int n) {
  if (i == 0) return 0;
  int v = i - 1 + step;
  if (v >= n - 1) v -= n - 1;
  return v + 1;
}

// Rotation of the column pair (x, y) held as RQ entries per lane of a half-warp, given the
// reduced squared norms al, be and inner product ga; writes the rotated columns back. Rutishauser's
// angle; tau = tan(theta / 2) and sn = 2 tau / (1 + tau^2) keep the rotation orthogonal to
// rounding, so fast reciprocals suffice for the parameters. Returns whether it rotated.
template <int RQ>
ISKV_DEV bool small_rotate(float *x, float *y, const float (&xv)[RQ], const float (&yv)[RQ],
                           int rows, float al, float be, float ga, float tol) {
  if (!(ga != 0.f && ga * ga > (tol * tol * al) * be)) return false;
  const int l16 = threadIdx.x & 15;
  const float zeta = 0.5f * (be - al) * __fdividef(1.f, ga);
  const float az = fabsf(zeta);
  float t;
  if (az > 1e18f) {
    t = __fdividef(0.5f, zeta);
  } else {
    const float q = fmaf(zeta, zeta, 1.f);
    t = copysignf(__fdividef(1.f, az + q * rsqrtf(q)), zeta);
  }
  const float q2 = fmaf(t, t, 1.f);
  const float tau = __fdividef(t, 1.f + q2 * rsqrtf(q2));
  const float sn = __fdividef(2.f * tau, fmaf(tau, tau, 1.f));
#pragma unroll
  for (int q = 0; q < RQ; ++q) {
    const int i = l16 + 16 * q;
    if (i < rows) {
      x[i] = fmaf(-sn, fmaf(tau, xv[q], yv[q]), xv[q]);
      y[i] = fmaf(sn, fmaf(-tau, yv[q], xv[q]), yv[q]);
    }
  }
  return true;
}

// Orthogonalise the `ncols` columns of M (column-major, leading dimension ld, `rows` <= 16 RQ rows)
// in place, in float32. All threads of the CTA must call it (blockDim a multiple of 32). Each
// half-warp rotates column pairs (16 lanes x RQ rows each), two independent pairs per pass so
// their reductions and parameter chains overlap; a 256-thread CTA covers 32 pairs of a round in
// one pass. Rotations use the half-angle form
//   x' = x - s (y + tau x),  y' = y + s (x - tau y),  tau = t / (1 + sqrt(1 + t^2)),
// which stays orthogonal when c = 1 / sqrt(1 + t^2) rounds to 1. A pair is skipped when
// gamma^2 <= tol^2 alpha beta. Returns the sweeps used, or -1 when the cap was reached.
template <int RQ>
ISKV_DEV int cta_jacobi_columns(float *M, int rows, int ncols, int ld, float tol, int max_sweeps) {
  __shared__ int rotated;
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int half = (threadIdx.x >> 4) & 1, l16 = threadIdx.x & 15;
  const int ne = ncols + (ncols & 1);
  const int npairs = ne / 2;
  const int stride = 2 * nwarps;  // half-warps
  if (ne < 2) return 0;
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    if (threadIdx.x == 0) rotated = 0;
    __syncthreads();
    for (int step = 0; step < ne - 1; ++step) {
      // Both half-warps of a warp run the same number of passes (they shuffle together).
      for (int base = 2 * warp; base < npairs; base += 2 * stride) {
        int pa[2], pb[2];
        bool live[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int pr = base + half + u * stride;
          pa[u] = 0;
          pb[u] = 0;
          live[u] = pr < npairs;
          if (live[u]) {
            pa[u] = circle_player(pr, step, ne);
            pb[u] = circle_player(ne - 1 - pr, step, ne);
            live[u] = pa[u] < ncols && pb[u] < ncols;
          }
        }
        float xv[2][RQ], yv[2][RQ], al[2], be[2], ga[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float *x = M + (size_t)pa[u] * ld, *y = M + (size_t)pb[u] * ld;
          al[u] = 0.f;
          be[u] = 0.f;
          ga[u] = 0.f;
#pragma unroll
          for (int q = 0; q < RQ; ++q) {
            const int i = l16 + 16 * q;
            const bool in = live[u] && i < rows;
            xv[u][q] = in ? x[i] : 0.f;
            yv[u][q] = in ? y[i] : 0.f;
            al[u] = fmaf(xv[u][q], xv[u][q], al[u]);
            be[u] = fmaf(yv[u][q], yv[u][q], be[u]);
            ga[u] = fmaf(xv[u][q], yv[u][q], ga[u]);
          }
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            al[u] += __shfl_xor_sync(0xffffffffu, al[u], o);
            be[u] += __shfl_xor_sync(0xffffffffu, be[u], o);
            ga[u] += __shfl_xor_sync(0xffffffffu, ga[u], o);
          }
        }
        bool any = false;
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (live[u])
            any |= small_rotate<RQ>(M + (size_t)pa[u] * ld, M + (size_t)pb[u] * ld, xv[u], yv[u],
                                    rows, al[u], be[u], ga[u], tol);
        if (any && l16 == 0) rotated = 1;
      }
      __syncthreads();
    }
    if (!rotated) return sweep + 1;
    __syncthreads();
  }
  return -1;
}

}  // namespace iskv
