// Fold step 4 (iS-KV reading notes, Section 4.1 and Algorithm 2 step 4): reduced Householder QR
// of the residual E^T (d x b), SVD of the b x b factor R_R, the residual threshold, the kept
// residual basis P = Q_R W_R[:, :p], and the core block F P (Algorithm 2 step 5).
//
// One thread-block cluster per fold. CTA c of the cluster holds rows [c d/CQ, (c+1) d/CQ) of E^T in
// shared memory. Each reflector needs one cluster-wide reduction: every CTA publishes, for the
// current column j, its partial dot products of column j with every column and (if it owns row j)
// row j itself; after one cluster barrier every CTA sums the CQ payloads in rank order, so all CTAs
// hold bit-identical reflector data. The reflectors are accumulated in compact WY form
// (Q = I - V T V^T, Schreiber and Van Loan 1989), so P is formed with one more exchange instead of b
// sequential reflector applications.
#include <cooperative_groups.h>

#include "jacobi_small.cuh"
#include "kernels.h"
#include "profiling.h"

namespace cg = cooperative_groups;

namespace iskv {

constexpr int RES_NTH = 256;

struct ResidualSmem {
  int rpc, b;
  size_t a, rm, fpp, pay, tot, part, vdiag, alph, tauv, total;
};

__host__ __device__ inline ResidualSmem residual_smem(int d, int b, int cq) {
  ResidualSmem s;
  s.rpc = d / cq;
  s.b = b;
  size_t o = 0;
  auto take = [&](size_t n) { size_t at = o; o += n; return at; };  // counts in 4-byte words
  s.a = take((size_t)s.rpc * b);
  s.rm = take((size_t)b * b);
  s.fpp = take((size_t)b * b);
  s.pay = take((size_t)2 * 2 * b);
  s.tot = take((size_t)2 * b);
  s.part = take((size_t)2 * RES_NTH);  // doubles
  s.vdiag = take(b);
  s.alph = take(b);
  s.tauv = take(b);
  s.total = o * 4;
  return s;
}

// Smallest power-of-two cluster whose per-CTA row slice holds at most 64 KiB of E^T, subject to
// every CTA holding at least b rows (rank 0 must own all b rows of R_R). Returns -1 if none.
static int residual_cluster_size(int d, int b) {
  int best = -1;
  for (int cq = 1; cq <= 8; cq *= 2) {
    if (d % cq) break;
    const int rpc = d / cq;
    if (rpc < b) break;
    best = cq;
    if ((size_t)rpc * b * 4 <= 64 * 1024) return cq;
  }
  return best;
}

template <typename TF>
__global__ void __launch_bounds__(RES_NTH) k_fold_residual(const FoldJob *jobs, FoldParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int cq = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const FoldJob &jb = jobs[blockIdx.x / cq];
  int32_t *sc = reinterpret_cast<int32_t *>(jb.h.ws + p.ws.scal);
  if (sc[FS_SKIP]) return;  // uniform over the cluster

  const int d = p.d, b = p.b, k = sc[FS_K_OLD];
  const ResidualSmem L = residual_smem(d, b, cq);
  const int rpc = L.rpc, row0 = rank * rpc;
  extern __shared__ float smem[];
  float *A = smem + L.a;          // [rpc][b] rows of E^T, then reflectors / R
  float *Rm = smem + L.rm;        // [b][b] column-major R_R (rank 0)
  float *fpp = smem + L.fpp;      // [b][b] partial F P
  float *pay = smem + L.pay;      // [2][2b] reduction payload
  float *tot = smem + L.tot;      // [2b] reduced payload
  double *part = reinterpret_cast<double *>(smem + L.part);
  float *vdiag = smem + L.vdiag, *alph = smem + L.alph, *tauv = smem + L.tauv;
  const int tid = threadIdx.x;
  const float *E = reinterpret_cast<const float *>(jb.h.ws + p.ws.E);
  // Compact-WY factor T (b x b, rank 0): kept in the F P partial buffer, which is idle until
  // the end; each thread of rank 0 builds and re-reads only its own row.
  float *T = fpp;
  float *W = reinterpret_cast<float *>(jb.h.ws + p.ws.W);
  float *Y2 = reinterpret_cast<float *>(jb.h.ws + p.ws.Y2);
  float *P = reinterpret_cast<float *>(jb.h.ws + p.ws.P);
  float *FP = reinterpret_cast<float *>(jb.h.ws + p.ws.FP);
  float *rho_out = reinterpret_cast<float *>(jb.h.ws + p.ws.rho);

  // Load my rows of E^T: A[i][c] = E[c][row0 + i].
  for (int e = tid; e < rpc * b; e += RES_NTH) {
    const int c = e / rpc, i = e % rpc;
    A[i * b + c] = E[(size_t)c * d + row0 + i];
  }
  __syncthreads();

  const int G = RES_NTH / b;        // row groups in the dot / update phases
  const int my_c = tid % b, my_g = tid / b;
  const bool active = my_g < G;

  for (int j = 0; j < b; ++j) {
    // Partial dots of column j with every column over my rows with global index >= j: four
    // independent float32 accumulators (short dependency chains), combined in float64.
    if (active) {
      int i = my_g;
      if (row0 + i < j) i += ((j - row0 - i) + G - 1) / G * G;  // first of my rows at or past j
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (; i + 3 * G < rpc; i += 4 * G) {
        a0 = fmaf(A[i * b + j], A[i * b + my_c], a0);
        a1 = fmaf(A[(i + G) * b + j], A[(i + G) * b + my_c], a1);
        a2 = fmaf(A[(i + 2 * G) * b + j], A[(i + 2 * G) * b + my_c], a2);
        a3 = fmaf(A[(i + 3 * G) * b + j], A[(i + 3 * G) * b + my_c], a3);
      }
      for (; i < rpc; i += G) a0 = fmaf(A[i * b + j], A[i * b + my_c], a0);
      part[my_g * b + my_c] = ((double)a0 + (double)a1) + ((double)a2 + (double)a3);
    }
    __syncthreads();
    float *slot = pay + (j & 1) * 2 * b;
    if (tid < b) {
      double s = 0.0;
      for (int g = 0; g < G; ++g) s += part[g * b + tid];
      slot[tid] = (float)s;
      const int jl = j - row0;
      slot[b + tid] = (jl >= 0 && jl < rpc) ? A[jl * b + tid] : 0.f;
    }
    cluster.sync();
    if (tid < 2 * b) {
      float s = 0.f;
      for (int q = 0; q < cq; ++q) {
        const float *rs = cluster.map_shared_rank(slot, q);
        s += rs[tid];
      }
      tot[tid] = s;
    }
    __syncthreads();
    // Reflector for column j (identical on every CTA).
    const double norm2 = tot[j], xj = tot[b + j];
    const double norm = sqrt(norm2);
    double alpha = 0.0, vj = 0.0, tau = 0.0;
    if (norm > 0.0) {
      alpha = xj >= 0.0 ? -norm : norm;
      vj = xj - alpha;
      const double vtv = vj * vj + fmax(norm2 - xj * xj, 0.0);
      tau = vtv > 0.0 ? 2.0 / vtv : 0.0;
    }
    if (tid == 0) {
      vdiag[j] = (float)vj;
      alph[j] = (float)alpha;
      tauv[j] = (float)tau;
    }
    // WY factor column j (rank 0 only): T[j][j] = tau, T[i][j] = -tau sum_l T[i][l] w_l.
    if (rank == 0 && tid <= j) {
      if (tid == j) {
        T[j * b + j] = (float)tau;
      } else {
        double s = 0.0;
        for (int l = tid; l < j; ++l) s += (double)T[tid * b + l] * ((double)tot[l] - alpha * tot[b + l]);
        T[tid * b + j] = (float)(-tau * s);
      }
    }
    // Apply H_j to the trailing columns: A[i][c] -= tau v_i w_c, w_c = x^T A_c - alpha A[j][c].
    if (active && my_c > j && tau != 0.0) {
      const double wc = (double)tot[my_c] - alpha * tot[b + my_c];
      const float tw = (float)(tau * wc);
      int i = my_g;
      if (row0 + i < j) i += ((j - row0 - i) + G - 1) / G * G;  // first of my rows at or past j
      if (i < rpc && row0 + i == j) {  // the reflector's leading entry is vj, not A[j][j]
        A[i * b + my_c] -= tw * (float)vj;
        i += G;
      }
#pragma unroll 4
      for (; i < rpc; i += G) A[i * b + my_c] = fmaf(-tw, A[i * b + j], A[i * b + my_c]);
    }
    __syncthreads();
  }
  cluster.sync();

  // ---- rank 0: SVD of R_R by one-sided Jacobi on its columns; R_R V = W_R diag(rho).
  __shared__ int s_p;
  if (rank == 0) {
    for (int e = tid; e < b * b; e += RES_NTH) {
      const int c = e / b, i = e % b;  // Rm column-major
      Rm[c * b + i] = i < c ? A[i * b + c] : (i == c ? alph[c] : 0.f);
    }
    __syncthreads();
    // Float32 inner products carry relative error ~ sqrt(b) 2^-24; the tolerance sits a few units
    // above it (a residual cosine of that size moves the rho only at second order). W_R reaches
    // the stored basis through P, so two-byte factors take the fold core's floor (see
    // core_tol_floor).
    const float tol = fmaxf(4.f * sqrtf((float)b) * 5.9604645e-08f, core_tol_floor(p.storage, false));
    const int sw = b <= 16   ? cta_jacobi_columns<1>(Rm, b, b, b, tol, 60)
                   : b <= 32 ? cta_jacobi_columns<2>(Rm, b, b, b, tol, 60)
                   : b <= 64 ? cta_jacobi_columns<4>(Rm, b, b, b, tol, 60)
                             : cta_jacobi_columns<8>(Rm, b, b, b, tol, 60);
    __shared__ float nrm[128];
    __shared__ int order[128];
    if (tid < b) {
      double s = 0.0;
      for (int i = 0; i < b; ++i) s = fma((double)Rm[tid * b + i], (double)Rm[tid * b + i], s);
      const float v = (float)sqrt(s);
      nrm[tid] = isfinite(v) ? v : -1.f;  // non-finite input ranks last; the order stays total
      if (!isfinite(v)) record_status(jb.h.meta, ISKV_ERR_NONFINITE);
    }
    __syncthreads();
    if (tid < b) {  // rank by (norm desc, index asc): a permutation of 0..b-1
      int rk = 0;
      for (int c = 0; c < b; ++c)
        rk += (nrm[c] > nrm[tid]) || (nrm[c] == nrm[tid] && c < tid);
      order[min(rk, b - 1)] = tid;
    }
    __syncthreads();
    if (tid == 0) {
      const float sigma1 = k > 0 ? jb.h.sigma[0] : 0.f;
      const double rho1 = nrm[order[0]];
      const double s_ref = fmax((double)sigma1, rho1);
      const double tol_r = fmax((double)p.tau_rel, 1.1920928955078125e-07 * (double)max(b, d)) * s_ref;
      int pp = 0;
      if (k < d)
        while (pp < b && (double)nrm[order[pp]] > tol_r) ++pp;
      s_p = pp;
      sc[FS_P] = pp;
      sc[FS_RSWEEPS] = sw;
      if (sw < 0) record_status(jb.h.meta, ISKV_ERR_NOT_CONVERGED);
    }
    __syncthreads();
    const int pp = s_p;
    if (tid < b) rho_out[tid] = nrm[order[tid]];
    // W[i][q] = Rm[:, order[q]] / rho for q < p (row-major b x b).
    for (int e = tid; e < b * pp; e += RES_NTH) {
      const int i = e / pp, q = e % pp;
      const int c = min(max(order[q], 0), b - 1);
      W[i * b + q] = Rm[c * b + i] / nrm[c];
    }
    __syncthreads();
    // Y1 = V_top^T W_p (V_top = rows 0..b-1 of the reflectors, lower triangular), Y2 = T Y1.
    float *Y1 = Rm;  // scratch, b x b (R_R's columns are no longer needed once W is formed)
    for (int e = tid; e < b * pp; e += RES_NTH) {
      const int l = e / pp, q = e % pp;
      double s = (double)vdiag[l] * W[l * b + q];
      for (int i = l + 1; i < b; ++i) s = fma((double)A[i * b + l], (double)W[i * b + q], s);
      Y1[l * b + q] = (float)s;
    }
    __syncthreads();
    for (int e = tid; e < b * pp; e += RES_NTH) {
      const int l = e / pp, q = e % pp;
      double s = 0.0;
      for (int m = l; m < b; ++m) s = fma((double)T[l * b + m], (double)Y1[m * b + q], s);
      Y2[l * b + q] = (float)s;
    }
  } else {
    // Other ranks have not reached the rank-0 block; they wait at the next cluster barrier.
  }
  cluster.sync();
  // p broadcast: every CTA reads rank 0's s_p.
  const int pp = *cluster.map_shared_rank(&s_p, 0);

  // ---- P rows: P = [W_p; 0] - V Y2 for my rows, then my partial of F P. Both are small
  // products done with 8 x 8 (P) and 4 x 4 (F P) register tiles in float32; Y2 and my P rows are
  // staged in shared memory (R_R's buffer and the reflector buffer, both free by now).
  float *Y2s = Rm;  // b x b, Y2[l][q] at l * b + q
  for (int e = tid; e < b * b; e += RES_NTH) {
    const int l = e / b, q = e % b;
    Y2s[e] = q < pp ? Y2[l * b + q] : 0.f;
  }
  __syncthreads();
  {
    // Thread (ti, tq) owns rows ti*8 .. ti*8+7 (strided by rpc/8 groups) and columns tq*8 .. tq*8+7.
    constexpr int PT = 8;
    const int ncg = (b + PT - 1) / PT;              // column groups
    const int nrg = RES_NTH / ncg;                  // row groups
    const int tq = tid % ncg, tig = tid / ncg;
    const int niter = (rpc + nrg * PT - 1) / (nrg * PT);  // the same for every thread (barrier)
    float acc[PT][PT];
    for (int it = 0; it < niter; ++it) {
      const int i0 = (it * nrg + tig) * PT;
#pragma unroll
      for (int u = 0; u < PT; ++u)
#pragma unroll
        for (int v = 0; v < PT; ++v) acc[u][v] = 0.f;
      for (int l = 0; l < b; ++l) {
        float yv[PT], vv[PT];
#pragma unroll
        for (int v = 0; v < PT; ++v) yv[v] = Y2s[l * b + tq * PT + v];
#pragma unroll
        for (int u = 0; u < PT; ++u) {
          const int i = i0 + u, gi = row0 + i;
          vv[u] = (i < rpc && gi >= l) ? (gi == l ? vdiag[l] : A[i * b + l]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < PT; ++u)
#pragma unroll
          for (int v = 0; v < PT; ++v) acc[u][v] = fmaf(vv[u], yv[v], acc[u][v]);
      }
      __syncthreads();  // every thread has read the reflectors of its rows before any is replaced
#pragma unroll
      for (int u = 0; u < PT; ++u) {
        const int i = i0 + u, gi = row0 + i;
        if (i >= rpc) continue;
#pragma unroll
        for (int v = 0; v < PT; ++v) {
          const int q = tq * PT + v;
          if (q >= b) continue;
          const float wv = (gi < b && q < pp) ? W[gi * b + q] : 0.f;
          const float pv = q < pp ? wv - acc[u][v] : 0.f;
          A[i * b + q] = pv;                 // my P rows, for F P below
          if (q < pp) P[(size_t)gi * b + q] = pv;
        }
      }
    }
  }
  __syncthreads();
  // F P partial over my rows: fpp[m][q] = sum_i F[m][row0 + i] P[row0 + i][q].
  const TF *F = static_cast<const TF *>(jb.F);
  {
    constexpr int FT = 4;
    const int ncg = (b + FT - 1) / FT, nmg = (b + FT - 1) / FT;
    for (int g = tid; g < ncg * nmg; g += RES_NTH) {
      const int tq = g % ncg, tm = g / ncg;
      float acc[FT][FT];
#pragma unroll
      for (int u = 0; u < FT; ++u)
#pragma unroll
        for (int v = 0; v < FT; ++v) acc[u][v] = 0.f;
      for (int i = 0; i < rpc; ++i) {
        float fv[FT], pv[FT];
#pragma unroll
        for (int u = 0; u < FT; ++u) {
          const int m = tm * FT + u;
          fv[u] = m < b ? to_f<TF>(F[(size_t)m * d + row0 + i]) : 0.f;
        }
#pragma unroll
        for (int v = 0; v < FT; ++v) {
          const int q = tq * FT + v;
          pv[v] = q < b ? A[i * b + q] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < FT; ++u)
#pragma unroll
          for (int v = 0; v < FT; ++v) acc[u][v] = fmaf(fv[u], pv[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < FT; ++u)
#pragma unroll
        for (int v = 0; v < FT; ++v) {
          const int m = tm * FT + u, q = tq * FT + v;
          if (m < b && q < b) fpp[m * b + q] = acc[u][v];
        }
    }
  }
  cluster.sync();
  if (rank == 0) {
    for (int e = tid; e < b * pp; e += RES_NTH) {
      const int m = e / pp, q = e % pp;
      float s = 0.f;
      for (int c = 0; c < cq; ++c) s += cluster.map_shared_rank(fpp, c)[m * b + q];
      FP[m * b + q] = s;
    }
  }
  cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
}

size_t fold_residual_smem(int d, int b) {
  const int cq = residual_cluster_size(d, b);
  return cq < 0 ? (size_t)-1 : residual_smem(d, b, cq).total;
}

cudaError_t launch_fold_residual(const FoldJob *jobs, const FoldParams &p, cudaStream_t s) {
  const int cq = residual_cluster_size(p.d, p.b);
  const ResidualSmem L = residual_smem(p.d, p.b, cq);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.count * cq);
  cfg.blockDim = dim3(RES_NTH);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cq;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaSuccess;
  with_dtype(p.f_dtype, [&](auto tf) {
    using TF = decltype(tf);
    e = cudaFuncSetAttribute(k_fold_residual<TF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L.total);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, k_fold_residual<TF>, jobs, p);
  });
  if (e != cudaSuccess) return e;
  count_launches(1);
  return e;
}

}  // namespace iskv
