// Fold steps 5-6 (iS-KV reading notes, Section 4.2 and Algorithm 2 steps 5-6): build the small core
// Z = [[diag(sigma), 0], [F B, F P]] ((k+b) x (k+p)) and take its SVD Z = G diag(sigma+) H^T,
// truncated to the top k' = min(r, k+p) components.
//
// Method: one-sided Jacobi (Hestenes 1958) on the columns of Z, A <- Z V, until the columns of A
// are mutually orthogonal; then sigma+ = column norms, G = normalised columns, H = V. Parallel
// ordering: block Jacobi on a thread-block cluster of CJ CTAs. The k+p columns (padded to 2 CJ w)
// are cut into 2 CJ blocks of w columns; each CTA holds two blocks in shared memory and a
// round-robin tournament over the blocks (2 CJ - 1 rounds per sweep) moves blocks between CTAs
// through distributed shared memory. Inside a round a CTA rotates every cross pair of its two
// blocks (w steps of w disjoint pairs, one warp per pair); in the first round of a sweep it also
// rotates the pairs inside each block. Dot products accumulate in float64, rotations apply in
// float32.
//
// Structure used: the top k rows of A equal diag(sigma) times the top k rows of V (they start as
// diag(sigma) and I and see the same column rotations), so those k rows of V are not stored:
// H[l, q] = A[l, q] / sigma_l. A column therefore holds its k+b entries of A plus the p explicit
// rows of V.
#include <cooperative_groups.h>

#include "jacobi_small.cuh"
#include "kernels.h"
#include "profiling.h"

namespace cg = cooperative_groups;

namespace iskv {


struct CoreSmem {
  size_t buf, pairs, where, nrm_local, nrm_all, flags, total;
};

__host__ __device__ inline CoreSmem core_smem(int cj, int w, int ne) {
  CoreSmem s;
  size_t o = 0;
  auto take = [&](size_t words) { size_t at = o; o += words; return at; };
  const int M = 2 * cj;
  s.buf = take((size_t)2 * w * 32 * ne);
  s.pairs = take((size_t)(M - 1) * cj * 2);
  s.where = take((size_t)(M - 1) * M);
  s.nrm_local = take((size_t)2 * w);
  s.nrm_all = take((size_t)M * w);
  s.flags = take(4);
  s.total = o * 4;
  return s;
}

JacobiCfg jacobi_cfg(int ncols_max, int col_len_max) {
  JacobiCfg c;
  int cj = 1;
  for (;;) {
    int w = (ncols_max + 2 * cj - 1) / (2 * cj);
    w += w & 1;
    if (w <= 20 || cj == 16) {
      c.cj = cj;
      c.w = w < 2 ? 2 : w;
      break;
    }
    cj *= 2;
  }
  int ne = (col_len_max + 31) / 32;
  const int choices[] = {2, 4, 8, 12, 16, 20, 24};
  for (int v : choices)
    if (v >= ne) { ne = v; break; }
  c.ne = ne;
  c.smem = core_smem(c.cj, c.w, c.ne).total;
  return c;
}

// Rotate the pair of columns x, y (length 32 * NE, this warp) if they are not yet orthogonal to
// tolerance; the dot products cover the first m entries only.
template <int NE>
ISKV_DEV bool warp_rotate_pair(float *x, float *y, int m, double tol) {
  const int lane = threadIdx.x & 31;
  float xr[NE], yr[NE];
  double al = 0.0, be = 0.0, ga = 0.0;
#pragma unroll
  for (int t = 0; t < NE; ++t) {
    xr[t] = x[lane + 32 * t];
    yr[t] = y[lane + 32 * t];
    if (lane + 32 * t < m) {
      const double xv = xr[t], yv = yr[t];
      al = fma(xv, xv, al);
      be = fma(yv, yv, be);
      ga = fma(xv, yv, ga);
    }
  }
  al = warp_sum(al);
  be = warp_sum(be);
  ga = warp_sum(ga);
  if (!(ga != 0.0 && fabs(ga) > tol * sqrt(al * be))) return false;
  double c, s;
  jacobi_rotation(al, be, ga, c, s);
  const float cf = (float)c, sf = (float)s;
#pragma unroll
  for (int t = 0; t < NE; ++t) {
    const float xv = xr[t], yv = yr[t];
    x[lane + 32 * t] = cf * xv - sf * yv;
    y[lane + 32 * t] = sf * xv + cf * yv;
  }
  return true;
}

template <int NE>
__global__ void __launch_bounds__(640) k_core(const char *jobs, CoreParams p, int w) {
  cg::cluster_group cluster = cg::this_cluster();
  const int cj = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
  const JobHead &jh = job_head(jobs, p.job_stride, blockIdx.x / cj);
  int32_t *sc = reinterpret_cast<int32_t *>(jh.ws);
  if (sc[FS_SKIP]) return;  // uniform over the cluster

  constexpr int LP = 32 * NE;
  const int M = 2 * cj;
  const bool dense = p.mode == 1;
  const int k = sc[FS_K_OLD], b = dense ? 0 : p.b, r = p.r, hs = p.hs;
  const int pp = dense ? k : sc[FS_P];          // explicit V rows stored after the A part
  const int m = k + b;                          // A rows
  const int ncol = dense ? k : k + pp, kn = min(r, ncol);
  const CoreSmem S = core_smem(cj, w, NE);
  extern __shared__ float smem[];
  float *buf = smem + S.buf;
  int *pairs = reinterpret_cast<int *>(smem + S.pairs);   // [M-1][cj][2]
  int *where = reinterpret_cast<int *>(smem + S.where);   // [M-1][M] = cta * 2 + slot
  float *nrm_local = smem + S.nrm_local;
  float *nrm_all = smem + S.nrm_all;
  int *flags = reinterpret_cast<int *>(smem + S.flags);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // Tournament: round t, CTA 0 plays block M-1 against block t; CTA i plays (t+i) vs (t-i).
  for (int e = tid; e < (M - 1) * cj; e += blockDim.x) {
    const int t = e / cj, i = e % cj;
    int a, bb;
    if (i == 0) { a = M - 1; bb = t; }
    else { a = (t + i) % (M - 1); bb = (t - i + (M - 1)) % (M - 1); }
    pairs[(t * cj + i) * 2 + 0] = a;
    pairs[(t * cj + i) * 2 + 1] = bb;
    where[t * M + a] = i * 2 + 0;
    where[t * M + bb] = i * 2 + 1;
  }
  if (tid < 4) flags[tid] = 0;
  __syncthreads();

  // Build my two blocks for round 0.
  const float *sig_old = jh.sigma;
  const float *C = reinterpret_cast<const float *>(jh.ws + p.C);
  const float *FP = reinterpret_cast<const float *>(jh.ws + p.FP);
  const float *Md = reinterpret_cast<const float *>(jh.ws + p.M);
  for (int e = tid; e < 2 * w * LP; e += blockDim.x) {
    const int slot = e / (w * LP), lc = (e / LP) % w, el = e % LP;
    const int j = pairs[(0 * cj + rank) * 2 + slot] * w + lc;
    float v = 0.f;
    if (dense) {
      if (j < k) {
        if (el < k) v = Md[(size_t)el * p.ldm + j];
        else if (el < m + pp) v = (el - m == j) ? 1.f : 0.f;
      }
    } else if (el < k) {
      v = (j < k && el == j) ? sig_old[j] : 0.f;
    } else if (el < m) {
      const int i = el - k;
      v = j < k ? C[(size_t)i * r + j] : (j < ncol ? FP[(size_t)i * b + (j - k)] : 0.f);
    } else if (el < m + pp) {
      v = (j >= k && j < ncol && el - m == j - k) ? 1.f : 0.f;
    }
    buf[e] = v;
  }
  __syncthreads();

  const double tol = 2.0 * sqrt((double)(m > 1 ? m : 1)) * 5.960464477539063e-08;
  int sweeps_used = -1;
  for (int sweep = 0; sweep < p.max_sweeps; ++sweep) {
    bool rot = false;
    for (int t = 0; t < M - 1; ++t) {
      if (t == 0) {
        for (int st = 0; st < w - 1; ++st) {
          if (warp < w) {
            const int slot = warp < w / 2 ? 0 : 1, q = warp % (w / 2);
            const int a = circle_player(q, st, w), bb = circle_player(w - 1 - q, st, w);
            rot |= warp_rotate_pair<NE>(buf + (slot * w + a) * LP, buf + (slot * w + bb) * LP, m,
                                        tol);
          }
          __syncthreads();
        }
      }
      for (int st = 0; st < w; ++st) {
        if (warp < w) {
          const int bb = (warp + st) % w;
          rot |= warp_rotate_pair<NE>(buf + warp * LP, buf + (w + bb) * LP, m, tol);
        }
        __syncthreads();
      }
      if (cj > 1) {
        // Move both blocks to where round t+1 needs them (single buffer: read, barrier, write).
        const int tn = (t + 1) % (M - 1);
        float reg[2][NE];
        int dst[2];
#pragma unroll
        for (int slot = 0; slot < 2; ++slot) {
          const int X = pairs[(t * cj + rank) * 2 + slot];
          dst[slot] = where[tn * M + X];
          if (dst[slot] != rank * 2 + slot && warp < w) {
#pragma unroll
            for (int q = 0; q < NE; ++q) reg[slot][q] = buf[(slot * w + warp) * LP + lane + 32 * q];
          }
        }
        cluster.sync();
#pragma unroll
        for (int slot = 0; slot < 2; ++slot) {
          if (dst[slot] != rank * 2 + slot && warp < w) {
            const int dc = dst[slot] >> 1, ds = dst[slot] & 1;
            float *rb = cluster.map_shared_rank(buf, dc) + (ds * w + warp) * LP;
#pragma unroll
            for (int q = 0; q < NE; ++q) rb[lane + 32 * q] = reg[slot][q];
          }
        }
        cluster.sync();
      }
    }
    // Cluster-wide "any rotation in this sweep".
    const int any_local = __syncthreads_or(rot ? 1 : 0);
    if (tid == 0) flags[sweep & 1] = any_local;
    cluster.sync();
    int any = 0;
    for (int c = 0; c < cj; ++c) any |= *cluster.map_shared_rank(flags + (sweep & 1), c);
    if (!any) {
      sweeps_used = sweep + 1;
      break;
    }
  }

  // Column norms of my columns (blocks are at their round-0 places again).
  for (int slot = 0; slot < 2; ++slot) {
    if (warp < w) {
      const float *x = buf + (slot * w + warp) * LP;
      double s = 0.0;
#pragma unroll
      for (int t = 0; t < NE; ++t) {
        if (lane + 32 * t < m) {
          const double v = x[lane + 32 * t];
          s = fma(v, v, s);
        }
      }
      s = warp_sum(s);
      if (lane == 0) nrm_local[slot * w + warp] = (float)sqrt(s);
    }
  }
  cluster.sync();
  for (int e = tid; e < M * w; e += blockDim.x) {
    const int c = e / (2 * w), rest = e % (2 * w), slot = rest / w, lc = rest % w;
    const int X = pairs[(0 * cj + c) * 2 + slot];
    nrm_all[X * w + lc] = cluster.map_shared_rank(nrm_local, c)[slot * w + lc];
  }
  __syncthreads();

  // Outputs for my kept columns: rank q of column j by (norm desc, index asc).
  float *Gt = reinterpret_cast<float *>(jh.ws + p.Gt);
  __nv_bfloat16 *Gtb = reinterpret_cast<__nv_bfloat16 *>(jh.ws + p.Gtb);
  float *Gbot = reinterpret_cast<float *>(jh.ws + p.Gbot);
  float *Ht = reinterpret_cast<float *>(jh.ws + p.Ht);
  float *sig = reinterpret_cast<float *>(jh.ws + p.sig);
  const int npad = M * w;
  for (int slot = 0; slot < 2; ++slot) {
    if (warp >= w) continue;
    const int j = pairs[(0 * cj + rank) * 2 + slot] * w + warp;
    const float nj = nrm_all[j];
    // Rank by (norm desc, index asc) on a key where a non-finite norm sorts last, so the ranks
    // form a permutation even for NaN input.
    const float kj = isfinite(nj) ? nj : -1.f;
    int cnt = 0;
    for (int i = lane; i < npad; i += 32) {
      const float ni = nrm_all[i];
      const float ki = isfinite(ni) ? ni : -1.f;
      cnt += (ki > kj) || (ki == kj && i < j);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    const int q = cnt;
    if (j >= ncol || q >= kn) continue;
    if (!isfinite(nj) && lane == 0) record_status(jh.meta, ISKV_ERR_NONFINITE);
    const float *x = buf + (slot * w + warp) * LP;
    const float inv = nj > 0.f ? 1.f / nj : 0.f;
    if (lane == 0) sig[q] = nj;
    for (int l = lane; l < r; l += 32) {
      const float g = l < k ? x[l] * inv : 0.f;
      Gt[(size_t)q * r + l] = g;
      Gtb[(size_t)q * r + l] = __float2bfloat16_rn(g);
    }
    for (int i = lane; i < b; i += 32) Gbot[(size_t)i * r + q] = x[k + i] * inv;
    for (int l = lane; l < hs; l += 32) {
      float h = 0.f;
      if (dense) h = l < k ? x[m + l] : 0.f;
      else if (l < k) h = sig_old[l] > 0.f ? x[l] / sig_old[l] : 0.f;
      else if (l < ncol) h = x[m + (l - k)];
      Ht[(size_t)q * hs + l] = h;
    }
  }
  // Zero the rows / columns beyond k'.
  for (int q = kn + rank; q < r; q += cj) {
    for (int l = tid; l < r; l += blockDim.x) {
      Gt[(size_t)q * r + l] = 0.f;
      Gtb[(size_t)q * r + l] = __float2bfloat16_rn(0.f);
    }
    for (int l = tid; l < hs; l += blockDim.x) Ht[(size_t)q * hs + l] = 0.f;
    for (int i = tid; i < b; i += blockDim.x) Gbot[(size_t)i * r + q] = 0.f;
    if (tid == 0) sig[q] = 0.f;
  }
  if (rank == 0 && tid == 0) {
    sc[FS_K_NEW] = kn;
    sc[FS_SWEEPS] = sweeps_used;
    if (sweeps_used < 0) record_status(jh.meta, ISKV_ERR_NOT_CONVERGED);
  }
  cluster.sync();  // my shared memory stays valid until every CTA has read nrm_local
}

template <int NE>
static cudaError_t core_launch(const char *jobs, const CoreParams &p, const JacobiCfg &c,
                               cudaStream_t s) {
  auto kern = k_core<NE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)c.smem);
  if (e != cudaSuccess) return e;
  if (c.cj > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.count * c.cj);
  cfg.blockDim = dim3(32 * c.w);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = c.cj;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launches(1);
  return cudaLaunchKernelEx(&cfg, kern, jobs, p, c.w);
}

cudaError_t launch_core(const char *jobs, const CoreParams &p, cudaStream_t s) {
  const JacobiCfg c = p.mode == 1 ? jacobi_cfg(p.r, 2 * p.r) : jacobi_cfg(p.r + p.b, p.r + 2 * p.b);
  switch (c.ne) {
    case 2: return core_launch<2>(jobs, p, c, s);
    case 4: return core_launch<4>(jobs, p, c, s);
    case 8: return core_launch<8>(jobs, p, c, s);
    case 12: return core_launch<12>(jobs, p, c, s);
    case 16: return core_launch<16>(jobs, p, c, s);
    case 20: return core_launch<20>(jobs, p, c, s);
    default: return core_launch<24>(jobs, p, c, s);
  }
}

CoreParams fold_core_params(const FoldParams &p) {
  CoreParams c;
  c.r = p.r;
  c.b = p.b;
  c.count = p.count;
  c.job_stride = sizeof(FoldJob);
  c.mode = 0;
  c.C = p.ws.C;
  c.FP = p.ws.FP;
  c.M = 0;
  c.Gt = p.ws.Gt;
  c.Gtb = p.ws.Gtb;
  c.Gbot = p.ws.Gbot;
  c.Ht = p.ws.Ht;
  c.sig = p.ws.sig;
  c.hs = p.ws.hs;
  c.ldm = 0;
  c.max_sweeps = 40;
  return c;
}

}  // namespace iskv
