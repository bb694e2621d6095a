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
// blocks (w steps of w disjoint pairs, one half-warp per pair); in the first round of a sweep it
// also rotates the pairs inside each block. Rotations apply in float32; inner products accumulate
// in float32, or in float64 for the re-orthogonalisation of float32-stored factors.
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

// Work counters of the core SVD, per mode (0: fold, 1: re-orthogonalisation), accumulated over
// every launch until reset: {cores solved, sweeps summed over cores, largest sweep count, pair
// checks taken (inner products of a column pair), rotations applied, float32 flops}. The flop
// count charges 2 m per pair check (one inner product over the m rows of A) and 8 (m + pp) per
// rotation (two FMAs per element of each of the two columns, V rows included); the per-round norm
// recomputations are not counted.
static __device__ unsigned long long g_core_stats[2][CORE_STATS];

struct CoreSmem {
  size_t buf, stamp, pairs, where, nP, nQ, nrm_local, anrm, vnrm, nrm_all, flags, total;
};

// Shared-memory plan (4-byte words). Column blocks are double-buffered when `dbuf` so a round's
// block exchange needs a single cluster barrier.
__host__ __device__ inline CoreSmem core_smem(int cj, int w, int ne, bool dbuf) {
  CoreSmem s;
  size_t o = 0;
  auto take = [&](size_t words) { size_t at = o; o += words; return at; };
  const int M = 2 * cj;
  s.buf = take((size_t)(dbuf ? 2 : 1) * 2 * w * 32 * ne);
  s.stamp = take((size_t)(dbuf ? 2 : 1) * 2 * w);
  s.pairs = take((size_t)(M - 1) * cj * 2);
  s.where = take((size_t)(M - 1) * M);
  s.nP = take((size_t)w);
  s.nQ = take((size_t)w);
  s.nrm_local = take((size_t)2 * w);
  s.anrm = take((size_t)2 * w);
  s.vnrm = take((size_t)2 * w);
  s.nrm_all = take((size_t)M * w);
  s.flags = take(4);
  s.total = o * 4;
  return s;
}

constexpr size_t kCoreSmemCap = 200 * 1024;

// Threads per CTA the register file allows for NE column entries per lane (four columns live in
// registers): 640 x 96, 512 x 128, 384 x 170 or 256 x 255 registers.
__host__ __device__ constexpr int core_max_threads(int ne) {
  return ne <= 12 ? 640 : (ne <= 16 ? 512 : (ne <= 24 ? 384 : 256));
}

// Columns per block w (two blocks per CTA, two column pairs per warp, so w / 2 warps): the
// smallest cluster whose blocks fit the warp budget and the shared-memory cap; column blocks are
// double-buffered when that fits too. `ne` = 0 when no register template covers the column.
JacobiCfg jacobi_cfg(int ncols_max, int col_len_max) {
  JacobiCfg c;
  int ne = (col_len_max + 31) / 32;
  const int choices[] = {2, 4, 8, 12, 16, 20, 24, 32};
  int pick = 0;
  for (int v : choices)
    if (v >= ne) { pick = v; break; }
  c.ne = pick;
  const int nes = pick ? pick : 32;
  for (int cj = 1; cj <= 16; cj *= 2) {
    int w = (ncols_max + 2 * cj - 1) / (2 * cj);
    w += w & 1;
    if (w < 4) w = 4;
    c.cj = cj;
    c.w = w;
    c.dbuf = core_smem(cj, w, nes, true).total <= kCoreSmemCap;
    c.smem = core_smem(cj, w, nes, c.dbuf).total;
    if (16 * w <= core_max_threads(nes) && c.smem <= kCoreSmemCap) break;
  }
  return c;
}

bool core_cfg(int r, int b, bool dense, JacobiCfg &c) {
  // Column length: the A part zero-padded to a multiple of 32, then the explicit V rows.
  const int pad32 = dense ? (r + 31) / 32 * 32 : (r + b + 31) / 32 * 32;
  const int len = dense ? pad32 + r : pad32 + b;
  c = jacobi_cfg(dense ? r : r + b, len);
  return c.ne > 0 && 16 * c.w <= core_max_threads(c.ne) && c.smem <= kCoreSmemCap;
}

// Register layout of a column: each half-warp holds one column; lane l16 = lane % 16 holds the
// float2 pairs l16 + 16 q (elements 2 l16 + 32 q and 2 l16 + 32 q + 1), q < NE, so loads, stores
// and the arithmetic run on packed float2 (sm_100 issues one FFMA2 for two FMAs), and the two
// half-warps of a warp work on two column pairs with one instruction stream: the per-pair
// rotation parameters and the 4-step reduction serve both pairs at once.
template <int NE>
ISKV_DEV void col_load(float2 (&x)[NE], const float *src) {
  const float2 *s2 = reinterpret_cast<const float2 *>(src);
  const int l16 = threadIdx.x & 15;
#pragma unroll
  for (int q = 0; q < NE; ++q) x[q] = s2[l16 + 16 * q];
}

template <int NE>
ISKV_DEV void col_store(float *dst, const float2 (&x)[NE]) {
  float2 *d2 = reinterpret_cast<float2 *>(dst);
  const int l16 = threadIdx.x & 15;
#pragma unroll
  for (int q = 0; q < NE; ++q) d2[l16 + 16 * q] = x[q];
}

// Dot product of two half-warp-resident columns over their first 32 nq entries (the A part,
// zero-padded to a multiple of 32); every lane of the half-warp receives the sum. Both half-warps
// of the warp must call it together (the reduction shuffles across the whole warp).
template <int NE, bool DD>
ISKV_DEV float half_dot(const float2 (&x)[NE], const float2 (&y)[NE], int nq) {
  if (DD) {  // float64 accumulation of the exact float32 products
    double a0 = 0.0, a1 = 0.0;
#pragma unroll
    for (int q = 0; q < NE; ++q)
      if (q < nq) {
        a0 = fma((double)x[q].x, (double)y[q].x, a0);
        a1 = fma((double)x[q].y, (double)y[q].y, a1);
      }
    double v = a0 + a1;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return (float)v;
  }
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < NE; ++q)
    if (q < nq) {
      if (q & 1) a1 = __ffma2_rn(x[q], y[q], a1);
      else a0 = __ffma2_rn(x[q], y[q], a0);
    }
  float v = (a0.x + a1.x) + (a0.y + a1.y);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One Jacobi rotation of the pair (x, y) with squared norms ax, by and inner product g, when the
// pair is not orthogonal to tolerance (g^2 > tol^2 ax by). Rutishauser's angle: zeta =
// (by - ax) / 2g, t = tan(theta) = sign(zeta) / (|zeta| + sqrt(1 + zeta^2)); applied in the
// half-angle form
//   x' = x - s (y + tau x),  y' = y + s (x - tau y),  tau = tan(theta / 2),  s = 2 tau / (1 + tau^2),
// which equals (c x - s y, s x + c y) and stays orthogonal to rounding because s is derived from
// tau. The parameters only have to define some rotation that nearly orthogonalises the pair (a
// residual cosine is removed by a later sweep), so they use the hardware reciprocal and
// reciprocal square root. Norms follow Rutishauser: ax -= t g, by += t g. Both accumulation modes
// (DD: the inner products were summed in float64) use these float32 parameters.
template <int NE, bool DD>
ISKV_DEV bool rotate_regs(float2 (&x)[NE], float2 (&y)[NE], float &ax, float &by, float g,
                          float tol2) {
  if (!(g != 0.f && g * g > (tol2 * ax) * by)) return false;
  const float zeta = 0.5f * (by - ax) * __fdividef(1.f, g);
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
  const float s = __fdividef(2.f * tau, fmaf(tau, tau, 1.f));
  const float2 s2 = make_float2(s, s), ms2 = make_float2(-s, -s);
  const float2 t2 = make_float2(tau, tau), mt2 = make_float2(-tau, -tau);
#pragma unroll
  for (int q = 0; q < NE; ++q) {
    const float2 xv = x[q], yv = y[q];
    x[q] = __ffma2_rn(ms2, __ffma2_rn(t2, xv, yv), xv);
    y[q] = __ffma2_rn(s2, __ffma2_rn(mt2, yv, xv), yv);
  }
  ax -= t * g;
  by += t * g;
  if (ax < 0.f) ax = 0.f;
  if (by < 0.f) by = 0.f;
  return true;
}

template <int NE, bool DD>
__global__ void __launch_bounds__(core_max_threads(NE)) k_core(const char *jobs, CoreParams p, int w, int dbuf) {
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
  const int mp = (m + 31) / 32 * 32;            // A part zero-padded to whole half-warp rows
  const int nq = mp / 32;                       // float2 pairs per lane in the A part
  const int ncol = dense ? k : k + pp, kn = min(r, ncol);
  const CoreSmem S = core_smem(cj, w, NE, dbuf != 0);
  extern __shared__ float smem[];
  float *buf0 = smem + S.buf;
  const int bufw = 2 * w * LP;                  // words per buffer
  // Per column: 1 + the step at which it was last rotated (0: never), moved with the column.
  int *stamp0 = reinterpret_cast<int *>(smem + S.stamp);
  int *pairs = reinterpret_cast<int *>(smem + S.pairs);   // [M-1][cj][2]
  int *where = reinterpret_cast<int *>(smem + S.where);   // [M-1][M] = cta * 2 + slot
  float *nP = smem + S.nP, *nQ = smem + S.nQ;
  float *nrm_local = smem + S.nrm_local;
  float *anrm = smem + S.anrm, *vnrm = smem + S.vnrm;
  float *nrm_all = smem + S.nrm_all;
  int *flags = reinterpret_cast<int *>(smem + S.flags);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = w / 2;                         // warps; half-warp h of warp i owns column i + h nw
  const int l16 = lane & 15;
  const int c = warp + (lane >> 4) * nw;

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
  for (int e = tid; e < (dbuf ? 2 : 1) * 2 * w; e += blockDim.x) stamp0[e] = 0;
  __syncthreads();

  // Build my two blocks for round 0.
  const float *sig_old = jh.sigma;
  const float *C = reinterpret_cast<const float *>(jh.ws + p.C);
  const float *FP = reinterpret_cast<const float *>(jh.ws + p.FP);
  const float *Md = reinterpret_cast<const float *>(jh.ws + p.M);
  for (int e = tid; e < bufw; e += blockDim.x) {
    const int slot = e / (w * LP), lc = (e / LP) % w, el = e % LP;
    const int j = pairs[(0 * cj + rank) * 2 + slot] * w + lc;
    // Column layout: A rows [0, m), zeros [m, mp), explicit V rows [mp, mp + pp), zeros after.
    float v = 0.f;
    if (dense) {
      if (j < k) {
        if (el < k) v = Md[(size_t)el * p.ldm + j];
        else if (el >= mp && el < mp + pp) v = (el - mp == j) ? 1.f : 0.f;
      }
    } else if (el < k) {
      v = (j < k && el == j) ? sig_old[j] : 0.f;
    } else if (el < m) {
      const int i = el - k;
      v = j < k ? C[(size_t)i * r + j] : (j < ncol ? FP[(size_t)i * b + (j - k)] : 0.f);
    } else if (el >= mp && el < mp + pp) {
      v = (j >= k && j < ncol && el - mp == j - k) ? 1.f : 0.f;
    }
    buf0[e] = v;
  }
  __syncthreads();

  // Rotate unless |cos| <= tol. In float32 the inner product has relative error ~ sqrt(m) 2^-24 and
  // the tolerance sits a few units above it; residual cosines of that size change singular values
  // only at second order. The re-orthogonalisation of float32 factors (whose purpose is
  // orthonormal factors to float32 accuracy) accumulates inner products in float64 and uses a
  // tighter tolerance.
  const float tol = fmaxf((DD ? 2.f : 4.f) * sqrtf((float)(m > 1 ? m : 1)) * 5.9604645e-08f,
                          p.tol_floor);
  const float tol2 = tol * tol;
  int sweeps_used = -1;
  int cur = 0;  // which buffer holds the current blocks (double-buffered exchange)
  // Every sweep takes the same pairs at the same steps, steps_per_sweep apart. A pair whose two
  // columns have not been rotated since it was checked one sweep ago would give the same inner
  // product and again no rotation, so its check is skipped -- when both pairs of a warp are such
  // pairs (the warp's shuffle reductions stay warp-uniform). The result is unchanged bit for bit;
  // the late sweeps, where most columns have stopped moving, shrink to their barriers.
  const int steps_per_sweep = (w - 1) + (M - 1) * w;
  int gs = 0;  // steps taken so far
  for (int sweep = 0; sweep < p.max_sweeps; ++sweep) {
    unsigned rot = 0;  // rotations this half-warp applied in this sweep
    for (int t = 0; t < M - 1; ++t) {
      float *buf = buf0 + (dbuf ? cur * bufw : 0);
      float *Pb = buf, *Qb = buf + w * LP;
      int *stP = stamp0 + (dbuf ? cur * 2 * w : 0), *stQ = stP + w;
      // Exact squared norms at the start of the round; tracked through the round's rotations.
      {
        float2 x[NE], y[NE];
        col_load<NE>(x, Pb + c * LP);
        col_load<NE>(y, Qb + c * LP);
        const float a = half_dot<NE, DD>(x, x, nq), cq = half_dot<NE, DD>(y, y, nq);
        if (l16 == 0) { nP[c] = a; nQ[c] = cq; }
      }
      __syncthreads();
      if (t == 0) {
        // Pairs inside each block (both columns from shared memory): half-warp c takes pair
        // c mod w/2 of block c / (w/2).
        for (int st = 0; st < w - 1; ++st, ++gs) {
          const int slot = c < w / 2 ? 0 : 1, q = slot ? c - w / 2 : c;
          const int a = circle_player(q, st, w), bb = circle_player(w - 1 - q, st, w);
          float *base = slot ? Qb : Pb;
          float *nb = slot ? nQ : nP;
          int *sb = slot ? stQ : stP;
          const int seen = gs - steps_per_sweep;  // the step that last checked this pair
          const bool idle = sweep > 0 && sb[a] <= seen && sb[bb] <= seen;
          if (__all_sync(0xffffffffu, idle)) {
            if (lane == 0) atomicAdd(reinterpret_cast<unsigned *>(flags + 3), 2u);
          } else {
            float2 x[NE], y[NE];
            col_load<NE>(x, base + a * LP);
            col_load<NE>(y, base + bb * LP);
            float ax = nb[a], by = nb[bb];
            const float g = half_dot<NE, DD>(x, y, nq);
            if (rotate_regs<NE, DD>(x, y, ax, by, g, tol2)) {
              col_store<NE>(base + a * LP, x);
              col_store<NE>(base + bb * LP, y);
              if (l16 == 0) { nb[a] = ax; nb[bb] = by; sb[a] = gs + 1; sb[bb] = gs + 1; }
              ++rot;
            }
          }
          __syncthreads();
        }
      }
      // Cross pairs: half-warp c keeps P[c] in registers while the Q columns circulate.
      float2 x[NE];
      col_load<NE>(x, Pb + c * LP);
      float ax = nP[c];
      int sx = stP[c];
      for (int st = 0; st < w; ++st, ++gs) {
        int qc = c + st;  // (c + st) mod w, with c, st < w
        if (qc >= w) qc -= w;
        const int seen = gs - steps_per_sweep;
        const bool idle = sweep > 0 && sx <= seen && stQ[qc] <= seen;
        if (__all_sync(0xffffffffu, idle)) {
          if (lane == 0) atomicAdd(reinterpret_cast<unsigned *>(flags + 3), 2u);
        } else {
          float2 y[NE];
          col_load<NE>(y, Qb + qc * LP);
          float by = nQ[qc];
          const float g = half_dot<NE, DD>(x, y, nq);
          if (rotate_regs<NE, DD>(x, y, ax, by, g, tol2)) {
            col_store<NE>(Qb + qc * LP, y);
            if (l16 == 0) { nQ[qc] = by; stQ[qc] = gs + 1; }
            sx = gs + 1;
            ++rot;
          }
        }
        __syncthreads();
      }
      if (cj == 1) {
        col_store<NE>(Pb + c * LP, x);
        if (l16 == 0) stP[c] = sx;
        __syncthreads();
        continue;
      }
      // Move both blocks to where round t+1 needs them.
      const int tn = (t + 1) % (M - 1);
      const int X0 = pairs[(t * cj + rank) * 2 + 0], X1 = pairs[(t * cj + rank) * 2 + 1];
      const int d0 = where[tn * M + X0], d1 = where[tn * M + X1];
      float2 y[NE];
      col_load<NE>(y, Qb + c * LP);
      const int sy = stQ[c];
      float *dst = dbuf ? buf0 + (cur ^ 1) * bufw : buf0;
      int *sdst = stamp0 + (dbuf ? (cur ^ 1) * 2 * w : 0);
      if (!dbuf) cluster.sync();  // single buffer: everyone has read its blocks before writes
      {
        float *r0 = cluster.map_shared_rank(dst, d0 >> 1) + (d0 & 1) * w * LP;
        float *r1 = cluster.map_shared_rank(dst, d1 >> 1) + (d1 & 1) * w * LP;
        col_store<NE>(r0 + c * LP, x);
        col_store<NE>(r1 + c * LP, y);
        if (l16 == 0) {
          cluster.map_shared_rank(sdst, d0 >> 1)[(d0 & 1) * w + c] = sx;
          cluster.map_shared_rank(sdst, d1 >> 1)[(d1 & 1) * w + c] = sy;
        }
      }
      cluster.sync();
      if (dbuf) cur ^= 1;
    }
    // Cluster-wide "any rotation in this sweep".
    if (l16 == 0 && rot) atomicAdd(reinterpret_cast<unsigned *>(flags + 2), rot);
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
  float *buf = buf0 + (dbuf ? cur * bufw : 0);

  // Singular values of my columns (blocks are at their round-0 places again). A column of A is
  // Z times the matching column of V, and both come out of the float32 rotations a little too
  // long: a rotation by a small angle theta should shorten a column's dominant entry (near +-1 in
  // V, near sigma in A) by theta^2 / 2 of itself, which float32 cannot represent below half an
  // ulp, while the first-order growth of the small entries is kept. Over a fold's few hundred
  // rotations per column this lengthens both by ~1e-6 relative, the same for A and V. So
  // sigma' = |A_q| / |V_q|, G_q = A_q / |A_q| and H_q = V_q / |V_q|: then Z H_q = G_q sigma'_q, and
  // the kept product is Z times a projector instead of growing by |V_q|^2 at every fold.
  const int nv = dense ? k : pp;  // explicit V rows after the A part
  for (int e = warp; e < 2 * w; e += nw) {
    const float *x = buf + e * LP;
    double sa = 0.0, sv = 0.0;
#pragma unroll
    for (int t = 0; t < NE; ++t) {
      const int idx = lane + 32 * t;
      const double v = x[idx];
      if (idx < m) {
        sa = fma(v, v, sa);
        if (!dense && idx < k && sig_old[idx] > 0.f) {
          const double hv = v / (double)sig_old[idx];
          sv = fma(hv, hv, sv);
        }
      } else if (idx >= mp && idx < mp + nv) {
        sv = fma(v, v, sv);
      }
    }
    sa = warp_sum(sa);
    sv = warp_sum(sv);
    if (lane == 0) {
      const double vn = sv > 0.0 ? sqrt(sv) : 1.0;
      anrm[e] = (float)sqrt(sa);
      vnrm[e] = (float)vn;
      nrm_local[e] = (float)(sqrt(sa) / vn);
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
  __half *Gtb = reinterpret_cast<__half *>(jh.ws + p.Gtb);  // fp16: the tensor-core rotation's type
  float *Gbot = reinterpret_cast<float *>(jh.ws + p.Gbot);
  float *Ht = reinterpret_cast<float *>(jh.ws + p.Ht);
  float *sig = reinterpret_cast<float *>(jh.ws + p.sig);
  const int npad = M * w;
  for (int e = warp; e < 2 * w; e += nw) {
    const int slot = e / w, lc = e % w;
    const int j = pairs[(0 * cj + rank) * 2 + slot] * w + lc;
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
    const float *x = buf + e * LP;
    const float inv = anrm[e] > 0.f ? 1.f / anrm[e] : 0.f;
    const float vinv = 1.f / vnrm[e];
    if (lane == 0) sig[q] = nj;
    for (int l = lane; l < r; l += 32) {
      const float g = l < k ? x[l] * inv : 0.f;
      Gt[(size_t)q * r + l] = g;
      Gtb[(size_t)q * r + l] = __float2half_rn(g);
    }
    for (int i = lane; i < b; i += 32) Gbot[(size_t)i * r + q] = x[k + i] * inv;
    for (int l = lane; l < hs; l += 32) {
      float h = 0.f;
      if (dense) h = l < k ? x[mp + l] : 0.f;
      else if (l < k) h = sig_old[l] > 0.f ? x[l] / sig_old[l] : 0.f;
      else if (l < ncol) h = x[mp + (l - k)];
      Ht[(size_t)q * hs + l] = h * vinv;
    }
  }
  // Zero the rows / columns beyond k'.
  for (int q = kn + rank; q < r; q += cj) {
    for (int l = tid; l < r; l += blockDim.x) {
      Gt[(size_t)q * r + l] = 0.f;
      Gtb[(size_t)q * r + l] = __float2half_rn(0.f);
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
  {
    // Work counters. Every sweep takes each pair of the M w (padded) columns once, less the pair
    // checks skipped as unchanged (counted per CTA); the CTA's rotations were summed in shared
    // memory at the end of each sweep. Subtractions go in as two's-complement additions.
    unsigned long long *st = g_core_stats[dense ? 1 : 0];
    const unsigned long long rsum = *reinterpret_cast<const unsigned *>(flags + 2);
    const unsigned long long skipped = *reinterpret_cast<const unsigned *>(flags + 3);
    if (tid == 0 && rsum) {
      atomicAdd(&st[4], rsum);
      atomicAdd(&st[5], rsum * (8ull * (unsigned)(m + pp)));
    }
    if (tid == 0 && skipped) {
      atomicAdd(&st[3], 0ull - skipped);
      atomicAdd(&st[5], 0ull - skipped * (2ull * (unsigned)m));
    }
    if (rank == 0 && tid == 0) {
      const unsigned long long sw = sweeps_used < 0 ? (unsigned long long)p.max_sweeps
                                                    : (unsigned long long)sweeps_used;
      const unsigned long long np = (unsigned long long)(M * w);
      const unsigned long long chk = sw * (np * (np - 1) / 2);
      atomicAdd(&st[0], 1ull);
      atomicAdd(&st[1], sw);
      atomicMax(&st[2], sw);
      atomicAdd(&st[3], chk);
      atomicAdd(&st[5], chk * (2ull * (unsigned)m));
    }
  }
  cluster.sync();  // my shared memory stays valid until every CTA has read nrm_local
}

template <int NE>
static cudaError_t core_launch(const char *jobs, const CoreParams &p, const JacobiCfg &c,
                               cudaStream_t s) {
  auto kern = p.dd ? k_core<NE, true> : k_core<NE, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)c.smem);
  if (e != cudaSuccess) return e;
  if (c.cj > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.count * c.cj);
  cfg.blockDim = dim3(16 * c.w);  // w / 2 warps
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
  return cudaLaunchKernelEx(&cfg, kern, jobs, p, c.w, c.dbuf ? 1 : 0);
}

cudaError_t launch_core(const char *jobs, const CoreParams &p, cudaStream_t s) {
  JacobiCfg c;
  if (!core_cfg(p.r, p.b, p.mode == 1, c)) return cudaErrorInvalidConfiguration;
  switch (c.ne) {
    case 2: return core_launch<2>(jobs, p, c, s);
    case 4: return core_launch<4>(jobs, p, c, s);
    case 8: return core_launch<8>(jobs, p, c, s);
    case 12: return core_launch<12>(jobs, p, c, s);
    case 16: return core_launch<16>(jobs, p, c, s);
    case 20: return core_launch<20>(jobs, p, c, s);
    case 24: return core_launch<24>(jobs, p, c, s);
    default: return core_launch<32>(jobs, p, c, s);
  }
}

cudaError_t core_stats(long long *out, bool reset) {
  unsigned long long h[2][CORE_STATS];
  cudaError_t e = cudaMemcpyFromSymbol(h, g_core_stats, sizeof h);
  if (e != cudaSuccess) return e;
  for (int m = 0; m < 2; ++m)
    for (int i = 0; i < CORE_STATS; ++i) out[m * CORE_STATS + i] = (long long)h[m][i];
  if (reset) {
    unsigned long long z[2][CORE_STATS] = {};
    e = cudaMemcpyToSymbol(g_core_stats, z, sizeof z);
  }
  return e;
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
  // Float32 factors (the parity-grade storage) take float64 inner products and the tighter
  // tolerance: the kept subspace is then decided to float32 accuracy at the truncation boundary,
  // where a nearly flat spectrum magnifies any residual cosine over a long trajectory. Two-byte
  // factors round far above that, and keep the float32 sweep.
  c.dd = p.storage == ISKV_F32 ? 1 : 0;
  c.tol_floor = core_tol_floor(p.storage, false);
  return c;
}

}  // namespace iskv
