// Decode attention over the compressed cache (iS-KV reading notes, Algorithm 3 steps 7-9; Section
// 5.2 names this factor-aware form as the route to a speed-up): one query per (sequence, layer),
// grouped-query heads, without writing the dense cache.
//
//   scores  S[j][p] = scale * q_j . RoPE_p(k_p) for every key position p: compressed keys
//           k_p = (U_k[i] * sigma_k) B_k^T at p = pos_k[i] (tensor-core kernel in tc_kernels.cu or
//           the CUDA-core kernel below), exact keys at their positions; -inf where no key is;
//   softmax per query head j over the positions (max and sum of exponentials);
//   values  o_j = B_v,h sigma_v (sum_i P_j(pos_v[i]) U_v[i]) + sum_e P_j(pos_e) v_e:
//           the compressed values are mixed in the r-dimensional coordinate space and projected
//           once per query head (h = j / (n_q / n_kv)); exact values are mixed directly.
// The probability mass that lands on value rows is summed as well: a key position without a value
// row leaves it short of 1 and records ISKV_ERR_SHAPE.
#include "attention.h"
#include "gemm_tile.cuh"
#include "profiling.h"
#include "rope.cuh"

namespace iskv {

ISKV_DEV int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// ------------------------------------------------------------------------------------------------
__global__ void k_attn_init(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int64_t n = (int64_t)p.n_q * jb.n_total;
  const float ninf = -__int_as_float(0x7f800000);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    jb.S[e] = ninf;
}

cudaError_t launch_attn_init(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  const int64_t per = (int64_t)p.n_q * p.n_total_max;
  const int64_t blocks = (per + 1023) / 1024;
  const int gx = (int)(blocks < 1024 ? blocks : 1024);
  k_attn_init<<<dim3(gx > 0 ? gx : 1, p.count), 256, 0, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

// RoPE cosines and sines of position pos for the pairs j = lane + 32 t of this lane.
template <int T>
ISKV_DEV void key_angles(int64_t pos, int half, const double *invf, float (&c)[T], float (&s)[T]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int j = lane + 32 * t;
    c[t] = 1.f;
    s[t] = 0.f;
    if (j < half) rope_sincos(pos, invf[j], c[t], s[t]);
  }
}

// Scale, rotate and dot one key of KV head h, held as pairs (lo = k[j], hi = k[j + hd/2]) for
// j = lane + 32 t, with every query head of its group; lane 0 writes the scores.
template <int T>
ISKV_DEV void score_key(const AttnJob &jb, const AttnParams &p, int h, int64_t pos,
                        const float (&lo)[T], const float (&hi)[T], const float (&c)[T],
                        const float (&s)[T]) {
  const int lane = threadIdx.x & 31, half = p.head_dim / 2, qpk = p.n_q / p.n_kv;
  float rl[T], rh[T];
#pragma unroll
  for (int t = 0; t < T; ++t) {
    rl[t] = lo[t] * c[t] - hi[t] * s[t];
    rh[t] = hi[t] * c[t] + lo[t] * s[t];
  }
  for (int g = 0; g < qpk; ++g) {
    const int qh = h * qpk + g;
    const float *qv = jb.q + (size_t)qh * p.head_dim;
    float acc = 0.f;
#pragma unroll
    for (int t = 0; t < T; ++t) {
      const int j = lane + 32 * t;
      if (j < half) acc = fmaf(qv[j], rl[t], fmaf(qv[j + half], rh[t], acc));
    }
    acc = warp_sum(acc);
    if (lane == 0) jb.S[(size_t)qh * jb.n_total + pos] = p.scale * acc;
  }
}

// Compressed keys on CUDA cores (float32 factors, or shapes the tensor-core kernel does not take):
// one block per 8 rows of one history; each row is rebuilt in shared memory, then one warp per KV
// head rotates and scores it.
template <typename TS>
__global__ void __launch_bounds__(256) k_attn_scores_ffma(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int64_t n = jb.metak[ISKV_META_N];
  const int k = (int)jb.metak[ISKV_META_K];
  const int d = p.d, r = p.rk, hd = p.head_dim, half = hd / 2;
  extern __shared__ float sm[];
  float *us = sm;                 // [r] sigma-scaled coordinates
  float *krow = sm + r;           // [d] rebuilt key
  __shared__ double invf[128];
  for (int j = threadIdx.x; j < half; j += blockDim.x) invf[j] = rope_inv_freq(j, hd, log(p.theta));
  const TS *U = static_cast<const TS *>(jb.Uk);
  const TS *B = static_cast<const TS *>(jb.Bk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rr = 0; rr < 8; ++rr) {
    const int64_t i = (int64_t)blockIdx.x * 8 + rr;
    if (i >= n) break;  // uniform over the block
    __syncthreads();
    for (int l = threadIdx.x; l < r; l += blockDim.x)
      us[l] = l < k ? to_f<TS>(U[(size_t)i * r + l]) * jb.sk[l] : 0.f;
    __syncthreads();
    for (int f = threadIdx.x; f < d; f += blockDim.x) {
      float acc = 0.f;
      for (int l = 0; l < k; ++l) acc = fmaf(to_f<TS>(B[(size_t)f * r + l]), us[l], acc);
      krow[f] = acc;
    }
    __syncthreads();
    const int64_t pos = jb.posk[i];
    if (pos < 0 || pos >= jb.n_total) {
      if (threadIdx.x == 0) record_status(jb.metak, ISKV_ERR_SHAPE);
      continue;
    }
    float cs[4], sn[4];
    key_angles<4>(pos, half, invf, cs, sn);
    for (int h = warp; h < p.n_kv; h += blockDim.x >> 5) {
      float lo[4], hi[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int j = lane + 32 * t;
        lo[t] = j < half ? krow[h * hd + j] : 0.f;
        hi[t] = j < half ? krow[h * hd + j + half] : 0.f;
      }
      score_key<4>(jb, p, h, pos, lo, hi, cs, sn);
    }
  }
}

cudaError_t launch_attn_scores_ffma(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  const int gx = (int)((p.n_cap_max + 7) / 8);
  const size_t smem = sizeof(float) * (size_t)(p.rk + p.d);
  if (gx < 1) return cudaSuccess;
  with_dtype(p.storage, [&](auto ts) {
    k_attn_scores_ffma<decltype(ts)><<<dim3(gx, p.count), 256, smem, s>>>(jobs, p);
  });
  count_launches(1);
  return cudaGetLastError();
}

// Exact keys: one warp per exact row, every KV head of it.
template <typename TE>
__global__ void __launch_bounds__(256) k_attn_scores_exact(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int hd = p.head_dim, half = hd / 2;
  __shared__ double invf[128];
  for (int j = threadIdx.x; j < half; j += blockDim.x) invf[j] = rope_inv_freq(j, hd, log(p.theta));
  __syncthreads();
  const int64_t e = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= jb.n_kex) return;  // uniform over the warp; no block barrier follows
  const int lane = threadIdx.x & 31;
  const int64_t pos = jb.kexpos[e];
  if (pos < 0 || pos >= jb.n_total) {
    if (lane == 0) record_status(jb.metak, ISKV_ERR_SHAPE);
    return;
  }
  const TE *x = static_cast<const TE *>(jb.kex) + (size_t)e * p.d;
  float cs[4], sn[4];
  key_angles<4>(pos, half, invf, cs, sn);  // the same angles for every head of the row
  for (int h = 0; h < p.n_kv; ++h) {
    float lo[4], hi[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int j = lane + 32 * t;
      lo[t] = j < half ? to_f<TE>(x[h * hd + j]) : 0.f;
      hi[t] = j < half ? to_f<TE>(x[h * hd + j + half]) : 0.f;
    }
    score_key<4>(jb, p, h, pos, lo, hi, cs, sn);
  }
}

cudaError_t launch_attn_scores_exact(const AttnJob *jobs, const AttnParams &p, int64_t max_kex,
                                     cudaStream_t s) {
  if (max_kex <= 0) return cudaSuccess;
  const dim3 g((unsigned)((max_kex + 7) / 8), p.count);
  with_dtype(p.exact_dtype, [&](auto te) {
    k_attn_scores_exact<decltype(te)><<<g, 256, 0, s>>>(jobs, p);
  });
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Softmax statistics of one query head: max score and sum of exp(score - max) over positions.
__global__ void __launch_bounds__(256) k_attn_stats(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int qh = blockIdx.x;
  const float *s = jb.S + (size_t)qh * jb.n_total;
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m = -__int_as_float(0x7f800000);
  for (int64_t i = threadIdx.x; i < jb.n_total; i += blockDim.x) m = fmaxf(m, s[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(~0u, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  const bool any = m > -__int_as_float(0x7f800000);
  float z = 0.f;
  if (any)
    for (int64_t i = threadIdx.x; i < jb.n_total; i += blockDim.x) z += __expf(s[i] - m);
  z = warp_sum(z);
  if (lane == 0) red[warp] = z;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
    if (!any) {  // no key at all: nothing to attend to
      record_status(jb.metak, ISKV_ERR_SHAPE);
      m = 0.f;
      tot = 1.f;
    }
    jb.stats[2 * qh] = m;
    jb.stats[2 * qh + 1] = 1.f / tot;
  }
}

cudaError_t launch_attn_stats(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  k_attn_stats<<<dim3(p.n_q, p.count), 256, 0, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Probabilities at the compressed value rows, P_j(pos_v[i]), laid out densely by row so that the
// value mixing streams them: float32 [n_q][n_cap] for the CUDA-core GEMM, or bf16 [n_cap][64]
// (queries padded to 64 columns) for the tensor cores. Rows past the history, and rows outside
// the cache (flagged), get 0. Each block also sums its rows' probabilities per query head.
__global__ void __launch_bounds__(256) k_attn_probs(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int64_t n = jb.metav[ISKV_META_N], nt = jb.n_total;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jend = p.tc_values ? 64 : p.n_q;  // columns written per row
  __shared__ float red[8][ATTN_MAX_Q];
  float mass[ATTN_MAX_Q];
#pragma unroll
  for (int j = 0; j < ATTN_MAX_Q; ++j) mass[j] = 0.f;
  for (int u = 0; u < ATTN_PROB_ROWS; ++u) {
    // Rows of this block, strided by the block so that a warp's accesses stay contiguous.
    const int64_t i = ((int64_t)blockIdx.x * ATTN_PROB_ROWS + u) * blockDim.x + threadIdx.x;
    if (i >= p.n_cap_max) break;
    bool ok = false;
    int64_t pos = 0;
    if (i < n) {
      pos = jb.posv[i];
      ok = pos >= 0 && pos < nt;
      if (!ok) record_status(jb.metav, ISKV_ERR_SHAPE);
    }
    __nv_bfloat16 *pb = static_cast<__nv_bfloat16 *>(jb.Pb) + (size_t)i * 64;
#pragma unroll
    for (int j0 = 0; j0 < ATTN_MAX_Q; j0 += 2) {
      if (j0 >= jend) break;
      float v[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int j = j0 + t;
        v[t] = (ok && j < p.n_q)
                   ? __expf(jb.S[(size_t)j * nt + pos] - jb.stats[2 * j]) * jb.stats[2 * j + 1]
                   : 0.f;
        mass[j] += v[t];
      }
      if (p.tc_values)
        *reinterpret_cast<__nv_bfloat162 *>(pb + j0) = __floats2bfloat162_rn(v[0], v[1]);
      else
        for (int t = 0; t < 2; ++t)
          if (j0 + t < p.n_q) jb.P[(size_t)(j0 + t) * p.n_cap_max + i] = v[t];
    }
  }
#pragma unroll
  for (int j = 0; j < ATTN_MAX_Q; ++j) {
    if (j >= p.n_q) break;
    const float m = warp_sum(mass[j]);
    if (lane == 0) red[warp][j] = m;
  }
  __syncthreads();
  if (threadIdx.x < p.n_q) {
    float m = 0.f;
    for (int w = 0; w < 8; ++w) m += red[w][threadIdx.x];
    jb.mpart[(size_t)blockIdx.x * p.n_q + threadIdx.x] = m;
  }
}

cudaError_t launch_attn_probs(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  const unsigned gx = (unsigned)p.nblk;
  if (gx == 0) return cudaSuccess;
  k_attn_probs<<<dim3(gx, p.count), 256, 0, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Compressed values, mixed in coordinate space on CUDA cores: W_c = P_c^T U_v over the ATTN_CHUNK
// rows of chunk c -- a register-tiled GEMM (M = query heads, N = r, K = rows).
constexpr int AV_BM = 32, AV_BN = 64, AV_BK = 16, AV_TM = 4, AV_TN = 4;
constexpr int AV_THREADS = (AV_BM / AV_TM) * (AV_BN / AV_TN);

template <typename TS>
__global__ void __launch_bounds__(AV_THREADS) k_attn_values(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.z];
  const int mt = (p.n_q + AV_BM - 1) / AV_BM;
  const int c = blockIdx.y / mt, m0 = (blockIdx.y % mt) * AV_BM, n0 = blockIdx.x * AV_BN;
  const int nq = p.n_q, r = p.rv;
  const int64_t n = jb.metav[ISKV_META_N];
  const int k = (int)jb.metav[ISKV_META_K];
  const int64_t i0 = (int64_t)c * ATTN_CHUNK;
  const int rows = (int)min64(ATTN_CHUNK, n > i0 ? n - i0 : 0);
  const TS *U = static_cast<const TS *>(jb.Uv);
  const float *P = jb.P + i0;
  const size_t ldp = (size_t)p.n_cap_max;
  float *wp = jb.wpart + (size_t)c * nq * r;
  tile_gemm<AV_BM, AV_BN, AV_BK, AV_TM, AV_TN, true, true>(
      m0, n0, nq, r, rows,
      [&](int j, int i) { return P[(size_t)j * ldp + i]; },
      [&](int i, int l) { return l < k ? to_f<TS>(U[(size_t)(i0 + i) * r + l]) : 0.f; },
      [&](int j, int l, float acc) { wp[(size_t)j * r + l] = acc; });
}

cudaError_t launch_attn_values(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  const int mt = (p.n_q + AV_BM - 1) / AV_BM;
  const dim3 g((p.rv + AV_BN - 1) / AV_BN, mt * p.nchunk, p.count);
  with_dtype(p.storage, [&](auto ts) {
    k_attn_values<decltype(ts)><<<g, AV_THREADS, 0, s>>>(jobs, p);
  });
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Outputs of the query group of one KV head h, in AO_SPLIT parts per (head, job): part s takes
// a slice of the coordinates, o_j += B_v,h[:, slice] (sigma_v * sum_c wpart[c][j])[slice], and a
// slice of the exact rows, o_j += sum_e P_j(pos_e) v_e[h], and writes its partial outputs and
// probability mass; k_attn_final adds the parts in order and checks the mass. Each value row of
// the head is read once for the whole query group.
constexpr int AO_ROWS = 512;  // exact rows per staged batch

template <typename TS, typename TE>
__global__ void __launch_bounds__(256) k_attn_out(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int h = blockIdx.x, part_id = blockIdx.z, nq = p.n_q, r = p.rv, hd = p.head_dim;
  const int qpk = nq / p.n_kv, q0 = h * qpk;
  const int k = (int)jb.metav[ISKV_META_K];
  extern __shared__ float sm[];
  float *w = sm;                        // [qpk][lslice]
  float *pe = w + (size_t)qpk * r;      // [qpk][AO_ROWS]
  float *part = pe + qpk * AO_ROWS;     // [NS][qpk][hd] partial outputs of the thread groups
  __shared__ float mass[8];
  const int tid = threadIdx.x, f = tid % hd, grp = tid / hd;
  const int NS = blockDim.x / hd;
  // This part's coordinates [la, lb) and exact rows [ea, eb).
  const int lsz = (k + AO_SPLIT - 1) / AO_SPLIT, la = min(k, part_id * lsz), lb = min(k, la + lsz);
  const int64_t esz = (jb.n_vex + AO_SPLIT - 1) / AO_SPLIT;
  const int64_t ea = min64(jb.n_vex, part_id * esz), eb = min64(jb.n_vex, ea + esz);
  const int nl = lb - la;
  for (int e = tid; e < qpk * nl; e += blockDim.x) {
    const int g = p.tc_values ? e % qpk : e / nl, li = p.tc_values ? e / qpk : e % nl;
    const int l = la + li;
    float acc = 0.f;
    for (int c = 0; c < p.nchunk; ++c)
      acc += p.tc_values ? jb.wpart[((size_t)c * r + l) * 64 + q0 + g]
                         : jb.wpart[((size_t)c * nq + q0 + g) * r + l];
    w[g * r + li] = acc * jb.sv[l];
  }
  if (tid < qpk) {
    float m = 0.f;
    if (part_id == 0)
      for (int c = 0; c < p.nblk; ++c) m += jb.mpart[(size_t)c * nq + q0 + tid];
    mass[tid] = m;
  }
  __syncthreads();
  float acc[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) acc[g] = 0.f;
  // Compressed part: feature f of the head over this part's coordinates, split by thread group.
  const TS *B = static_cast<const TS *>(jb.Bv) + (size_t)(h * hd + f) * r + la;
#pragma unroll 4
  for (int li = grp; li < nl; li += NS) {
    const float b = to_f<TS>(B[li]);
#pragma unroll
    for (int g = 0; g < 8; ++g)
      if (g < qpk) acc[g] = fmaf(b, w[g * r + li], acc[g]);
  }
  // Exact values of this part, in staged batches; the thread groups take rows in turn.
  const TE *V = static_cast<const TE *>(jb.vex) + h * hd + f;
  const float *S = jb.S;
  const int64_t nt = jb.n_total;
  for (int64_t e0 = ea; e0 < eb; e0 += AO_ROWS) {
    const int ne = (int)min64(AO_ROWS, eb - e0);
    __syncthreads();
    for (int e = tid; e < qpk * ne; e += blockDim.x) {
      const int g = e / ne, i = e % ne;
      const int64_t pos = jb.vexpos[e0 + i];
      float pv = 0.f;
      if (pos >= 0 && pos < nt)
        pv = __expf(S[(size_t)(q0 + g) * nt + pos] - jb.stats[2 * (q0 + g)]) *
             jb.stats[2 * (q0 + g) + 1];
      else if (g == 0)
        record_status(jb.metav, ISKV_ERR_SHAPE);
      pe[g * AO_ROWS + i] = pv;
    }
    __syncthreads();
    if (tid < qpk) {
      float m = 0.f;
      for (int i = 0; i < ne; ++i) m += pe[tid * AO_ROWS + i];
      mass[tid] += m;
    }
#pragma unroll 4
    for (int i = grp; i < ne; i += NS) {
      const float v = to_f<TE>(V[(size_t)(e0 + i) * p.d]);
#pragma unroll
      for (int g = 0; g < 8; ++g)
        if (g < qpk) acc[g] = fmaf(pe[g * AO_ROWS + i], v, acc[g]);
    }
  }
#pragma unroll
  for (int g = 0; g < 8; ++g)
    if (g < qpk) part[(grp * qpk + g) * hd + f] = acc[g];
  __syncthreads();
  float *op = jb.opart + (size_t)part_id * nq * hd;
  for (int e = tid; e < qpk * hd; e += blockDim.x) {
    const int g = e / hd, ff = e % hd;
    float o = 0.f;
    for (int t = 0; t < NS; ++t) o += part[(t * qpk + g) * hd + ff];
    op[(size_t)(q0 + g) * hd + ff] = o;
  }
  if (tid < qpk) jb.omass[(size_t)part_id * nq + q0 + tid] = mass[tid];
}

// Sum of the AO_SPLIT parts in order, and the probability-mass check per query head.
__global__ void __launch_bounds__(256) k_attn_final(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int nq = p.n_q, hd = p.head_dim;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < nq * hd; e += gridDim.x * blockDim.x) {
    float o = 0.f;
    for (int s = 0; s < AO_SPLIT; ++s) o += jb.opart[(size_t)s * nq * hd + e];
    jb.out[e] = o;
    if (e % hd == 0) {
      const int j = e / hd;
      float m = 0.f;
      for (int s = 0; s < AO_SPLIT; ++s) m += jb.omass[(size_t)s * nq + j];
      if (!(fabsf(m - 1.f) <= 1e-3f)) record_status(jb.metav, ISKV_ERR_SHAPE);
    }
  }
}

cudaError_t launch_attn_out(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  const int qpk = p.n_q / p.n_kv;
  if (qpk > 8) return cudaErrorInvalidValue;
  const int ns = 256 / p.head_dim > 0 ? 256 / p.head_dim : 1;  // thread groups
  const size_t smem = sizeof(float) * ((size_t)qpk * p.rv + (size_t)qpk * AO_ROWS +
                                       (size_t)ns * qpk * p.head_dim);
  const dim3 g(p.n_kv, p.count, AO_SPLIT);
  const int nth = ns * p.head_dim;
  cudaError_t e = cudaSuccess;
  with_dtype(p.storage, [&](auto ts) {
    with_dtype(p.exact_dtype, [&](auto te) {
      auto kern = k_attn_out<decltype(ts), decltype(te)>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) kern<<<g, nth, smem, s>>>(jobs, p);
    });
  });
  if (e != cudaSuccess) return e;
  k_attn_final<<<dim3(4, p.count), 256, 0, s>>>(jobs, p);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace iskv
