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

// Scale, rotate and dot one key of KV head h, held as pairs (lo = k[j], hi = k[j + hd/2]) for
// j = lane + 32 t, with every query head of its group; lane 0 writes the scores.
template <int T>
ISKV_DEV void score_key(const AttnJob &jb, const AttnParams &p, int h, int64_t pos,
                        const float (&lo)[T], const float (&hi)[T], const double *invf) {
  const int lane = threadIdx.x & 31, half = p.head_dim / 2, qpk = p.n_q / p.n_kv;
  float rl[T], rh[T];
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int j = lane + 32 * t;
    rl[t] = rh[t] = 0.f;
    if (j < half) {
      float c, s;
      rope_sincos(pos, invf[j], c, s);
      rl[t] = lo[t] * c - hi[t] * s;
      rh[t] = hi[t] * c + lo[t] * s;
    }
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
  const int d = p.d, r = p.r, hd = p.head_dim, half = hd / 2;
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
    for (int h = warp; h < p.n_kv; h += blockDim.x >> 5) {
      float lo[4], hi[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int j = lane + 32 * t;
        lo[t] = j < half ? krow[h * hd + j] : 0.f;
        hi[t] = j < half ? krow[h * hd + j + half] : 0.f;
      }
      score_key<4>(jb, p, h, pos, lo, hi, invf);
    }
  }
}

cudaError_t launch_attn_scores_ffma(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  const int gx = (int)((p.n_cap_max + 7) / 8);
  const size_t smem = sizeof(float) * (size_t)(p.r + p.d);
  if (gx < 1) return cudaSuccess;
  if (p.storage == ISKV_BF16)
    k_attn_scores_ffma<__nv_bfloat16><<<dim3(gx, p.count), 256, smem, s>>>(jobs, p);
  else
    k_attn_scores_ffma<float><<<dim3(gx, p.count), 256, smem, s>>>(jobs, p);
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
  for (int h = 0; h < p.n_kv; ++h) {
    float lo[4], hi[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int j = lane + 32 * t;
      lo[t] = j < half ? to_f<TE>(x[h * hd + j]) : 0.f;
      hi[t] = j < half ? to_f<TE>(x[h * hd + j + half]) : 0.f;
    }
    score_key<4>(jb, p, h, pos, lo, hi, invf);
  }
}

cudaError_t launch_attn_scores_exact(const AttnJob *jobs, const AttnParams &p, int64_t max_kex,
                                     cudaStream_t s) {
  if (max_kex <= 0) return cudaSuccess;
  const dim3 g((unsigned)((max_kex + 7) / 8), p.count);
  if (p.exact_dtype == ISKV_BF16)
    k_attn_scores_exact<__nv_bfloat16><<<g, 256, 0, s>>>(jobs, p);
  else
    k_attn_scores_exact<float><<<g, 256, 0, s>>>(jobs, p);
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
// Compressed values, mixed in coordinate space: block c of a job sums P_j(pos_v[i]) U_v[i] over its
// ATTN_CHUNK rows for every query head j (one column of U per thread, one accumulator per head),
// 64 rows at a time with the probabilities staged in shared memory.
constexpr int AV_SUB = 64;

template <typename TS>
__global__ void __launch_bounds__(256) k_attn_values(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int c = blockIdx.x, nq = p.n_q, r = p.r;
  const int64_t n = jb.metav[ISKV_META_N];
  const int k = (int)jb.metav[ISKV_META_K];
  __shared__ float P[AV_SUB][ATTN_MAX_Q];
  __shared__ float mass[ATTN_MAX_Q];
  const TS *U = static_cast<const TS *>(jb.Uv);
  const int64_t i0 = (int64_t)c * ATTN_CHUNK, i1 = min64(n, i0 + ATTN_CHUNK);
  if (threadIdx.x < ATTN_MAX_Q) mass[threadIdx.x] = 0.f;
  for (int l0 = 0; l0 < r; l0 += blockDim.x) {
    const int l = l0 + threadIdx.x;
    float acc[ATTN_MAX_Q];
#pragma unroll
    for (int j = 0; j < ATTN_MAX_Q; ++j) acc[j] = 0.f;
    for (int64_t s0 = i0; s0 < i1; s0 += AV_SUB) {
      const int rows = (int)min64(AV_SUB, i1 - s0);
      __syncthreads();
      for (int e = threadIdx.x; e < AV_SUB * nq; e += blockDim.x) {
        const int ii = e / nq, j = e % nq;
        float pv = 0.f;
        if (ii < rows) {
          const int64_t pos = jb.posv[s0 + ii];
          if (pos >= 0 && pos < jb.n_total) {
            pv = __expf(jb.S[(size_t)j * jb.n_total + pos] - jb.stats[2 * j]) * jb.stats[2 * j + 1];
          } else if (j == 0) {
            record_status(jb.metav, ISKV_ERR_SHAPE);
          }
        }
        P[ii][j] = pv;
      }
      __syncthreads();
      if (l0 == 0 && threadIdx.x < nq) {
        float m = 0.f;
        for (int ii = 0; ii < rows; ++ii) m += P[ii][threadIdx.x];
        mass[threadIdx.x] += m;
      }
      if (l < k) {
        for (int ii = 0; ii < rows; ++ii) {
          const float u = to_f<TS>(U[(size_t)(s0 + ii) * r + l]);
#pragma unroll
          for (int j = 0; j < ATTN_MAX_Q; j += 4) {
            if (j >= nq) break;
            const float4 pv = *reinterpret_cast<const float4 *>(&P[ii][j]);
            acc[j] = fmaf(pv.x, u, acc[j]);
            acc[j + 1] = fmaf(pv.y, u, acc[j + 1]);
            acc[j + 2] = fmaf(pv.z, u, acc[j + 2]);
            acc[j + 3] = fmaf(pv.w, u, acc[j + 3]);
          }
        }
      }
    }
    if (l < r) {
      float *wp = jb.wpart + (size_t)c * nq * r;
#pragma unroll
      for (int j = 0; j < ATTN_MAX_Q; ++j)
        if (j < nq) wp[(size_t)j * r + l] = acc[j];
    }
  }
  __syncthreads();
  if (threadIdx.x < nq) jb.mpart[(size_t)c * nq + threadIdx.x] = mass[threadIdx.x];
}

cudaError_t launch_attn_values(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  if (p.storage == ISKV_BF16)
    k_attn_values<__nv_bfloat16><<<dim3(p.nchunk, p.count), 256, 0, s>>>(jobs, p);
  else
    k_attn_values<float><<<dim3(p.nchunk, p.count), 256, 0, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Output of one query head: o = B_v,h (sigma_v * sum_c wpart[c]) + sum_e P(pos_e) v_e[h], and the
// probability-mass check.
template <typename TS, typename TE>
__global__ void __launch_bounds__(256) k_attn_out(const AttnJob *jobs, AttnParams p) {
  const AttnJob &jb = jobs[blockIdx.y];
  const int qh = blockIdx.x, nq = p.n_q, r = p.r, hd = p.head_dim;
  const int h = qh / (nq / p.n_kv);
  const int k = (int)jb.metav[ISKV_META_K];
  extern __shared__ float sm[];
  float *w = sm;            // [r]
  float *pe = sm + r;       // [256] exact-row probabilities of the current batch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const float mx = jb.stats[2 * qh], inv = jb.stats[2 * qh + 1];
  for (int l = threadIdx.x; l < r; l += blockDim.x) {
    float acc = 0.f;
    if (l < k) {
      for (int c = 0; c < p.nchunk; ++c) acc += jb.wpart[((size_t)c * nq + qh) * r + l];
      acc *= jb.sv[l];
    }
    w[l] = acc;
  }
  float mass = 0.f;
  if (threadIdx.x == 0)
    for (int c = 0; c < p.nchunk; ++c) mass += jb.mpart[(size_t)c * nq + qh];
  __syncthreads();
  // Compressed part: o[f] = sum_l B[h hd + f][l] w[l], one warp per output feature at a time.
  const TS *B = static_cast<const TS *>(jb.Bv);
  float *o = jb.out + (size_t)qh * hd;
  float ofeat = 0.f;  // thread f < hd accumulates the exact part of feature f
  for (int f = warp; f < hd; f += nw) {
    float acc = 0.f;
    for (int l = lane; l < k; l += 32) acc = fmaf(to_f<TS>(B[(size_t)(h * hd + f) * r + l]), w[l], acc);
    acc = warp_sum(acc);
    if (lane == 0) o[f] = acc;
  }
  // Exact values.
  const TE *V = static_cast<const TE *>(jb.vex);
  for (int64_t e0 = 0; e0 < jb.n_vex; e0 += blockDim.x) {
    __syncthreads();
    const int64_t e = e0 + threadIdx.x;
    float pv = 0.f;
    if (e < jb.n_vex) {
      const int64_t pos = jb.vexpos[e];
      if (pos >= 0 && pos < jb.n_total)
        pv = __expf(jb.S[(size_t)qh * jb.n_total + pos] - mx) * inv;
      else
        record_status(jb.metav, ISKV_ERR_SHAPE);
    }
    pe[threadIdx.x] = pv;
    __syncthreads();
    const int ne = (int)min64(blockDim.x, jb.n_vex - e0);
    if (threadIdx.x < hd)
      for (int i = 0; i < ne; ++i)
        ofeat = fmaf(pe[i], to_f<TE>(V[(size_t)(e0 + i) * p.d + h * hd + threadIdx.x]), ofeat);
    if (threadIdx.x == 0)
      for (int i = 0; i < ne; ++i) mass += pe[i];
  }
  __syncthreads();  // the compressed part of o is written
  if (threadIdx.x < hd) o[threadIdx.x] += ofeat;
  if (threadIdx.x == 0 && !(fabsf(mass - 1.f) <= 1e-3f)) record_status(jb.metav, ISKV_ERR_SHAPE);
}

cudaError_t launch_attn_out(const AttnJob *jobs, const AttnParams &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)(p.r + 256);
  const bool sb = p.storage == ISKV_BF16, eb = p.exact_dtype == ISKV_BF16;
  const dim3 g(p.n_q, p.count);
  if (sb && eb) k_attn_out<__nv_bfloat16, __nv_bfloat16><<<g, 256, smem, s>>>(jobs, p);
  else if (sb) k_attn_out<__nv_bfloat16, float><<<g, 256, smem, s>>>(jobs, p);
  else if (eb) k_attn_out<float, __nv_bfloat16><<<g, 256, smem, s>>>(jobs, p);
  else k_attn_out<float, float><<<g, 256, smem, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace iskv
