// Per-step reconstruction (iS-KV reading notes, Algorithm 3 steps 7-8): compressed row i of a
// history is (U[i] * sigma) B^T, written to its original position pos[i]; exact rows are copied to
// their own positions; keys are rotated by their own position with rotate-half RoPE (angles
// reduced in float64, rope.cuh).
#include "profiling.h"
#include "recon.h"
#include "rope.cuh"

namespace iskv {

// ------------------------------------------------------------------------------------------------
// CUDA-core path (float32 storage, and any storage when the tensor-core path is not selected).
// Tile: 32 rows x one head; thread = (row, pair group); each thread owns pairs (c, c + hd/2).
constexpr int RRM = 32, RBK = 16;

template <typename TS, typename TO>
__global__ void __launch_bounds__(256) k_recon_ffma(const ReconJob *jobs, ReconParams p) {
  const ReconJob &jb = jobs[blockIdx.z];
  const int64_t n = jb.meta[ISKV_META_N];
  const int k = (int)jb.meta[ISKV_META_K];
  const int i0 = blockIdx.x * RRM;
  if (i0 >= n) return;
  const int h = blockIdx.y, hd = p.head_dim, half = hd / 2, r = p.r, d = p.d;
  __shared__ float Us[RBK][RRM + 1];
  __shared__ float Bs[RBK][256 + 1];
  __shared__ double invf[128];
  const int tid = threadIdx.x;
  if (jb.apply_rope)
    for (int j = tid; j < half; j += 256) invf[j] = rope_inv_freq(j, hd, log(p.theta));
  __syncthreads();
  const TS *U = static_cast<const TS *>(jb.U);
  const TS *B = static_cast<const TS *>(jb.B);
  const float *sg = jb.sigma;
  const int row = tid / 8, g = tid % 8;
  constexpr int HPMAX = 16;  // pairs per thread for head_dim <= 256
  float lo[HPMAX], hi[HPMAX];
#pragma unroll
  for (int u = 0; u < HPMAX; ++u) lo[u] = hi[u] = 0.f;
  for (int l0 = 0; l0 < k; l0 += RBK) {
    for (int e = tid; e < RRM * RBK; e += 256) {
      const int i = e / RBK, ll = e % RBK;
      Us[ll][i] = (i0 + i < n && l0 + ll < k) ? to_f<TS>(U[(size_t)(i0 + i) * r + l0 + ll]) : 0.f;
    }
    for (int e = tid; e < hd * RBK; e += 256) {
      const int c = e / RBK, ll = e % RBK;
      const int l = l0 + ll;
      Bs[ll][c] = l < k ? sg[l] * to_f<TS>(B[(size_t)(h * hd + c) * r + l]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int ll = 0; ll < RBK; ++ll) {
      const float a = Us[ll][row];
#pragma unroll
      for (int u = 0; u < HPMAX; ++u) {
        const int c = g + 8 * u;
        if (c < half) {
          lo[u] = fmaf(a, Bs[ll][c], lo[u]);
          hi[u] = fmaf(a, Bs[ll][c + half], hi[u]);
        }
      }
    }
    __syncthreads();
  }
  const int64_t gi = i0 + row;
  if (gi >= n) return;
  const int64_t ps = jb.pos[gi];
  if (ps < 0 || ps >= jb.n_total) {  // a position outside the output: skip and flag
    if (g == 0) record_status(jb.meta, ISKV_ERR_SHAPE);
    return;
  }
  TO *out = static_cast<TO *>(jb.out) + (size_t)ps * d + (size_t)h * hd;
#pragma unroll
  for (int u = 0; u < HPMAX; ++u) {
    const int c = g + 8 * u;
    if (c >= half) continue;
    float x1 = lo[u], x2 = hi[u];
    if (jb.apply_rope) {
      float cs, sn;
      rope_sincos(ps, invf[c], cs, sn);
      const float y1 = x1 * cs - x2 * sn, y2 = x2 * cs + x1 * sn;
      x1 = y1;
      x2 = y2;
    }
    store_checked(&out[c], x1, jb.meta);
    store_checked(&out[c + half], x2, jb.meta);
  }
}

// Eight consecutive elements as floats (16-byte aligned source / destination).
ISKV_DEV void load8(const __nv_bfloat16 *p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
ISKV_DEV void load8(const __half *p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
ISKV_DEV void load8(const float *p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
ISKV_DEV void store8(__nv_bfloat16 *p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
ISKV_DEV void store8(float *p, const float (&v)[8]) {
  reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
// fp16: finite values beyond 65504 become infinities; that is recorded as ISKV_ERR_NONFINITE.
ISKV_DEV void store8(__half *p, const float (&v)[8], int64_t *meta) {
  uint32_t w[4];
  bool over = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
    over |= (__hisinf(h.x) && isfinite(v[2 * i])) || (__hisinf(h.y) && isfinite(v[2 * i + 1]));
    w[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  if (over) record_status(meta, ISKV_ERR_NONFINITE);
  *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
template <typename T>
ISKV_DEV void store8(T *p, const float (&v)[8], int64_t *) { store8(p, v); }

// Exact rows: copy (and rotate) exact_rows[e] to out[exact_pos[e]]. Thread = (row, head, group of
// V consecutive pairs); consecutive threads take consecutive groups of a head, so loads and stores
// are contiguous. V = 8 moves 16-byte vectors (head_dim a multiple of 16, rows 16-byte aligned).
template <typename TE, typename TO, int V>
__global__ void __launch_bounds__(256) k_recon_exact(const ReconJob *jobs, ReconParams p) {
  const ReconJob &jb = jobs[blockIdx.y];
  const int hd = p.head_dim, half = hd / 2, d = p.d, H = p.n_heads;
  __shared__ double invf[128];
  if (jb.apply_rope) {
    const double lt = log(p.theta);
    for (int j = threadIdx.x; j < half; j += blockDim.x) invf[j] = rope_inv_freq(j, hd, lt);
  }
  __syncthreads();
  const int groups = half / V, per_row = H * groups;
  const int64_t nwork = jb.n_exact * (int64_t)per_row;
  const TE *X = static_cast<const TE *>(jb.exact_rows);
  TO *out = static_cast<TO *>(jb.out);
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < nwork;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = t / per_row;
    const int rem = (int)(t - e * per_row);
    const int h = rem / groups, c = (rem - h * groups) * V;
    const int64_t ps = jb.exact_pos[e];
    if (ps < 0 || ps >= jb.n_total) {
      record_status(jb.meta, ISKV_ERR_SHAPE);
      continue;
    }
    const TE *src = X + (size_t)e * d + h * hd + c;
    TO *dst = out + (size_t)ps * d + h * hd + c;
    float x1[V], x2[V];
    if constexpr (V == 8) {
      load8(src, x1);
      load8(src + half, x2);
    } else {
      x1[0] = to_f<TE>(src[0]);
      x2[0] = to_f<TE>(src[half]);
    }
    if (jb.apply_rope) {
#pragma unroll
      for (int i = 0; i < V; ++i) {
        float cs, sn;
        rope_sincos(ps, invf[c + i], cs, sn);
        const float y1 = x1[i] * cs - x2[i] * sn, y2 = x2[i] * cs + x1[i] * sn;
        x1[i] = y1;
        x2[i] = y2;
      }
    }
    if constexpr (V == 8) {
      store8(dst, x1, jb.meta);
      store8(dst + half, x2, jb.meta);
    } else {
      store_checked(&dst[0], x1[0], jb.meta);
      store_checked(&dst[half], x2[0], jb.meta);
    }
  }
}

template <typename TS, typename TO>
static cudaError_t recon_ffma_t(const ReconJob *jobs, const ReconParams &p, cudaStream_t s) {
  const dim3 g((unsigned)((p.n_cap_max + RRM - 1) / RRM), p.n_heads, p.count);
  k_recon_ffma<TS, TO><<<g, 256, 0, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_recon_compressed_ffma(const ReconJob *jobs, const ReconParams &p,
                                         cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  with_dtype(p.storage, [&](auto ts) {
    with_dtype(p.out_dtype, [&](auto to) {
      e = recon_ffma_t<decltype(ts), decltype(to)>(jobs, p, s);
    });
  });
  return e;
}

cudaError_t launch_recon_compressed(const ReconJob *jobs, const ReconParams &p, cudaStream_t s) {
  return launch_recon_compressed_ffma(jobs, p, s);
}

cudaError_t launch_recon_exact(const ReconJob *jobs, const ReconParams &p, int64_t max_exact,
                               cudaStream_t s) {
  if (max_exact <= 0) return cudaSuccess;
  const int V = p.exact_vec ? 8 : 1;
  const int64_t work = max_exact * (int64_t)p.n_heads * (p.head_dim / 2 / V);
  const unsigned gx = (unsigned)((work + 255) / 256 < 4096 ? (work + 255) / 256 : 4096);
  const dim3 g(gx, p.count);
  with_dtype(p.exact_dtype, [&](auto te) {
    with_dtype(p.out_dtype, [&](auto to) {
      using TE = decltype(te);
      using TO = decltype(to);
      if (V == 8) k_recon_exact<TE, TO, 8><<<g, 256, 0, s>>>(jobs, p);
      else k_recon_exact<TE, TO, 1><<<g, 256, 0, s>>>(jobs, p);
    });
  });
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace iskv
