// Prompt-block protection (iS-KV reading notes, Section 3.1 and Algorithm 1 steps 2-4).
//
//   score[h][j] = min over the tokens t of block j of cos(k_t^h, mean_j^h)   (float64)
//   per head: the per_head lowest (score, j) among the full blocks before the suffix
//   P_K = union of picked blocks' tokens + suffix (last suffix_blocks full blocks + partial tail)
//   P_V = { q in [0, L) : |p - q| <= v_radius for some p in P_K }
//
// Kernels: block scores (one warp per (head, block)), an exact radix select per head (one CTA
// per head; 8 passes of 8-bit digits over an order-preserving 64-bit key, ties taken in block
// order), and a three-phase scan that compacts P_K and P_V.
#include "profiling.h"
#include "select.h"

namespace iskv {

SelectWsLayout select_ws_layout(int64_t L, int H, int block) {
  SelectWsLayout s;
  const int64_t nb = L / block;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  s.scores = take(sizeof(double) * (size_t)H * (nb > 0 ? nb : 1));
  s.blkflag = take((size_t)(nb > 0 ? nb : 1));
  s.prot = take((size_t)L);
  s.near = take((size_t)L);
  s.cntK = take(sizeof(int32_t) * (size_t)L);
  s.cntV = take(sizeof(int32_t) * (size_t)L);
  const int64_t nchunks = (L + SCAN_CHUNK - 1) / SCAN_CHUNK;
  s.chunk = take(sizeof(int32_t) * (size_t)(nchunks + 1));
  s.total = o;
  return s;
}

// ---------------------------------------------------------------------------------------------
template <typename TK>
__global__ void k_block_scores(const TK *keys, int64_t n_cand, int H, int hd, int block,
                               double *scores) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  if (gw >= n_cand * H) return;
  const int h = (int)(gw % H);
  const int64_t j = gw / H;
  constexpr int EMAX = 8;  // head_dim <= 256
  double mean[EMAX];
#pragma unroll
  for (int u = 0; u < EMAX; ++u) mean[u] = 0.0;
  for (int t = 0; t < block; ++t) {
    const TK *kt = keys + ((size_t)(j * block + t) * H + h) * hd;
#pragma unroll
    for (int u = 0; u < EMAX; ++u) {
      const int e = lane + 32 * u;
      if (e < hd) mean[u] += (double)to_f<TK>(kt[e]);
    }
  }
  double mn2 = 0.0;
#pragma unroll
  for (int u = 0; u < EMAX; ++u) {
    mean[u] /= (double)block;
    mn2 = fma(mean[u], mean[u], mn2);
  }
  const double mn = sqrt(warp_sum(mn2));
  double best = 0.0;
  for (int t = 0; t < block; ++t) {
    const TK *kt = keys + ((size_t)(j * block + t) * H + h) * hd;
    double dot = 0.0, k2 = 0.0;
#pragma unroll
    for (int u = 0; u < EMAX; ++u) {
      const int e = lane + 32 * u;
      if (e < hd) {
        const double v = (double)to_f<TK>(kt[e]);
        dot = fma(v, mean[u], dot);
        k2 = fma(v, v, k2);
      }
    }
    dot = warp_sum(dot);
    k2 = warp_sum(k2);
    const double cs = dot / fmax(sqrt(k2) * mn, 1e-30);
    best = t == 0 ? cs : fmin(best, cs);
  }
  if (lane == 0) scores[(size_t)h * n_cand + j] = best;
}

// Fast path for 8-token blocks of 128-dimensional heads: one warp per (head, block), lane l holds
// dimensions 4l .. 4l+3 of all 8 tokens (one 8- or 16-byte load per token). The 16 per-token
// sums (dot with the mean, squared norm) are reduced together by a transposed butterfly: at each
// of 4 levels a lane keeps half of its values and adds the partner's other half, so after 4 + 1
// shuffle levels lanes 4t, 4t+1 hold token t's dot and lanes 4t+2, 4t+3 its squared norm.
ISKV_DEV void load4(const __nv_bfloat16 *p, double (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
ISKV_DEV void load4(const float *p, double (&v)[4]) {
  const float4 f = *reinterpret_cast<const float4 *>(p);
  v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

template <typename TK>
__global__ void __launch_bounds__(256) k_block_scores_8x128(const TK *keys, int64_t n_cand, int H,
                                                            double *scores) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  if (gw >= n_cand * H) return;  // whole warps
  const int h = (int)(gw % H);
  const int64_t j = gw / H;
  double x[8][4];
#pragma unroll
  for (int t = 0; t < 8; ++t) load4(keys + ((size_t)(j * 8 + t) * H + h) * 128 + 4 * lane, x[t]);
  double mean[4], mn2 = 0.0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    double m = 0.0;
#pragma unroll
    for (int t = 0; t < 8; ++t) m += x[t][u];
    mean[u] = m / 8.0;
    mn2 = fma(mean[u], mean[u], mn2);
  }
  const double mn = sqrt(warp_sum(mn2));
  // v[2t] = partial dot of token t with the mean, v[2t+1] = partial squared norm of token t.
  double v[16];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    double dt = 0.0, k2 = 0.0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dt = fma(x[t][u], mean[u], dt);
      k2 = fma(x[t][u], x[t][u], k2);
    }
    v[2 * t] = dt;
    v[2 * t + 1] = k2;
  }
  // Transposed butterfly over lane bits 4, 3, 2, 1: value index bits 3, 2, 1, 0.
#pragma unroll
  for (int lev = 0; lev < 4; ++lev) {
    const int half = 8 >> lev;                // values kept after this level
    const int bit = 16 >> lev;                // lane bit deciding which half is kept
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < half) {
        const double send = upper ? v[i] : v[i + half];
        const double keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
      }
    }
  }
  const double tot = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);  // lanes 2i, 2i+1: value i
  // Lane 4t: dot of token t; lane 4t + 2: its squared norm.
  const double k2t = __shfl_down_sync(0xffffffffu, tot, 2);
  double cs = 0.0;
  if ((lane & 3) == 0) cs = tot / fmax(sqrt(k2t) * mn, 1e-30);
  // Minimum over the 8 tokens (lanes 0, 4, ..., 28).
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    const double other = __shfl_xor_sync(0xffffffffu, cs, o);
    cs = fmin(cs, other);
  }
  if (lane == 0) scores[(size_t)h * n_cand + j] = cs;
}

// Order-preserving map from a finite double to uint64 (-0 is folded onto +0).
ISKV_DEV unsigned long long order_key(double v) {
  if (v == 0.0) v = 0.0;
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Block-wide exclusive scan of one int per thread (blockDim = 1024). Returns the exclusive prefix;
// *total receives the block sum.
ISKV_DEV int block_excl_scan(int v, int *total) {
  __shared__ int wsum[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;
  }
  __syncthreads();
  const int before = (warp > 0 ? wsum[warp - 1] : 0) + x - v;
  *total = wsum[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

constexpr int SEL_NTH = 1024;

__global__ void __launch_bounds__(SEL_NTH) k_select_head(const double *scores, int64_t n_cand,
                                                         int per_head, int32_t *head_blocks,
                                                         int64_t *counts, uint8_t *blkflag) {
  const int h = blockIdx.x, tid = threadIdx.x;
  const double *sc = scores + (size_t)h * n_cand;
  const int take_n = (int)(n_cand < per_head ? n_cand : per_head);
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ long long s_need;
  unsigned long long T = ~0ull;
  long long need = take_n;
  if (take_n < n_cand) {
    if (tid == 0) { s_prefix = 0ull; s_need = take_n; }
    __syncthreads();
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      const unsigned long long hi_mask = pass == 0 ? 0ull : (~0ull << (shift + 8));
      for (int i = tid; i < 256; i += SEL_NTH) hist[i] = 0u;
      __syncthreads();
      const unsigned long long pre = s_prefix;
      for (int64_t j = tid; j < n_cand; j += SEL_NTH) {
        const unsigned long long key = order_key(sc[j]);
        if ((key & hi_mask) == pre) atomicAdd(&hist[(key >> shift) & 0xffu], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        long long nd = s_need;
        int bsel = 0;
        for (; bsel < 256; ++bsel) {
          if ((long long)hist[bsel] >= nd) break;
          nd -= hist[bsel];
        }
        s_prefix = pre | ((unsigned long long)bsel << shift);
        s_need = nd;
      }
      __syncthreads();
    }
    T = s_prefix;
    need = s_need;
  }
  // Collect in block order: key < T, or key == T among the first `need` such blocks.
  int written = 0, eq_seen = 0;
  for (int64_t base = 0; base < n_cand; base += SEL_NTH) {
    const int64_t j = base + tid;
    unsigned long long key = 0;
    bool inb = j < n_cand;
    if (inb) key = order_key(sc[j]);
    const int eq = (inb && key == T) ? 1 : 0;
    int eq_total;
    const int eq_before = block_excl_scan(eq, &eq_total);
    const bool take = inb && (key < T || (eq && eq_seen + eq_before < need));
    int tk_total;
    const int tk_before = block_excl_scan(take ? 1 : 0, &tk_total);
    if (take && written + tk_before < per_head) {
      head_blocks[(size_t)h * per_head + written + tk_before] = (int32_t)j;
      blkflag[j] = 1;
    }
    written += tk_total;
    eq_seen += eq_total;
  }
  for (int i = written + tid; i < per_head; i += SEL_NTH) head_blocks[(size_t)h * per_head + i] = -1;
  if (tid == 0) counts[2 + h] = written;
}

__global__ void k_mark_protected(const uint8_t *blkflag, int64_t L, int block, int64_t n_cand,
                                 uint8_t *prot) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < L;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = t / block;
    prot[t] = (j >= n_cand) ? 1 : blkflag[j];
  }
}

// Three-phase inclusive scan of uint8 flags into int32 counts.
__global__ void k_scan_chunk_sums(const uint8_t *f, int64_t L, int32_t *chunk) {
  const int64_t c = blockIdx.x;
  const int64_t b0 = c * SCAN_CHUNK;
  int s = 0;
  for (int64_t i = b0 + threadIdx.x; i < b0 + SCAN_CHUNK && i < L; i += blockDim.x) s += f[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __shared__ int ws[32];
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += ws[w];
    chunk[c] = t;
  }
}

__global__ void __launch_bounds__(SEL_NTH) k_scan_chunk_offsets(int32_t *chunk, int64_t nchunks) {
  int carry = 0;
  for (int64_t base = 0; base < nchunks; base += SEL_NTH) {
    const int64_t i = base + threadIdx.x;
    const int v = i < nchunks ? chunk[i] : 0;
    int tot;
    const int ex = block_excl_scan(v, &tot);
    if (i < nchunks) chunk[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) chunk[nchunks] = carry;
}

__global__ void __launch_bounds__(SEL_NTH) k_scan_apply(const uint8_t *f, int64_t L,
                                                        const int32_t *chunk, int32_t *cnt) {
  const int64_t c = blockIdx.x;
  const int64_t b0 = c * SCAN_CHUNK;
  int carry = chunk[c];
  for (int64_t base = b0; base < b0 + SCAN_CHUNK && base < L; base += SEL_NTH) {
    const int64_t i = base + threadIdx.x;
    const int v = i < L ? f[i] : 0;
    int tot;
    const int ex = block_excl_scan(v, &tot);
    if (i < L) cnt[i] = carry + ex + v;
    carry += tot;
  }
}

static cudaError_t scan_u8(const uint8_t *f, int64_t L, int32_t *chunk, int32_t *cnt,
                           cudaStream_t s) {
  const int64_t nchunks = (L + SCAN_CHUNK - 1) / SCAN_CHUNK;
  k_scan_chunk_sums<<<(unsigned)nchunks, 256, 0, s>>>(f, L, chunk);
  k_scan_chunk_offsets<<<1, SEL_NTH, 0, s>>>(chunk, nchunks);
  k_scan_apply<<<(unsigned)nchunks, SEL_NTH, 0, s>>>(f, L, chunk, cnt);
  count_launches(3);
  return cudaGetLastError();
}

__global__ void k_compact_pk_near(const uint8_t *prot, const int32_t *cntK, int64_t L,
                                  int v_radius, int32_t *pk_out, uint8_t *nearf,
                                  int64_t *counts) {
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < L;
       q += (int64_t)gridDim.x * blockDim.x) {
    if (prot[q]) pk_out[cntK[q] - 1] = (int32_t)q;
    const int64_t hi = q + v_radius < L - 1 ? q + v_radius : L - 1;
    const int64_t lo = q - v_radius - 1;
    const int c = cntK[hi] - (lo >= 0 ? cntK[lo] : 0);
    nearf[q] = c > 0 ? 1 : 0;
    if (q == L - 1) counts[0] = cntK[q];
  }
}

__global__ void k_compact_pv(const uint8_t *nearf, const int32_t *cntV, int64_t L, int32_t *pv_out,
                             int64_t *counts) {
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < L;
       q += (int64_t)gridDim.x * blockDim.x) {
    if (nearf[q]) pv_out[cntV[q] - 1] = (int32_t)q;
    if (q == L - 1) counts[1] = cntV[q];
  }
}

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s) {
  const SelectWsLayout W = select_ws_layout(a.L, a.H, a.block);
  char *ws = static_cast<char *>(a.ws);
  double *scores = reinterpret_cast<double *>(ws + W.scores);
  uint8_t *blkflag = reinterpret_cast<uint8_t *>(ws + W.blkflag);
  uint8_t *prot = reinterpret_cast<uint8_t *>(ws + W.prot);
  uint8_t *nearf = reinterpret_cast<uint8_t *>(ws + W.near);
  int32_t *cntK = reinterpret_cast<int32_t *>(ws + W.cntK);
  int32_t *cntV = reinterpret_cast<int32_t *>(ws + W.cntV);
  int32_t *chunk = reinterpret_cast<int32_t *>(ws + W.chunk);
  const int64_t nb = a.L / a.block;
  const int64_t n_cand = nb > a.suffix_blocks ? nb - a.suffix_blocks : 0;
  cudaError_t e;
  if (n_cand > 0) {
    e = cudaMemsetAsync(blkflag, 0, (size_t)n_cand, s);
    if (e != cudaSuccess) return e;
    const int64_t warps = n_cand * a.H;
    const unsigned g = (unsigned)((warps * 32 + 255) / 256);
    const bool fast = a.block == 8 && a.hd == 128 &&
                      reinterpret_cast<uintptr_t>(a.keys) % (a.k_dtype == ISKV_BF16 ? 8 : 16) == 0;
    if (fast && a.k_dtype == ISKV_BF16)
      k_block_scores_8x128<<<g, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(a.keys), n_cand,
                                             a.H, scores);
    else if (fast)
      k_block_scores_8x128<<<g, 256, 0, s>>>(static_cast<const float *>(a.keys), n_cand, a.H,
                                             scores);
    else if (a.k_dtype == ISKV_BF16)
      k_block_scores<<<g, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(a.keys), n_cand, a.H,
                                       a.hd, a.block, scores);
    else
      k_block_scores<<<g, 256, 0, s>>>(static_cast<const float *>(a.keys), n_cand, a.H, a.hd,
                                       a.block, scores);
    count_launches(1);
  }
  k_select_head<<<a.H, SEL_NTH, 0, s>>>(scores, n_cand, a.per_head, a.head_blocks, a.counts,
                                        blkflag);
  const unsigned gL = (unsigned)((a.L + 255) / 256 < 65535 ? (a.L + 255) / 256 : 65535);
  k_mark_protected<<<gL, 256, 0, s>>>(blkflag, a.L, a.block, n_cand, prot);
  count_launches(2);
  e = scan_u8(prot, a.L, chunk, cntK, s);
  if (e != cudaSuccess) return e;
  k_compact_pk_near<<<gL, 256, 0, s>>>(prot, cntK, a.L, a.v_radius, a.pk_out, nearf, a.counts);
  count_launches(1);
  e = scan_u8(nearf, a.L, chunk, cntV, s);
  if (e != cudaSuccess) return e;
  k_compact_pv<<<gL, 256, 0, s>>>(nearf, cntV, a.L, a.pv_out, a.counts);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace iskv
