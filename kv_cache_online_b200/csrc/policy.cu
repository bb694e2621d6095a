// Cache policy kernels (iS-KV reading notes, Section 3.1, Section 3.2, Algorithm 1 steps 5-7,
// Algorithm 3 steps 1-2 and 6): the prefill partition of one side's prompt rows into protected,
// live (unprotected initial-window) and compressed rows, the append of a decode row to the
// exact-row table, and the removal of a folded block from it.
#include "policy.h"
#include "profiling.h"

namespace iskv {
namespace {

// First index i in [0, n) with P[i] >= x (n when there is none).
ISKV_DEV int64_t lower_bound_pos(const int32_t *P, int64_t n, int64_t x) {
  int64_t lo = 0, hi = n;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(P + mid) < x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// The protected positions must be strictly ascending inside [0, L).
__global__ void k_prefill_check(const int32_t *P, int64_t n_p, int64_t L, int64_t *st) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_p; i += stride) {
    const int64_t p = P[i];
    if (p < 0 || p >= L || (i + 1 < n_p && p >= (int64_t)P[i + 1])) record_status(st, ISKV_ERR_ARG);
  }
}

// One warp per prompt row p. Its class and slot follow from c = #{protected positions < p}:
//   protected:             slot c of the protected rows;
//   inside the window:     live slot (p - edge) - #{protected positions in [edge, p)};
//   before the window:     compressed slot p - c.
// Slots are range-checked, so protected positions that break the ordering contract record an error
// instead of writing outside the table.
template <typename TX, typename TT>
__global__ void __launch_bounds__(256) k_prefill_partition(PrefillArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t edge = a.L - a.w;  // first position of the initial window
  const int64_t lbw = lower_bound_pos(a.P, a.n_p, edge);
  if (warp == 0 && lane == 0) a.st[0] = a.w - (a.n_p - lbw);
  const TX *X = static_cast<const TX *>(a.X);
  for (int64_t p = warp; p < a.L; p += nwarps) {
    const int64_t lb = lower_bound_pos(a.P, a.n_p, p);
    const TX *src = X + p * a.d;
    int64_t slot;
    bool exact = true;
    if (lb < a.n_p && (int64_t)a.P[lb] == p) {
      slot = lb;
    } else if (p >= edge) {
      slot = a.n_p + (p - edge) - (lb - lbw);
      if (slot < a.n_p || slot >= a.n_p + a.w) {
        if (lane == 0) record_status(a.st, ISKV_ERR_ARG);
        continue;
      }
    } else {
      exact = false;
      slot = p - lb;
      if (slot < 0 || slot >= edge) {
        if (lane == 0) record_status(a.st, ISKV_ERR_ARG);
        continue;
      }
    }
    if (exact) {
      TT *dst = static_cast<TT *>(a.rows) + slot * a.d;
      for (int c = lane; c < a.d; c += 32) store_checked<TT>(dst + c, to_f<TX>(src[c]), a.st);
      if (lane == 0) a.pos[slot] = (int32_t)p;
    } else {
      TX *dst = static_cast<TX *>(a.comp) + slot * a.d;
      for (int c = lane; c < a.d; c += 32) dst[c] = src[c];
      if (lane == 0) a.comp_pos[slot] = (int32_t)p;
    }
  }
}

// One CTA per table: the new row, converted to the table's element type, and its position.
template <typename TS, typename TT>
__global__ void __launch_bounds__(128) k_cache_append(const AppendJob *jobs, int d) {
  const AppendJob j = jobs[blockIdx.x];
  const TS *src = static_cast<const TS *>(j.src);
  TT *dst = static_cast<TT *>(j.dst);
  for (int c = threadIdx.x; c < d; c += blockDim.x) store_checked<TT>(dst + c, to_f<TS>(src[c]), j.meta);
  if (threadIdx.x == 0) *j.dst_pos = j.position;
}

// One CTA per table moves the remaining live rows down by `shift` rows. The source and destination
// overlap, so the CTA walks segments of at most `shift` rows' worth in ascending order: a segment
// is loaded into registers, the CTA synchronises, then stores it. A store never reaches an address
// that a later segment still has to load (those lie at least `shift` rows higher), and a load never
// reads one that an earlier segment stored.
constexpr int EV_THREADS = 256, EV_VEC = 4;

__global__ void __launch_bounds__(EV_THREADS) k_cache_evict(const EvictJob *jobs) {
  const EvictJob j = jobs[blockIdx.x];
  uint4 *rows = static_cast<uint4 *>(j.rows);
  const int64_t total = j.keep * j.row_bytes / 16;
  const int64_t shift = (int64_t)j.shift * j.row_bytes / 16;
  const int64_t seg = shift < (int64_t)EV_THREADS * EV_VEC ? shift : (int64_t)EV_THREADS * EV_VEC;
  for (int64_t s0 = 0; s0 < total; s0 += seg) {
    uint4 v[EV_VEC];
#pragma unroll
    for (int q = 0; q < EV_VEC; ++q) {
      const int64_t o = threadIdx.x + (int64_t)q * EV_THREADS;
      if (o < seg && s0 + o < total) v[q] = rows[s0 + o + shift];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < EV_VEC; ++q) {
      const int64_t o = threadIdx.x + (int64_t)q * EV_THREADS;
      if (o < seg && s0 + o < total) rows[s0 + o] = v[q];
    }
    __syncthreads();
  }
  const int64_t pseg = j.shift < EV_THREADS ? j.shift : EV_THREADS;
  for (int64_t s0 = 0; s0 < j.keep; s0 += pseg) {
    int32_t v = 0;
    const bool on = threadIdx.x < pseg && s0 + threadIdx.x < j.keep;
    if (on) v = j.pos[s0 + threadIdx.x + j.shift];
    __syncthreads();
    if (on) j.pos[s0 + threadIdx.x] = v;
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_prefill_partition(const PrefillArgs &a, cudaStream_t s) {
  if (a.n_p > 0) {
    const int64_t blocks = (a.n_p + 255) / 256;
    k_prefill_check<<<(unsigned)(blocks < 1184 ? blocks : 1184), 256, 0, s>>>(a.P, a.n_p, a.L, a.st);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.L == 0) return cudaSuccess;
  const int64_t blocks = (a.L + 7) / 8;  // 8 warps (rows) per CTA
  const unsigned grid = (unsigned)(blocks < 148 * 16 ? blocks : 148 * 16);
  with_dtype(a.x_dtype, [&](auto tx) {
    using TX = decltype(tx);
    with_dtype(a.t_dtype, [&](auto tt) {
      using TT = decltype(tt);
      k_prefill_partition<TX, TT><<<grid, 256, 0, s>>>(a);
    });
  });
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_cache_append(const AppendJob *jobs, int count, int d, int src_dtype,
                                int dst_dtype, cudaStream_t s) {
  with_dtype(src_dtype, [&](auto ts) {
    using TS = decltype(ts);
    with_dtype(dst_dtype, [&](auto tt) {
      using TT = decltype(tt);
      k_cache_append<TS, TT><<<count, 128, 0, s>>>(jobs, d);
    });
  });
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_cache_evict(const EvictJob *jobs, int count, cudaStream_t s) {
  k_cache_evict<<<count, EV_THREADS, 0, s>>>(jobs);
  count_launches(1);
  return cudaGetLastError();
}


// ------------------------------------------------------------------------------------------------
// Widening and narrowing of a history (the value side's first refit of a history that already
// holds compressed rows; Section 3.2 and Algorithm 3 step 3). Rows 0 .. n_cap - 1 are U's rows,
// rows n_cap .. n_cap + d - 1 are B's; one CTA per row walks it in 16-byte words.
__global__ void k_history_widen(WidenArgs a) {
  const int64_t row = blockIdx.x;
  const int64_t n = a.meta[ISKV_META_N];
  const bool is_u = row < a.n_cap;
  const int64_t i = is_u ? row : row - a.n_cap;
  const bool live = !is_u || row < n;  // U rows past n are zeroed (the workspace holds anything)
  const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const char *>(is_u ? a.U : a.B) +
                                                     (size_t)i * a.r * a.esz);
  uint4 *dst = reinterpret_cast<uint4 *>(static_cast<char *>(is_u ? a.Uw : a.Bw) +
                                         (size_t)i * a.rw * a.esz);
  const int wr = live ? a.r * a.esz / 16 : 0, ww = a.rw * a.esz / 16;
  for (int w = threadIdx.x; w < ww; w += blockDim.x) dst[w] = w < wr ? src[w] : make_uint4(0, 0, 0, 0);
  if (!live) return;
  if (is_u && threadIdx.x == 0) a.posw[i] = a.pos[i];
  if (row == 0) {
    for (int l = threadIdx.x; l < a.rw; l += blockDim.x) a.sigw[l] = l < a.r ? a.sigma[l] : 0.f;
    if (threadIdx.x < 4) a.metaw[threadIdx.x] = a.meta[threadIdx.x];
  }
}

__global__ void k_history_narrow(WidenArgs a) {
  const int64_t row = blockIdx.x;
  const int64_t n = a.metaw[ISKV_META_N];
  const bool is_u = row < a.n_cap;
  if (is_u && row >= n) return;
  const int64_t i = is_u ? row : row - a.n_cap;
  const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const char *>(is_u ? a.Uw : a.Bw) +
                                                     (size_t)i * a.rw * a.esz);
  uint4 *dst = reinterpret_cast<uint4 *>(static_cast<char *>(is_u ? a.U : a.B) +
                                         (size_t)i * a.r * a.esz);
  const int wr = a.r * a.esz / 16;
  for (int w = threadIdx.x; w < wr; w += blockDim.x) dst[w] = src[w];
  if (is_u && threadIdx.x == 0) a.pos[i] = a.posw[i];
  if (row == 0) {
    for (int l = threadIdx.x; l < a.r; l += blockDim.x) a.sigma[l] = a.sigw[l];
    if (threadIdx.x == 0) {
      const int64_t kw = a.metaw[ISKV_META_K];
      a.meta[ISKV_META_K] = kw < a.r ? kw : a.r;
      a.meta[ISKV_META_N] = n;
      a.meta[2] = a.metaw[2];
      a.meta[ISKV_META_STATUS] |= a.metaw[ISKV_META_STATUS];
    }
  }
}

cudaError_t launch_history_widen(const WidenArgs &a, cudaStream_t s) {
  k_history_widen<<<(unsigned)(a.n_cap + a.d), 128, 0, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_history_narrow(const WidenArgs &a, cudaStream_t s) {
  k_history_narrow<<<(unsigned)(a.n_cap + a.d), 128, 0, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Short last block of a prompt compression (Algorithm 1 step 7): padding before the fold, and the
// removal of the zero coordinate rows the padding appended.
__global__ void k_tail_pad(TailJob *jobs) {
  TailJob &j = jobs[blockIdx.x];
  if (threadIdx.x == 0) j.n0 = j.meta[ISKV_META_N];
  const int64_t words = j.row_bytes / 16;
  const uint4 *src = static_cast<const uint4 *>(j.src);
  uint4 *dst = static_cast<uint4 *>(j.dst);
  for (int64_t e = threadIdx.x; e < (int64_t)j.t8 * words; e += blockDim.x)
    dst[e] = e < (int64_t)j.t * words ? src[e] : make_uint4(0, 0, 0, 0);
  for (int i = threadIdx.x; i < j.t8; i += blockDim.x)
    j.dst_pos[i] = j.src_pos[i < j.t ? i : j.t - 1];
}

__global__ void k_tail_drop(const TailJob *jobs, int count) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const TailJob &j = jobs[i];
  // A fold skipped for capacity appended nothing: only a fold that ran leaves rows to drop.
  if (j.meta[ISKV_META_N] == j.n0 + j.t8) j.meta[ISKV_META_N] -= j.t8 - j.t;
}

cudaError_t launch_tail_pad(TailJob *jobs, int count, cudaStream_t s) {
  k_tail_pad<<<count, 256, 0, s>>>(jobs);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tail_drop(const TailJob *jobs, int count, cudaStream_t s) {
  k_tail_drop<<<(count + 127) / 128, 128, 0, s>>>(jobs, count);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace iskv
