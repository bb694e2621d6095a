// Cache policy kernels: prefill partition of the prompt rows, decode-step append and the removal of
// folded rows from the exact-row table (iS-KV reading notes, Section 3.1, Section 3.2,
// Algorithm 1 steps 5-7, Algorithm 3 steps 1-2 and 6).
#pragma once

#include "common.cuh"

namespace iskv {

// Prefill partition of one side's prompt rows. `st` is an int64[4] scratch word laid out like a
// history's meta: st[0] receives the live-row count, st[ISKV_META_STATUS] the error bits.
struct PrefillArgs {
  const void *X;          // [L][d] x_dtype
  const int32_t *P;       // [n_p] protected positions, strictly ascending inside [0, L)
  void *rows;             // exact-row table [cap_e][d] t_dtype
  int32_t *pos;           // [cap_e]
  void *comp;             // [L][d] x_dtype: the rows left for the prompt SVD
  int32_t *comp_pos;      // [L]
  int64_t *st;
  int64_t L, n_p, w;      // prompt rows, protected rows, initial window
  int d, x_dtype, t_dtype;
};

// One table's new decode row.
struct AppendJob {
  const void *src;        // [d] row dtype
  void *dst;              // rows + (n_prot + n_live) * d
  int32_t *dst_pos;       // pos + n_prot + n_live
  int64_t *meta;          // the side's history meta word (fp16 overflow is recorded there)
  int32_t position;
  int32_t pad_;
};

// Removal of the `shift` oldest live rows of one table: live rows [shift, shift + keep) move to
// [0, keep) (rows and positions), starting at the first live row.
struct EvictJob {
  void *rows;             // rows + n_prot * d
  int32_t *pos;           // pos + n_prot
  int64_t keep;           // live rows that remain
  int64_t row_bytes;      // d * element size (a multiple of 16)
  int32_t shift;          // rows removed (the fold block)
  int32_t pad_;
};

// A history copied into a wider one (rank budget rw >= r, the same n_cap) and back. Widening
// copies U's n rows (n from the device meta word) and B into rows of rw entries with zeros after
// the first r, and sigma, positions and meta; narrowing keeps the first r columns of the wide
// history (its components are sorted by singular value, so these are its top r), sets k to
// min(r, k') and n to n', and ORs the wide history's status bits into the history's.
struct WidenArgs {
  void *U, *B;            // [n_cap][r], [d][r] (storage dtype)
  float *sigma;           // [r]
  int32_t *pos;           // [n_cap]
  int64_t *meta;          // [4]
  void *Uw, *Bw;          // [n_cap][rw], [d][rw]
  float *sigw;            // [rw]
  int32_t *posw;          // [n_cap]
  int64_t *metaw;         // [4]
  int64_t n_cap;
  int d, r, rw, esz;      // esz: element bytes of U and B (r * esz and rw * esz multiples of 16)
};

// The last, short block of a prompt compression: t rows copied into a t8-row buffer (t8 = t
// rounded up to a multiple of 8) followed by zero rows, positions padded with the last real one;
// after the fold, the t8 - t zero coordinate rows it appended are dropped from the history.
struct TailJob {
  const void *src;         // [t][d] rows
  const int32_t *src_pos;  // [t]
  void *dst;               // [t8][d] buffer
  int32_t *dst_pos;        // [t8]
  int64_t *meta;           // the history's meta word
  int64_t row_bytes;       // d * element size (a multiple of 16)
  int64_t n0;              // device-written: the history's n before the fold
  int32_t t, t8;
};

cudaError_t launch_tail_pad(TailJob *jobs, int count, cudaStream_t s);
cudaError_t launch_tail_drop(const TailJob *jobs, int count, cudaStream_t s);

cudaError_t launch_history_widen(const WidenArgs &a, cudaStream_t s);
cudaError_t launch_history_narrow(const WidenArgs &a, cudaStream_t s);

cudaError_t launch_prefill_partition(const PrefillArgs &a, cudaStream_t s);
cudaError_t launch_cache_append(const AppendJob *jobs, int count, int d, int src_dtype,
                                int dst_dtype, cudaStream_t s);
cudaError_t launch_cache_evict(const EvictJob *jobs, int count, cudaStream_t s);

}  // namespace iskv
