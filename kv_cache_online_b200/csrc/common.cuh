// Shared device helpers for libiskv (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "iskv.h"

#define ISKV_DEV __device__ __forceinline__

namespace iskv {

// ---------------------------------------------------------------------------------------------
// Element access for the storage types (float32, bf16, fp16).
template <typename T> ISKV_DEV float to_f(T v);
template <> ISKV_DEV float to_f<float>(float v) { return v; }
template <> ISKV_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> ISKV_DEV float to_f<__half>(__half v) { return __half2float(v); }

template <typename T> ISKV_DEV T from_f(float v);
template <> ISKV_DEV float from_f<float>(float v) { return v; }
template <> ISKV_DEV __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> ISKV_DEV __half from_f<__half>(float v) { return __float2half_rn(v); }

// Host dispatch over an iskv_dtype: f(tag) with tag a value of the element type.
template <class F>
inline void with_dtype(int dtype, F &&f) {
  if (dtype == ISKV_BF16) f(__nv_bfloat16{});
  else if (dtype == ISKV_F16) f(__half{});
  else f(float{});
}

// ---------------------------------------------------------------------------------------------
// Warp reductions.
ISKV_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
ISKV_DEV double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Status bits recorded in meta[ISKV_META_STATUS].
ISKV_DEV void record_status(int64_t *meta, int code) {
  atomicOr(reinterpret_cast<unsigned long long *>(meta + ISKV_META_STATUS),
           (unsigned long long)(1ull << code));
}

// Store v as T. fp16 reaches only 65504: a finite value that overflows it (the failure the pages
// report for fp16 factors, Section 7.3) records ISKV_ERR_NONFINITE in meta.
template <typename T>
ISKV_DEV void store_checked(T *p, float v, int64_t *meta) {
  const T t = from_f<T>(v);
  if constexpr (sizeof(T) == 2 && !std::is_same<T, __nv_bfloat16>::value) {
    if (__hisinf(t) && isfinite(v)) record_status(meta, ISKV_ERR_NONFINITE);
  }
  *p = t;
}

// ---------------------------------------------------------------------------------------------
// Per-job fold workspace scalars (int32 slots at the start of each job's workspace).
enum FoldScalar {
  FS_K_OLD = 0,   // k before the fold
  FS_N_OLD = 1,   // n before the fold
  FS_P = 2,       // kept residual directions
  FS_K_NEW = 3,   // k' after the fold
  FS_SKIP = 4,    // 1 when the fold is skipped (capacity)
  FS_SWEEPS = 5,  // Jacobi sweeps used by the core SVD
  FS_RSWEEPS = 6, // Jacobi sweeps used by the residual SVD
  FS_COUNT = 32
};

// Fields every job descriptor starts with (fold and re-orthogonalisation jobs share them, so the
// rotation and Jacobi kernels can serve both through a byte stride).
struct JobHead {
  void *U;
  float *sigma;
  void *B;
  int32_t *pos;
  int64_t *meta;
  char *ws;  // this job's workspace slice; starts with FS_COUNT int32 scalars
};

// A fold job: one history plus its pending block.
struct FoldJob {
  JobHead h;
  const void *F;
  const int32_t *f_pos;
  int64_t n_cap;
  int64_t pad_;
};

// A re-orthogonalisation job.
struct ReorthJob {
  JobHead h;
  int64_t n_cap;
  int64_t n_exact;  // diagnostics: exact rows held beside the history (persistent bytes)
};

ISKV_DEV const JobHead &job_head(const char *jobs, int stride, int i) {
  return *reinterpret_cast<const JobHead *>(jobs + (size_t)i * stride);
}

// Byte offsets inside one job's fold workspace.
struct FoldWsLayout {
  size_t scal, C, E, C2, P, FP, rho, T, W, Y2, Gt, Gtb, Gbot, Ht, sig, Bn, Pb, Htb, E1, total;
  int hs;    // row stride (elements) of Ht: r_max + b
  int bpad;  // P's columns as fp16 (Pb), padded to a multiple of 64
  int kpad;  // K extent of the tensor-core basis rotation: r_max + bpad (row stride of Htb, fp16)
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline FoldWsLayout fold_ws_layout(int d, int r, int b) {
  FoldWsLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  L.hs = r + b;
  L.scal = take(FS_COUNT * sizeof(int32_t));
  L.C = take(sizeof(float) * (size_t)b * r);
  L.E = take(sizeof(float) * (size_t)b * d);
  L.C2 = take(sizeof(float) * (size_t)b * r);
  L.P = take(sizeof(float) * (size_t)d * b);
  L.FP = take(sizeof(float) * (size_t)b * b);
  L.rho = take(sizeof(float) * (size_t)b);
  L.T = take(sizeof(float) * (size_t)b * b);
  L.W = take(sizeof(float) * (size_t)b * b);
  L.Y2 = take(sizeof(float) * (size_t)b * b);
  L.Gt = take(sizeof(float) * (size_t)r * r);
  L.Gtb = take(sizeof(__half) * (size_t)r * r);
  L.Gbot = take(sizeof(float) * (size_t)b * r);
  L.Ht = take(sizeof(float) * (size_t)r * (r + b));
  L.sig = take(sizeof(float) * (size_t)r);
  L.Bn = take(sizeof(float) * (size_t)d * r);
  L.bpad = (b + 63) / 64 * 64;
  L.kpad = r + L.bpad;
  L.Pb = take(sizeof(__half) * (size_t)d * L.bpad);
  L.Htb = take(sizeof(__half) * (size_t)r * L.kpad);
  L.E1 = take(sizeof(__nv_bfloat16) * 2 * (size_t)b * d);  // tensor-core projection scratch
  L.total = o;
  return L;
}

}  // namespace iskv
