// A small register-tiled FFMA GEMM tile for the fp32-accuracy contractions of the fold
// (projection / residual passes, basis rotation). Operands are read through loader functors so
// that row-major, transposed and concatenated operands share one tile routine.
#pragma once

#include "common.cuh"

namespace iskv {

// Vector load of N consecutive floats from shared memory (N = 2 or 4, 8- or 16-byte aligned).
template <int N>
ISKV_DEV void lds_vec(float (&v)[N], const float *p) {
  static_assert(N == 2 || N == 4, "vector width");
  if constexpr (N == 4) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2 *>(p);
    v[0] = t.x; v[1] = t.y;
  }
}

// out(m, n) = sum_k A(m, k) * Bop(k, n) for the BM x BN tile at (m0, n0), handed to ep(m, n, acc).
// Threads: (BM / TM) * (BN / TN); thread (tr, tc) owns rows tr TM .. tr TM + TM - 1 and columns
// tc TN .. tc TN + TN - 1, so each k step reads its A and B fragments with one vector load each
// and accumulates column pairs with packed FFMA2. A_KFAST: consecutive threads load consecutive k
// of A (row-major A); otherwise consecutive m. B_NFAST: consecutive threads load consecutive n of
// Bop; otherwise consecutive k (transposed Bop).
template <int BM, int BN, int BK, int TM, int TN, bool A_KFAST, bool B_NFAST, class LA, class LB,
          class EP>
ISKV_DEV void tile_gemm(int m0, int n0, int M, int N, int K, const LA &la, const LB &lb,
                        const EP &ep) {
  static_assert(TN % 2 == 0 && (TM == 2 || TM == 4) && (TN == 2 || TN == 4), "thread tile");
  constexpr int TR = BM / TM, TC = BN / TN, NT = TR * TC;
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tr = tid / TC, tc = tid % TC;
  float2 acc[TM][TN / 2];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN / 2; ++j) acc[i][j] = make_float2(0.f, 0.f);

  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int e = tid; e < BM * BK; e += NT) {
      int mm, kk;
      if (A_KFAST) { mm = e / BK; kk = e % BK; } else { kk = e / BM; mm = e % BM; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? la(gm, gk) : 0.f;
    }
    for (int e = tid; e < BK * BN; e += NT) {
      int kk, nn;
      if (B_NFAST) { kk = e / BN; nn = e % BN; } else { nn = e / BK; kk = e % BK; }
      const int gk = k0 + kk, gn = n0 + nn;
      Bs[kk][nn] = (gk < K && gn < N) ? lb(gk, gn) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < BK; ++kk) {
      float a[TM], bb[TN];
      lds_vec<TM>(a, &As[kk][tr * TM]);
      lds_vec<TN>(bb, &Bs[kk][tc * TN]);
#pragma unroll
      for (int i = 0; i < TM; ++i) {
        const float2 ai = make_float2(a[i], a[i]);
#pragma unroll
        for (int j = 0; j < TN / 2; ++j)
          acc[i][j] = __ffma2_rn(ai, make_float2(bb[2 * j], bb[2 * j + 1]), acc[i][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN / 2; ++j) {
      const int m = m0 + tr * TM + i, n = n0 + tc * TN + 2 * j;
      if (m < M) {
        if (n < N) ep(m, n, acc[i][j].x);
        if (n + 1 < N) ep(m, n + 1, acc[i][j].y);
      }
    }
}

}  // namespace iskv
