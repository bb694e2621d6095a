// A small register-tiled FFMA GEMM tile for the fp32-accuracy contractions of the fold
// (projection / residual passes, basis rotation). Operands are read through loader functors so
// that row-major, transposed and concatenated operands share one tile routine.
#pragma once

#include "common.cuh"

namespace iskv {

// out(m, n) = sum_k A(m, k) * Bop(k, n) for the BM x BN tile at (m0, n0), handed to ep(m, n, acc).
// Threads: (BM / TM) * (BN / TN). A_KFAST: consecutive threads load consecutive k of A (row-major
// A); otherwise consecutive m. B_NFAST: consecutive threads load consecutive n of Bop; otherwise
// consecutive k (transposed Bop).
template <int BM, int BN, int BK, int TM, int TN, bool A_KFAST, bool B_NFAST, class LA, class LB,
          class EP>
ISKV_DEV void tile_gemm(int m0, int n0, int M, int N, int K, const LA &la, const LB &lb,
                        const EP &ep) {
  constexpr int TR = BM / TM, TC = BN / TN, NT = TR * TC;
  __shared__ float As[BK][BM + 1];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tr = tid / TC, tc = tid % TC;
  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

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
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = As[kk][tr + i * TR];
#pragma unroll
      for (int j = 0; j < TN; ++j) bb[j] = Bs[kk][tc + j * TC];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int m = m0 + tr + i * TR, n = n0 + tc + j * TC;
      if (m < M && n < N) ep(m, n, acc[i][j]);
    }
}

}  // namespace iskv
