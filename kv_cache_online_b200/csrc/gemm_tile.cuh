// A small register-tiled FFMA GEMM tile for the fp32-accuracy contractions of the fold
// (projection / residual passes, basis rotation). Operands are read through loader functors so
// that row-major, transposed and concatenated operands share one tile routine.
#pragma once

#include "common.cuh"

namespace iskv {

// Vector load of N consecutive floats from shared memory (N = 2, 4 or 8; 8- or 16-byte aligned).
template <int N>
ISKV_DEV void lds_vec(float (&v)[N], const float *p) {
  static_assert(N == 2 || N == 4 || N == 8, "vector width");
  if constexpr (N == 8) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    const float4 u = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    v[4] = u.x; v[5] = u.y; v[6] = u.z; v[7] = u.w;
  } else if constexpr (N == 4) {
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
  static_assert(TN % 2 == 0 && (TM == 2 || TM == 4 || TM == 8) && (TN == 2 || TN == 4 || TN == 8),
                "thread tile");
  constexpr int TR = BM / TM, TC = BN / TN, NT = TR * TC;
  constexpr int AE = (BM * BK + NT - 1) / NT, BE = (BK * BN + NT - 1) / NT;  // loads per thread
  // Two shared buffers: the next K block is fetched into registers while the current one is
  // multiplied, then stored into the other buffer (one barrier per K block).
  __shared__ __align__(16) float As[2][BK][BM + 4];
  __shared__ __align__(16) float Bs[2][BK][BN + 4];
  const int tid = threadIdx.x;
  const int tr = tid / TC, tc = tid % TC;
  float ra[AE], rb[BE];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int u = 0; u < AE; ++u) {
      const int e = tid + u * NT;
      int mm, kk;
      if (A_KFAST) { mm = e / BK; kk = e % BK; } else { kk = e / BM; mm = e % BM; }
      const int gm = m0 + mm, gk = k0 + kk;
      ra[u] = (e < BM * BK && gm < M && gk < K) ? la(gm, gk) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < BE; ++u) {
      const int e = tid + u * NT;
      int kk, nn;
      if (B_NFAST) { kk = e / BN; nn = e % BN; } else { nn = e / BK; kk = e % BK; }
      const int gk = k0 + kk, gn = n0 + nn;
      rb[u] = (e < BK * BN && gk < K && gn < N) ? lb(gk, gn) : 0.f;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int u = 0; u < AE; ++u) {
      const int e = tid + u * NT;
      if (e >= BM * BK) continue;
      int mm, kk;
      if (A_KFAST) { mm = e / BK; kk = e % BK; } else { kk = e / BM; mm = e % BM; }
      As[buf][kk][mm] = ra[u];
    }
#pragma unroll
    for (int u = 0; u < BE; ++u) {
      const int e = tid + u * NT;
      if (e >= BK * BN) continue;
      int kk, nn;
      if (B_NFAST) { kk = e / BN; nn = e % BN; } else { nn = e / BK; kk = e % BK; }
      Bs[buf][kk][nn] = rb[u];
    }
  };
  float2 acc[TM][TN / 2];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN / 2; ++j) acc[i][j] = make_float2(0.f, 0.f);

  const int nk = (K + BK - 1) / BK;
  if (nk > 0) {
    fetch(0);
    stash(0);
  }
  __syncthreads();
  for (int kb = 0; kb < nk; ++kb) {
    const int cur = kb & 1;
    if (kb + 1 < nk) fetch((kb + 1) * BK);  // in flight during the multiply below
#pragma unroll 4
    for (int kk = 0; kk < BK; ++kk) {
      float a[TM], bb[TN];
      lds_vec<TM>(a, &As[cur][kk][tr * TM]);
      lds_vec<TN>(bb, &Bs[cur][kk][tc * TN]);
#pragma unroll
      for (int i = 0; i < TM; ++i) {
        const float2 ai = make_float2(a[i], a[i]);
#pragma unroll
        for (int j = 0; j < TN / 2; ++j)
          acc[i][j] = __ffma2_rn(ai, make_float2(bb[2 * j], bb[2 * j + 1]), acc[i][j]);
      }
    }
    if (kb + 1 < nk) stash(cur ^ 1);
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
