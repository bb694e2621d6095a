// Re-orthogonalisation (iS-KV reading notes, Section 4.4).
//
// The pages take thin QR factorisations U = Q_U R_U, B = Q_B R_B, decompose
// R_U diag(sigma) R_B^T = X diag(sigma') Y^T and set U <- Q_U X, sigma <- sigma', B <- Q_B Y.
// Any factorisation with an orthonormal Q gives the same product and the same sigma', and the new
// U, B are the singular vectors of the product. Here R is the symmetric square root of the Gram
// matrix (the polar factor): R_U = (U^T U)^(1/2), Q_U = U R_U^(-1). Both roots come from the
// coupled Newton-Schulz iteration (Higham 1997), which is GEMM-only and converges quadratically
// for the near-orthonormal factors seen here:
//   Y_0 = A / c, Z_0 = I;  T = (3I - Z Y) / 2;  Y <- Y T;  Z <- T Z   ->  Y = (A/c)^(1/2),
//   Z = (A/c)^(-1/2), with c = trace(A) / k.
// Then M = R_U diag(sigma) R_B goes through the cluster Jacobi SVD (dense mode), and the two
// rotations U <- U (R_U^-1 X), B <- B (R_B^-1 Y) reuse the fold's rotation kernels.
#include "gemm_tile.cuh"
#include "profiling.h"
#include "reorth.h"
#include "tc_sm100.cuh"

namespace iskv {

// Scalar slots: the Newton-Schulz scales (float bits), and from RS_DEV on, per iteration `it` and
// factor `which`, the squared Frobenius norm of T - I accumulated by that iteration's first stage.
enum { RS_CU = 8, RS_CB = 9, RS_DEV = 16 };
static_assert(RS_DEV + 2 * NS_ITERS <= FS_COUNT, "scalar slots");

// Early exit of the iteration. With D = Z Y - I, one step maps D to -(3/4) D^2 + (1/4) D^3, and
// T - I = -D / 2. Once ||T - I||_F <= 5e-4 (so ||D||_2 <= 1e-3), the step that applies this T leaves
// ||D||_2 below 1e-6: further steps would change Y and Z only at float32 rounding level. Those
// steps are skipped (their outputs are copies). Rounding puts a floor near 2e-5 under ||T - I||_F
// for r = 256 (the diagonal's sums of r products near 1), well below the threshold.
constexpr float NS_STOP_SQ = 2.5e-7f;  // (5e-4)^2

ISKV_DEV bool ns_converged(const int32_t *sc, int it, int which) {
  return it > 0 && __int_as_float(sc[RS_DEV + 2 * (it - 1) + which]) <= NS_STOP_SQ;
}

// Iterations actually computed for factor `which` (a skipped iteration leaves Y, Z where they
// are). Iteration it reads the first buffer of its pair when it is even and writes the second, so
// the result sits in the first buffer after an even count and in the second after an odd count.
ISKV_DEV bool ns_result_in_second(const int32_t *sc, int which) {
  int done = 0;
  while (done < NS_ITERS && !ns_converged(sc, done, which)) ++done;
  return done & 1;
}

ReorthWsLayout reorth_ws_layout(int d, int r, int64_t n_cap) {
  ReorthWsLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  const size_t rr = sizeof(float) * (size_t)r * r;
  L.nsplit_u = (int)((n_cap + REORTH_SPLIT - 1) / REORTH_SPLIT);
  if (L.nsplit_u < 1) L.nsplit_u = 1;
  L.nsplit_b = (d + REORTH_SPLIT - 1) / REORTH_SPLIT;
  L.scal = take(FS_COUNT * sizeof(int32_t));
  L.gpart_u = take(rr * L.nsplit_u);
  L.gpart_b = take(rr * L.nsplit_b);
  for (int w = 0; w < 2; ++w) {
    L.G[w] = take(rr);
    L.Y[w] = take(rr);
    L.Z[w] = take(rr);
    L.T[w] = take(rr);
    L.Y2[w] = take(rr);
    L.Z2[w] = take(rr);
  }
  L.M = take(rr);
  L.Gt = take(rr);
  L.Gtb = take(sizeof(__nv_bfloat16) * (size_t)r * r);
  L.Ht = take(rr);
  L.sig = take(sizeof(float) * r);
  L.TUt = take(rr);
  L.TUtb = take(sizeof(__half) * (size_t)r * r);
  L.TBt = take(rr);
  L.TBtb = take(sizeof(__half) * (size_t)r * r);
  L.Bn = take(sizeof(float) * (size_t)d * r);
  L.total = o;
  return L;
}

__global__ void k_reorth_prepare(const ReorthJob *jobs, ReorthParams p) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= p.count) return;
  const ReorthJob &jb = jobs[j];
  int32_t *sc = reinterpret_cast<int32_t *>(jb.h.ws);
  const int64_t k = jb.h.meta[ISKV_META_K], n = jb.h.meta[ISKV_META_N];
  sc[FS_K_OLD] = (int32_t)k;
  sc[FS_N_OLD] = (int32_t)n;
  sc[FS_P] = 0;
  sc[FS_K_NEW] = (int32_t)k;
  sc[FS_SKIP] = (k <= 0 || k > p.r || n < 0 || n > jb.n_cap) ? 1 : 0;
  sc[FS_SWEEPS] = 0;
  for (int i = 0; i < 2 * NS_ITERS; ++i) sc[RS_DEV + i] = 0;  // float 0
}

// Register tiles of the r x r products: 128 x 64 blocks, 8 x 4 outputs per thread (each k step
// reads 12 floats from shared memory per 32 FMAs), two blocks resident per SM.
constexpr int GBM = 128, GBN = 64, GBK = 16, GTM = 8, GTN = 4;

// Gram partial: Gpart[s] = X[rows of split s]^T X[rows of split s] (k x k), X = U (n rows) or B.
template <typename TS>
__global__ void __launch_bounds__(256) k_gram_partial(const ReorthJob *jobs, ReorthParams p,
                                                      int which, int nsplit) {
  const int job = blockIdx.z / nsplit, s = blockIdx.z % nsplit;
  const ReorthJob &jb = jobs[job];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], r = p.r;
  const int rows = which == 0 ? sc[FS_N_OLD] : p.d;
  const TS *X = static_cast<const TS *>(which == 0 ? jb.h.U : jb.h.B);
  float *G = reinterpret_cast<float *>(jb.h.ws + (which == 0 ? p.ws.gpart_u : p.ws.gpart_b)) +
             (size_t)s * r * r;
  const int r0 = s * REORTH_SPLIT;
  const int nrows = max(0, min(REORTH_SPLIT, rows - r0));
  const int m0 = blockIdx.y * GBM, n0 = blockIdx.x * GBN;
  if (m0 >= k || n0 >= k) return;
  tile_gemm<GBM, GBN, GBK, GTM, GTN, false, true>(
      m0, n0, k, k, nrows,
      [&](int m, int kk) { return to_f<TS>(X[(size_t)(r0 + kk) * r + m]); },
      [&](int kk, int n) { return to_f<TS>(X[(size_t)(r0 + kk) * r + n]); },
      [&](int m, int n, float acc) { G[(size_t)m * r + n] = acc; });
}

// Sum the partials into G (the whole r x r matrix: entries beyond k are zero in every partial,
// since the factors' columns beyond k are), four floats per thread.
__global__ void __launch_bounds__(256) k_gram_reduce(const ReorthJob *jobs, ReorthParams p) {
  const int job = blockIdx.y >> 1, which = blockIdx.y & 1;
  const ReorthJob &jb = jobs[job];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  // The tensor-core Gram writes a single B chunk's matrix to G itself.
  if (which == 1 && p.gram_nsu > 0 && p.ws.nsplit_b == 1) return;
  const int r = p.r;
  const int rows = which == 0 ? sc[FS_N_OLD] : p.d;
  // Splits that hold rows: REORTH_SPLIT-row splits, or the tensor-core Gram's balanced U chunks.
  const bool bal = which == 0 && p.gram_nsu > 0;
  const int chunk = bal ? gram_chunk(rows, p.gram_nsu) : REORTH_SPLIT;
  const int ns = min(bal ? p.gram_nsu : (which == 0 ? p.ws.nsplit_u : p.ws.nsplit_b),
                     (rows + chunk - 1) / chunk);
  const float4 *part = reinterpret_cast<const float4 *>(jb.h.ws + (which == 0 ? p.ws.gpart_u : p.ws.gpart_b));
  float4 *G = reinterpret_cast<float4 *>(jb.h.ws + p.ws.G[which]);
  const int n4 = r * r / 4;  // r is a multiple of 4 on every path that reaches here
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += gridDim.x * blockDim.x) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < ns; ++q) {
      const float4 v = part[(size_t)q * n4 + e];
      a.x += v.x;
      a.y += v.y;
      a.z += v.z;
      a.w += v.w;
    }
    G[e] = a;
  }
}

__global__ void __launch_bounds__(256) k_ns_init(const ReorthJob *jobs, ReorthParams p) {
  const int job = blockIdx.y >> 1, which = blockIdx.y & 1;
  const ReorthJob &jb = jobs[job];
  int32_t *sc = reinterpret_cast<int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], r = p.r;
  const float *G = reinterpret_cast<const float *>(jb.h.ws + p.ws.G[which]);
  // Trace of G by a block reduction (every block computes it; one block publishes the scale).
  __shared__ double s_part[8];
  double t = 0.0;
  for (int i = threadIdx.x; i < k; i += blockDim.x) t += G[(size_t)i * r + i];
  t = warp_sum(t);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = t;
  __syncthreads();
  double tr = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tr += s_part[w];
  const double cmean = tr / k;
  if (blockIdx.x == 0 && threadIdx.x == 0) sc[which == 0 ? RS_CU : RS_CB] = __float_as_int((float)cmean);
  const float c = (float)cmean;
  const float inv = c > 0.f ? 1.f / c : 0.f;
  float *Y = reinterpret_cast<float *>(jb.h.ws + p.ws.Y[which]);
  float *Z = reinterpret_cast<float *>(jb.h.ws + p.ws.Z[which]);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < k * k; e += gridDim.x * blockDim.x) {
    const int i = e / k, j = e % k;
    Y[(size_t)i * r + j] = G[(size_t)i * r + j] * inv;
    Z[(size_t)i * r + j] = i == j ? 1.f : 0.f;
  }
}

// Newton-Schulz stages of iteration `it`. STAGE 0: T = 1.5 I - 0.5 Z Y, and ||T - I||_F^2 summed
// into the iteration's slot. STAGE 1: Y2 = Y T (g = 0), Z2 = T Z (g = 1). Once an earlier
// iteration's T met the stopping threshold, both stages do nothing: Y, Z stay in the buffers the
// last computed iteration wrote, which the consumers locate with ns_result_in_second.
template <int STAGE>
__global__ void __launch_bounds__(256, 2) k_ns_step(const ReorthJob *jobs, ReorthParams p, int it,
                                                 size_t y0, size_t z0, size_t y1, size_t z1,
                                                 size_t yb0, size_t zb0, size_t yb1, size_t zb1) {
  const int per = STAGE == 0 ? 2 : 4;
  const int job = blockIdx.z / per, rem = blockIdx.z % per, which = rem & 1, g = rem >> 1;
  const ReorthJob &jb = jobs[job];
  int32_t *sc = reinterpret_cast<int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], r = p.r;
  char *ws = jb.h.ws;
  const float *Y = reinterpret_cast<const float *>(ws + (which == 0 ? y0 : yb0));
  const float *Z = reinterpret_cast<const float *>(ws + (which == 0 ? z0 : zb0));
  float *T = reinterpret_cast<float *>(ws + p.ws.T[which]);
  const int m0 = blockIdx.y * GBM, n0 = blockIdx.x * GBN;
  if (m0 >= k || n0 >= k) return;
  const bool done = ns_converged(sc, it, which);  // uniform over the block
  if (STAGE == 0) {
    if (done) return;
    float ss = 0.f;
    tile_gemm<GBM, GBN, GBK, GTM, GTN, true, true>(
        m0, n0, k, k, k, [&](int m, int kk) { return Z[(size_t)m * r + kk]; },
        [&](int kk, int n) { return Y[(size_t)kk * r + n]; },
        [&](int m, int n, float acc) {
          const float t = (m == n ? 1.5f : 0.f) - 0.5f * acc;
          const float dv = t - (m == n ? 1.f : 0.f);
          ss = fmaf(dv, dv, ss);
          T[(size_t)m * r + n] = t;
        });
    __shared__ float red[8];
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      float tot = 0.f;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
      atomicAdd(reinterpret_cast<float *>(sc + RS_DEV + 2 * it + which), tot);
    }
    return;
  }
  float *Xo = reinterpret_cast<float *>(ws + (g == 0 ? (which == 0 ? y1 : yb1) : (which == 0 ? z1 : zb1)));
  if (done) return;
  // Y2 = Y T (g = 0) or Z2 = T Z (g = 1): one tile routine with the operands chosen per block.
  const float *A = g == 0 ? Y : T, *Bm = g == 0 ? T : Z;
  tile_gemm<GBM, GBN, GBK, GTM, GTN, true, true>(
      m0, n0, k, k, k, [&](int m, int kk) { return A[(size_t)m * r + kk]; },
      [&](int kk, int n) { return Bm[(size_t)kk * r + n]; },
      [&](int m, int n, float acc) { Xo[(size_t)m * r + n] = acc; });
}

// The same stages on the tensor cores, for bf16-stored factors (r a multiple of 64 up to 256).
// Each product is taken in three bf16 MMAs, A_hi B_hi + A_hi B_lo + A_lo B_hi with x = x_hi + x_lo
// (x_hi = bf16(x), x_lo = bf16(x - x_hi)): about 16 significant bits, far below the bf16 rounding of the factors
// the re-orthogonalisation serves, and enough for the stopping test (its rounding floor stays
// near 1e-4 in ||T - I||_F against the 5e-4 threshold). Y, Z and T are polynomials in the Gram
// matrix, hence symmetric, so the right operand's rows are read as its columns. One CTA takes
// 128 rows of one product (N = r, K = k): 8 warps convert the float32 K-slabs of both operands
// into two 96 KB stages of hi / lo tiles (128-byte-swizzled K-major), one thread issues the MMAs
// into TMEM, and the 8 warps then stage the result through the idle stages and write whole rows.
constexpr int NS_TC_THREADS = 288;  // 8 converter / epilogue warps + the MMA warp
constexpr uint64_t NS_WAIT_NS = 2000000000ull;

struct NsTcCtl {
  uint64_t full[2], empty[2], acc;
  uint32_t tmem;
  int abort;
};

__host__ __device__ constexpr size_t ns_tc_stage_bytes() { return 2 * 128 * 128 + 2 * 256 * 128; }
__host__ __device__ constexpr size_t ns_tc_smem() {
  return 1024 + 2 * ns_tc_stage_bytes() + sizeof(NsTcCtl);
}

// Row `row` of a K-major 128-byte-swizzled tile: 16-byte chunk c of its 128 bytes at chunk
// c ^ (row & 7).
ISKV_DEV void ns_put_chunk(uint8_t *tile, int row, int c, uint4 v) {
  *reinterpret_cast<uint4 *>(tile + row * 128 + ((c ^ (row & 7)) << 4)) = v;
}

// Eight floats to bf16 hi and lo parts, packed two per word (low half first).
ISKV_DEV void ns_split8(const float (&x)[8], uint4 &hi, uint4 &lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat16 a = __float2bfloat16_rn(x[2 * i]), b = __float2bfloat16_rn(x[2 * i + 1]);
    const __nv_bfloat16 c = __float2bfloat16_rn(x[2 * i] - __bfloat162float(a));
    const __nv_bfloat16 d = __float2bfloat16_rn(x[2 * i + 1] - __bfloat162float(b));
    h[i] = (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
    l[i] = (uint32_t)__bfloat16_as_ushort(c) | ((uint32_t)__bfloat16_as_ushort(d) << 16);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <int STAGE>
__global__ void __launch_bounds__(NS_TC_THREADS, 1) k_ns_tc(const ReorthJob *jobs, ReorthParams p,
                                                           int it, size_t y0, size_t z0, size_t y1,
                                                           size_t z1, size_t yb0, size_t zb0,
                                                           size_t yb1, size_t zb1) {
  using namespace tc;
  const int per = STAGE == 0 ? 2 : 4;
  const int job = blockIdx.y / per, rem = blockIdx.y % per, which = rem & 1, g = rem >> 1;
  const ReorthJob &jb = jobs[job];
  int32_t *sc = reinterpret_cast<int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], R = p.r, m0 = blockIdx.x * 128;
  if (m0 >= k || ns_converged(sc, it, which)) return;  // uniform over the CTA
  char *ws = jb.h.ws;
  const float *Y = reinterpret_cast<const float *>(ws + (which == 0 ? y0 : yb0));
  const float *Z = reinterpret_cast<const float *>(ws + (which == 0 ? z0 : zb0));
  const float *Am, *Bm;
  float *Out;
  if (STAGE == 0) {
    Am = Z;
    Bm = Y;
    Out = reinterpret_cast<float *>(ws + p.ws.T[which]);
  } else {
    const float *T = reinterpret_cast<const float *>(ws + p.ws.T[which]);
    Am = g == 0 ? Y : T;
    Bm = g == 0 ? T : Z;
    Out = reinterpret_cast<float *>(
        ws + (g == 0 ? (which == 0 ? y1 : yb1) : (which == 0 ? z1 : zb1)));
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  NsTcCtl *ctl = reinterpret_cast<NsTcCtl *>(smem + 2 * ns_tc_stage_bytes());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int KS = (k + 63) / 64;
  const uint32_t idesc = idesc_bf16_f32(128, R);
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->full[i], 8);
      mbar_init(&ctl->empty[i], 1);
    }
    mbar_init(&ctl->acc, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  const uint32_t ncols = R <= 64 ? 64 : (R <= 128 ? 128 : 256);
  if (warp == 8) tmem_alloc(&ctl->tmem, ncols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int *abort = &ctl->abort;

  if (warp < 8) {
    // ---------------- converters: K-slab s of A (rows m0 .. m0+127) and B (rows 0 .. R-1)
    bool ok = true;
    for (int s = 0; s < KS && ok; ++s) {
      const int st = s & 1;
      if (s >= 2 && !__all_sync(~0u, mbar_wait(&ctl->empty[st], ((s - 2) >> 1) & 1, abort,
                                               NS_WAIT_NS))) {
        ok = false;
        break;
      }
      uint8_t *ahi = smem + st * ns_tc_stage_bytes(), *alo = ahi + 128 * 128;
      uint8_t *bhi = alo + 128 * 128, *blo = bhi + 256 * 128;
      // A: thread -> (row tid / 2, 32 columns); B: thread -> (row tid, 64 columns). All of a
      // thread's 16-byte loads are issued before any is converted; entries outside the leading
      // k x k block count as zero.
      {
        const int row = tid >> 1, c0 = (tid & 1) * 32, gm = m0 + row;
        float4 xa[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          xa[u] = gm < R ? *reinterpret_cast<const float4 *>(Am + (size_t)gm * R + s * 64 + c0 + 4 * u)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 xb[16];
        const bool brow = tid < R;
#pragma unroll
        for (int u = 0; u < 16; ++u)
          xb[u] = brow ? *reinterpret_cast<const float4 *>(Bm + (size_t)tid * R + s * 64 + 4 * u)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float x[8] = {xa[2 * u].x, xa[2 * u].y, xa[2 * u].z, xa[2 * u].w,
                        xa[2 * u + 1].x, xa[2 * u + 1].y, xa[2 * u + 1].z, xa[2 * u + 1].w};
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (!(gm < k && s * 64 + c0 + u * 8 + e < k)) x[e] = 0.f;
          uint4 hv, lv;
          ns_split8(x, hv, lv);
          ns_put_chunk(ahi, row, (c0 >> 3) + u, hv);
          ns_put_chunk(alo, row, (c0 >> 3) + u, lv);
        }
        if (brow) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float x[8] = {xb[2 * u].x, xb[2 * u].y, xb[2 * u].z, xb[2 * u].w,
                          xb[2 * u + 1].x, xb[2 * u + 1].y, xb[2 * u + 1].z, xb[2 * u + 1].w};
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (!(tid < k && s * 64 + u * 8 + e < k)) x[e] = 0.f;
            uint4 hv, lv;
            ns_split8(x, hv, lv);
            ns_put_chunk(bhi, tid, u, hv);
            ns_put_chunk(blo, tid, u, lv);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->full[st]);
    }
    if (!ok) {
      ctl->abort = 1;
      record_status(jb.h.meta, ISKV_ERR_TIMEOUT);
    }
    // ---------------- epilogue: warp (q, half) takes TMEM lanes 32 q and columns 128 half ..
    const int q = warp & 3, half = warp >> 2, cols = R / 2, c0 = half * cols;
    const bool ready = ok && __all_sync(~0u, mbar_wait(&ctl->acc, 0, abort, NS_WAIT_NS));
    fence_after_sync();
    // The stages are idle once the MMAs are done: rows of R + 4 floats (bank-spread) hold the
    // 128 x R result before it leaves in whole rows.
    float *stg = reinterpret_cast<float *>(smem);
    const int LDS = R + 4, row = q * 32 + lane, gm = m0 + row;
    float ss = 0.f;
    if (ready) {
      for (int cc = 0; cc < cols; cc += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + c0 + cc, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int n = c0 + cc + e;
          float o = v[e];
          if (STAGE == 0) {
            const float t = (gm == n ? 1.5f : 0.f) - 0.5f * o;
            const float dv = t - (gm == n ? 1.f : 0.f);
            if (gm < k && n < k) ss = fmaf(dv, dv, ss);
            o = t;
          }
          stg[row * LDS + n] = o;
        }
      }
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ready) {
      for (int i = warp; i < 128; i += 8) {
        const int gi = m0 + i;
        if (gi >= k) continue;
        for (int n = lane; n < k; n += 32) Out[(size_t)gi * R + n] = stg[i * LDS + n];
      }
      if (STAGE == 0) {
        ss = warp_sum(ss);
        if (lane == 0) atomicAdd(reinterpret_cast<float *>(sc + RS_DEV + 2 * it + which), ss);
      }
    }
  } else if (lane == 0) {
    // ---------------- MMA issuer
    bool ok = true;
    for (int s = 0; s < KS; ++s) {
      const int st = s & 1;
      if (!mbar_wait(&ctl->full[st], (s >> 1) & 1, abort, NS_WAIT_NS)) { ok = false; break; }
      fence_after_sync();
      const uint64_t ahi = sw128_desc(smem_u32(smem + st * ns_tc_stage_bytes()));
      const uint64_t alo = desc_add(ahi, 128 * 128), bhi = desc_add(alo, 128 * 128);
      const uint64_t blo = desc_add(bhi, 256 * 128);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t o = kk * 32;
        mma_bf16(tmem, desc_add(ahi, o), desc_add(bhi, o), idesc, (s | kk) != 0);
        mma_bf16(tmem, desc_add(ahi, o), desc_add(blo, o), idesc, true);
        mma_bf16(tmem, desc_add(alo, o), desc_add(bhi, o), idesc, true);
      }
      mma_commit(&ctl->empty[st]);
    }
    if (!ok) {
      ctl->abort = 1;
      record_status(jb.h.meta, ISKV_ERR_TIMEOUT);
    }
    mma_commit(&ctl->acc);
    mbar_wait(&ctl->acc, 0, abort, NS_WAIT_NS / 4);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 8) tmem_dealloc(tmem, ncols);
}

// Convergence check of the iteration: the last computed T = 1.5 I - 0.5 Z Y must be I to working
// accuracy, ||T - I||_F <= 1e-3 (the first stage of every computed iteration summed the squares;
// after an early stop the remaining slots hold 0). Quadratic convergence from a Gram matrix within
// ~10 % of a multiple of I needs 4 iterations; the iteration stops after 5.
__global__ void k_ns_check(const ReorthJob *jobs, ReorthParams p) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= p.count * 2) return;
  const int job = e >> 1, which = e & 1;
  const ReorthJob &jb = jobs[job];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const float last = __int_as_float(sc[RS_DEV + 2 * (NS_ITERS - 1) + which]);
  if (!(last <= 1e-6f)) record_status(jb.h.meta, ISKV_ERR_NOT_CONVERGED);
}

// M = sqrt(c_u c_b) Y_u diag(sigma) Y_b  (= R_U diag(sigma) R_B^T with symmetric R_B).
__global__ void __launch_bounds__(256, 2) k_reorth_M(const ReorthJob *jobs, ReorthParams p) {
  const ReorthJob &jb = jobs[blockIdx.z];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], r = p.r;
  const size_t yu = ns_result_in_second(sc, 0) ? p.ws.Y2[0] : p.ws.Y[0];
  const size_t yb = ns_result_in_second(sc, 1) ? p.ws.Y2[1] : p.ws.Y[1];
  const float scale = sqrtf(__int_as_float(sc[RS_CU]) * __int_as_float(sc[RS_CB]));
  const float *Yu = reinterpret_cast<const float *>(jb.h.ws + yu);
  const float *Yb = reinterpret_cast<const float *>(jb.h.ws + yb);
  const float *sg = jb.h.sigma;
  float *M = reinterpret_cast<float *>(jb.h.ws + p.ws.M);
  const int m0 = blockIdx.y * GBM, n0 = blockIdx.x * GBN;
  if (m0 >= k || n0 >= k) return;
  tile_gemm<GBM, GBN, GBK, GTM, GTN, true, true>(
      m0, n0, k, k, k, [&](int m, int l) { return Yu[(size_t)m * r + l] * sg[l]; },
      [&](int l, int n) { return Yb[(size_t)l * r + n]; },
      [&](int m, int n, float acc) { M[(size_t)m * r + n] = scale * acc; });
}

// Rotations: TUt[q][l] = (Z_u X)[l][q] / sqrt(c_u) with X[j][q] = Gt[q][j];
//            TBt[q][l] = (Z_b Y)[l][q] / sqrt(c_b) with Y[j][q] = Ht[q][j].
__global__ void __launch_bounds__(256, 2) k_reorth_T(const ReorthJob *jobs, ReorthParams p) {
  const int job = blockIdx.z >> 1, which = blockIdx.z & 1;
  const ReorthJob &jb = jobs[job];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], r = p.r;
  const float inv = rsqrtf(__int_as_float(sc[which == 0 ? RS_CU : RS_CB]));
  const size_t zo = ns_result_in_second(sc, which) ? p.ws.Z2[which] : p.ws.Z[which];
  const float *Z = reinterpret_cast<const float *>(jb.h.ws + zo);
  const float *V = reinterpret_cast<const float *>(jb.h.ws + (which == 0 ? p.ws.Gt : p.ws.Ht));
  float *out = reinterpret_cast<float *>(jb.h.ws + (which == 0 ? p.ws.TUt : p.ws.TBt));
  // fp16 copies (the tensor-core rotations' operand type).
  __half *outh = reinterpret_cast<__half *>(jb.h.ws + (which == 0 ? p.ws.TUtb : p.ws.TBtb));
  const int m0 = blockIdx.y * GBM, n0 = blockIdx.x * GBN;
  // Entries outside the leading k x k block are zero: the tensor-core rotations multiply by the
  // whole r x r matrix.
  if (k < r)
    for (int e = threadIdx.x; e < GBM * GBN; e += blockDim.x) {
      const int q = n0 + e / GBM, l = m0 + e % GBM;
      if (l < r && q < r && (l >= k || q >= k)) {
        out[(size_t)q * r + l] = 0.f;
        outh[(size_t)q * r + l] = __float2half_rn(0.f);
      }
    }
  // B's columns k .. r-1 are cleared before the in-place tensor-core basis rotation (zero after
  // every fold; clearing keeps a stray non-finite value there out of the products).
  if (which == 1 && p.tc_basis && k < r) {
    __nv_bfloat16 *B = static_cast<__nv_bfloat16 *>(jb.h.B);
    const size_t w = (size_t)(r - k), nth = (size_t)gridDim.x * gridDim.y * blockDim.x;
    for (size_t e = ((size_t)blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
         e < (size_t)p.d * w; e += nth)
      B[(e / w) * r + k + e % w] = __float2bfloat16_rn(0.f);
  }
  if (m0 >= k || n0 >= k) return;
  tile_gemm<GBM, GBN, GBK, GTM, GTN, true, false>(
      m0, n0, k, k, k, [&](int l, int j) { return Z[(size_t)l * r + j]; },
      [&](int j, int q) { return V[(size_t)q * r + j]; },
      [&](int l, int q, float acc) {
        const float v = acc * inv;
        out[(size_t)q * r + l] = v;
        outh[(size_t)q * r + l] = __float2half_rn(v);
      });
}

template <typename TS>
__global__ void k_reorth_finalize(const ReorthJob *jobs, ReorthParams p) {
  const ReorthJob &jb = jobs[blockIdx.y];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], r = p.r, d = p.d;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
  TS *B = static_cast<TS *>(jb.h.B);
  const float *Bn = reinterpret_cast<const float *>(jb.h.ws + p.ws.Bn);
  const float *sig = reinterpret_cast<const float *>(jb.h.ws + p.ws.sig);
  if (!p.tc_basis)  // the tensor-core basis rotation wrote B in place
    for (int e = tid; e < d * r; e += nth) {
      const int q = e % r;
      store_checked(&B[e], q < k ? Bn[e] : 0.f, jb.h.meta);
    }
  for (int e = tid; e < r; e += nth) jb.h.sigma[e] = e < k ? sig[e] : 0.f;
  if (tid == 0) jb.h.meta[ISKV_META_FOLDS] = 0;
}

// Gram matrices U^T U and B^T B of every job into the workspace (G[0], G[1]), after the scalars.
static cudaError_t reorth_gram(const ReorthJob *jobs, const ReorthParams &p, cudaStream_t s) {
  const int r = p.r;
  const ReorthWsLayout &W = p.ws;
  k_reorth_prepare<<<(p.count + 127) / 128, 128, 0, s>>>(jobs, p);
  const unsigned tn = (r + GBN - 1) / GBN, tm = (r + GBM - 1) / GBM;
  if (p.gram_host) {
    GramParams gp;
    gp.r = r;
    gp.d = p.d;
    gp.count = p.count;
    gp.nsu = p.gram_nsu;
    gp.nsb = W.nsplit_b;
    gp.split = REORTH_SPLIT;
    gp.off_gu = W.gpart_u;
    gp.off_gb = W.gpart_b;
    gp.off_g1 = W.G[1];
    cudaError_t e0 = launch_tc_gram(p.gram_dev, gp, s);
    if (e0 != cudaSuccess) return e0;
  } else {
    with_dtype(p.storage, [&](auto ts) {
      using TS = decltype(ts);
      k_gram_partial<TS><<<dim3(tn, tm, p.count * W.nsplit_u), 256, 0, s>>>(jobs, p, 0, W.nsplit_u);
      k_gram_partial<TS><<<dim3(tn, tm, p.count * W.nsplit_b), 256, 0, s>>>(jobs, p, 1, W.nsplit_b);
    });
    count_launches(2);
  }
  k_gram_reduce<<<dim3(64, p.count * 2), 256, 0, s>>>(jobs, p);
  count_launches(2);
  return cudaGetLastError();
}

__global__ void __launch_bounds__(256) k_diag_finish(const ReorthJob *jobs, ReorthParams p,
                                                     int exact_bytes, double *orth_u,
                                                     double *orth_b, int64_t *pbytes) {
  const ReorthJob &jb = jobs[blockIdx.x];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws);
  const int64_t k = jb.h.meta[ISKV_META_K], n = jb.h.meta[ISKV_META_N];
  const int r = p.r;
  __shared__ double red[2][8];
  double acc[2] = {0.0, 0.0};
  const bool skip = sc[FS_SKIP] != 0;
  if (!skip)
    for (int w = 0; w < 2; ++w) {
      const float *G = reinterpret_cast<const float *>(jb.h.ws + p.ws.G[w]);
      for (int64_t e = threadIdx.x; e < k * k; e += blockDim.x) {
        const int64_t i = e / k, j = e % k;
        const double v = (double)G[i * r + j] - (i == j ? 1.0 : 0.0);
        acc[w] = fma(v, v, acc[w]);
      }
    }
  for (int w = 0; w < 2; ++w) {
    const double t = warp_sum(acc[w]);
    if ((threadIdx.x & 31) == 0) red[w][threadIdx.x >> 5] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tu = 0.0, tb = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      tu += red[0][i];
      tb += red[1][i];
    }
    // An empty history is orthonormal by convention; an inconsistent one reports NaN.
    const bool bad = skip && k != 0;
    orth_u[blockIdx.x] = bad ? nan("") : sqrt(tu);
    orth_b[blockIdx.x] = bad ? nan("") : sqrt(tb);
    const int64_t sf = p.storage == ISKV_F32 ? 4 : 2;
    pbytes[blockIdx.x] = sf * (n * k + (int64_t)p.d * k + k) + (int64_t)exact_bytes * jb.n_exact * p.d;
  }
}

cudaError_t launch_diagnostics(const ReorthJob *jobs, const ReorthParams &p, int exact_bytes,
                               double *orth_u, double *orth_b, int64_t *pbytes, cudaStream_t s) {
  cudaError_t e = reorth_gram(jobs, p, s);
  if (e != cudaSuccess) return e;
  k_diag_finish<<<p.count, 256, 0, s>>>(jobs, p, exact_bytes, orth_u, orth_b, pbytes);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_reorth(const ReorthJob *jobs, const ReorthParams &p, cudaStream_t s) {
  const int r = p.r;
  const ReorthWsLayout &W = p.ws;
  const unsigned tn = (r + GBN - 1) / GBN, tm = (r + GBM - 1) / GBM;
  {
    cudaError_t e0 = reorth_gram(jobs, p, s);
    if (e0 != cudaSuccess) return e0;
  }
  stage_mark(s, ST_REORTH_GRAM);
  k_ns_init<<<dim3(64, p.count * 2), 256, 0, s>>>(jobs, p);
  size_t y0[2] = {W.Y[0], W.Y[1]}, z0[2] = {W.Z[0], W.Z[1]};
  size_t y1[2] = {W.Y2[0], W.Y2[1]}, z1[2] = {W.Z2[0], W.Z2[1]};
  const bool ns_tc = p.tc_basis != 0;  // bf16 factors, r a multiple of 64 up to 256
  if (ns_tc) {
    cudaError_t e0 = cudaFuncSetAttribute(k_ns_tc<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)ns_tc_smem());
    if (e0 == cudaSuccess)
      e0 = cudaFuncSetAttribute(k_ns_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)ns_tc_smem());
    if (e0 != cudaSuccess) return e0;
  }
  for (int it = 0; it < NS_ITERS; ++it) {
    if (ns_tc) {
      k_ns_tc<0><<<dim3((r + 127) / 128, p.count * 2), NS_TC_THREADS, ns_tc_smem(), s>>>(
          jobs, p, it, y0[0], z0[0], y1[0], z1[0], y0[1], z0[1], y1[1], z1[1]);
      k_ns_tc<1><<<dim3((r + 127) / 128, p.count * 4), NS_TC_THREADS, ns_tc_smem(), s>>>(
          jobs, p, it, y0[0], z0[0], y1[0], z1[0], y0[1], z0[1], y1[1], z1[1]);
    } else {
      k_ns_step<0><<<dim3(tn, tm, p.count * 2), 256, 0, s>>>(jobs, p, it, y0[0], z0[0], y1[0],
                                                           z1[0], y0[1], z0[1], y1[1], z1[1]);
      k_ns_step<1><<<dim3(tn, tm, p.count * 4), 256, 0, s>>>(jobs, p, it, y0[0], z0[0], y1[0],
                                                           z1[0], y0[1], z0[1], y1[1], z1[1]);
    }
    for (int w = 0; w < 2; ++w) {
      size_t t = y0[w]; y0[w] = y1[w]; y1[w] = t;
      t = z0[w]; z0[w] = z1[w]; z1[w] = t;
    }
  }
  k_ns_check<<<(p.count * 2 + 127) / 128, 128, 0, s>>>(jobs, p);
  k_reorth_M<<<dim3(tn, tm, p.count), 256, 0, s>>>(jobs, p);
  count_launches(3 + 2 * NS_ITERS);
  stage_mark(s, ST_REORTH_NS);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  CoreParams c;
  c.r = r;
  c.b = 0;
  c.count = p.count;
  c.job_stride = sizeof(ReorthJob);
  c.mode = 1;
  c.C = 0;
  c.FP = 0;
  c.M = W.M;
  c.Gt = W.Gt;
  c.Gtb = W.Gtb;
  c.Gbot = W.Gt;  // unused in dense mode (b = 0)
  c.Ht = W.Ht;
  c.sig = W.sig;
  c.hs = r;
  c.ldm = r;
  c.max_sweeps = 40;
  // Float64 inner products only pay for float32 factors: the bf16 rounding of stored factors
  // (2^-9) is far above the float32 orthogonality the float32-accumulating sweep reaches.
  c.dd = p.storage == ISKV_F32 ? 1 : 0;
  c.tol_floor = core_tol_floor(p.storage, true);
  e = launch_core(reinterpret_cast<const char *>(jobs), c, s);
  if (e != cudaSuccess) return e;
  k_reorth_T<<<dim3(tn, tm, p.count * 2), 256, 0, s>>>(jobs, p);
  count_launches(1);
  stage_mark(s, ST_REORTH_CORE);

  RotParams q;
  q.d = p.d;
  q.r = r;
  q.storage = p.storage;
  q.count = p.count;
  q.job_stride = sizeof(ReorthJob);
  q.gt = W.TUt;
  q.gtb = W.TUtb;
  q.ht = W.TBt;
  q.pmat = W.TBt;  // unused: p = 0
  q.bn = W.Bn;
  q.hs = r;
  q.pld = 1;
  if (p.tc_host)
    e = launch_tc_rotation(p.tc_dev, p.count, r, p.n_cap, s);
  else
    e = launch_rotate_coords_ffma(reinterpret_cast<const char *>(jobs), q, p.n_cap, s);
  if (e != cudaSuccess) return e;
  stage_mark(s, ST_REORTH_COORDS);
  if (p.tc_basis)
    e = launch_tc_basis(p.basis_dev, p.count, p.d, r, r, s);
  else
    e = launch_rotate_basis(reinterpret_cast<const char *>(jobs), q, s);
  if (e != cudaSuccess) return e;
  with_dtype(p.storage, [&](auto ts) {
    k_reorth_finalize<decltype(ts)><<<dim3(32, p.count), 256, 0, s>>>(jobs, p);
  });
  count_launches(1);
  stage_mark(s, ST_REORTH_BASIS);
  return cudaGetLastError();
}

}  // namespace iskv
