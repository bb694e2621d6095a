// Fold stages that are small dense contractions or bookkeeping (iS-KV reading notes, Section 4,
// Algorithm 2): job upload, capacity check, projection and twice-subtracted residual (steps 2-3),
// basis rotation B <- [B, P] H (step 8), CUDA-core coordinate rotation (step 7), and the final
// write-back of the new factors, positions and meta word (steps 8-9). The basis and coordinate
// rotations also serve the re-orthogonalisation (Section 4.4) through RotParams offsets.
#include <cstring>

#include "gemm_tile.cuh"
#include "kernels.h"
#include "profiling.h"

namespace iskv {

// ------------------------------------------------------------------------------------------------
// Job upload: a host array travels as kernel parameters (up to 32736 bytes per launch, inside the
// 32764-byte parameter limit), so the copy is stream-ordered and needs no host buffer to outlive
// the call. Parameters live in a constant bank, where a warp's distinct addresses are served one
// at a time: the copy moves 16-byte words to keep that count low.
struct alignas(16) UploadChunk {
  unsigned char data[32736];
};

__global__ void k_upload(unsigned char *dst, UploadChunk c, int nbytes) {
  const int words = nbytes / 16;  // dst is 16-byte aligned (workspace tables, chunk offsets)
  const uint4 *src4 = reinterpret_cast<const uint4 *>(c.data);
  uint4 *dst4 = reinterpret_cast<uint4 *>(dst);
  for (int i = threadIdx.x; i < words; i += blockDim.x) dst4[i] = src4[i];
  for (int i = words * 16 + threadIdx.x; i < nbytes; i += blockDim.x) dst[i] = c.data[i];
}

cudaError_t upload_jobs(void *dst, const void *src, size_t bytes, cudaStream_t s) {
  const unsigned char *p = static_cast<const unsigned char *>(src);
  for (size_t off = 0; off < bytes; off += sizeof(UploadChunk)) {
    UploadChunk c;
    const size_t n = bytes - off < sizeof(UploadChunk) ? bytes - off : sizeof(UploadChunk);
    std::memcpy(c.data, p + off, n);
    k_upload<<<1, 256, 0, s>>>(static_cast<unsigned char *>(dst) + off, c, (int)n);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

RotParams fold_rot_params(const FoldParams &p) {
  RotParams q;
  q.d = p.d;
  q.r = p.r;
  q.storage = p.storage;
  q.count = p.count;
  q.job_stride = sizeof(FoldJob);
  q.gt = p.ws.Gt;
  q.gtb = p.ws.Gtb;
  q.ht = p.ws.Ht;
  q.pmat = p.ws.P;
  q.bn = p.ws.Bn;
  q.hs = p.ws.hs;
  q.pld = p.b;
  return q;
}

// ------------------------------------------------------------------------------------------------
// Capacity check and snapshot of k, n (read by every later stage of the same fold).
__global__ void k_fold_prepare(const FoldJob *jobs, FoldParams p) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= p.count) return;
  const FoldJob &jb = jobs[j];
  int32_t *sc = reinterpret_cast<int32_t *>(jb.h.ws + p.ws.scal);
  const int64_t k = jb.h.meta[ISKV_META_K], n = jb.h.meta[ISKV_META_N];
  sc[FS_K_OLD] = (int32_t)k;
  sc[FS_N_OLD] = (int32_t)n;
  sc[FS_SKIP] = (n < 0 || n + p.b > jb.n_cap || k > p.r || k < 0) ? 1 : 0;
  sc[FS_P] = 0;
  sc[FS_K_NEW] = (int32_t)k;
  sc[FS_SWEEPS] = 0;
  sc[FS_RSWEEPS] = 0;
}

cudaError_t launch_fold_prepare(const FoldJob *jobs, const FoldParams &p, cudaStream_t s) {
  k_fold_prepare<<<(p.count + 127) / 128, 128, 0, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Steps 2-3: C = F B; E = F - C B^T; C2 = E B; E <- E - C2 B^T (float32 accumulation).
constexpr int PBM = 32, PBN = 64, PBK = 16, PTM = 2, PTN = 4;  // 256 threads

template <int STAGE, typename TF, typename TS>
__global__ void __launch_bounds__(256) k_fold_project(const FoldJob *jobs, FoldParams p) {
  const FoldJob &jb = jobs[blockIdx.z];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws + p.ws.scal);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], d = p.d, r = p.r, b = p.b;
  const TF *F = static_cast<const TF *>(jb.F);
  const TS *B = static_cast<const TS *>(jb.h.B);
  float *C = reinterpret_cast<float *>(jb.h.ws + p.ws.C);
  float *E = reinterpret_cast<float *>(jb.h.ws + p.ws.E);
  float *C2 = reinterpret_cast<float *>(jb.h.ws + p.ws.C2);
  const int m0 = blockIdx.y * PBM, n0 = blockIdx.x * PBN;
  auto lb_n = [&](int kk, int n) { return to_f<TS>(B[(size_t)kk * r + n]); };   // B (d x k)
  auto lb_t = [&](int kk, int n) { return to_f<TS>(B[(size_t)n * r + kk]); };   // B^T (k x d)
  if (STAGE == 0) {
    if (n0 >= k) return;
    tile_gemm<PBM, PBN, PBK, PTM, PTN, true, true>(
        m0, n0, b, k, d, [&](int m, int kk) { return to_f<TF>(F[(size_t)m * d + kk]); }, lb_n,
        [&](int m, int n, float acc) { C[(size_t)m * r + n] = acc; });
  } else if (STAGE == 1) {
    tile_gemm<PBM, PBN, PBK, PTM, PTN, true, false>(
        m0, n0, b, d, k, [&](int m, int kk) { return C[(size_t)m * r + kk]; }, lb_t,
        [&](int m, int n, float acc) {
          E[(size_t)m * d + n] = to_f<TF>(F[(size_t)m * d + n]) - acc;
        });
  } else if (STAGE == 2) {
    if (n0 >= k) return;
    tile_gemm<PBM, PBN, PBK, PTM, PTN, true, true>(
        m0, n0, b, k, d, [&](int m, int kk) { return E[(size_t)m * d + kk]; }, lb_n,
        [&](int m, int n, float acc) { C2[(size_t)m * r + n] = acc; });
  } else {
    if (k == 0) return;
    tile_gemm<PBM, PBN, PBK, PTM, PTN, true, false>(
        m0, n0, b, d, k, [&](int m, int kk) { return C2[(size_t)m * r + kk]; }, lb_t,
        [&](int m, int n, float acc) { E[(size_t)m * d + n] -= acc; });
  }
}

template <typename TF, typename TS>
static cudaError_t project_t(const FoldJob *jobs, const FoldParams &p, cudaStream_t s) {
  const dim3 gk((p.r + PBN - 1) / PBN, (p.b + PBM - 1) / PBM, p.count);
  const dim3 gd((p.d + PBN - 1) / PBN, (p.b + PBM - 1) / PBM, p.count);
  k_fold_project<0, TF, TS><<<gk, 256, 0, s>>>(jobs, p);
  k_fold_project<1, TF, TS><<<gd, 256, 0, s>>>(jobs, p);
  k_fold_project<2, TF, TS><<<gk, 256, 0, s>>>(jobs, p);
  k_fold_project<3, TF, TS><<<gd, 256, 0, s>>>(jobs, p);
  count_launches(4);
  return cudaGetLastError();
}

cudaError_t launch_fold_project(const FoldJob *jobs, const FoldParams &p, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  with_dtype(p.f_dtype, [&](auto tf) {
    with_dtype(p.storage, [&](auto ts) {
      e = project_t<decltype(tf), decltype(ts)>(jobs, p, s);
    });
  });
  return e;
}

// ------------------------------------------------------------------------------------------------
// Basis rotation: Bn = [B, P] H  (d x k'), K = k + p, in 64 x 64 tiles (4 x 4 per thread). Written
// to workspace and copied into B afterwards, so that no tile reads basis columns another tile is
// overwriting.
constexpr int RBM = 64, RTM = 4;
template <typename TS>
__global__ void __launch_bounds__(256) k_rotate_basis(const char *jobs, RotParams p) {
  const JobHead &jh = job_head(jobs, p.job_stride, blockIdx.z);
  const int32_t *sc = reinterpret_cast<const int32_t *>(jh.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], pp = sc[FS_P], kn = sc[FS_K_NEW];
  const int r = p.r, pld = p.pld, hs = p.hs;
  const int m0 = blockIdx.y * RBM, n0 = blockIdx.x * PBN;
  if (n0 >= kn) return;
  const TS *B = static_cast<const TS *>(jh.B);
  const float *P = reinterpret_cast<const float *>(jh.ws + p.pmat);
  const float *Ht = reinterpret_cast<const float *>(jh.ws + p.ht);
  float *Bn = reinterpret_cast<float *>(jh.ws + p.bn);
  tile_gemm<RBM, PBN, PBK, RTM, PTN, true, false>(
      m0, n0, p.d, kn, k + pp,
      [&](int m, int l) {
        return l < k ? to_f<TS>(B[(size_t)m * r + l]) : P[(size_t)m * pld + (l - k)];
      },
      [&](int l, int q) { return Ht[(size_t)q * hs + l]; },
      [&](int m, int q, float acc) { Bn[(size_t)m * r + q] = acc; });
}

cudaError_t launch_rotate_basis(const char *jobs, const RotParams &p, cudaStream_t s) {
  const dim3 g((p.r + PBN - 1) / PBN, (p.d + RBM - 1) / RBM, p.count);
  with_dtype(p.storage, [&](auto ts) { k_rotate_basis<decltype(ts)><<<g, 256, 0, s>>>(jobs, p); });
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Operands of the tensor-core basis rotation (bf16 factors): P as fp16 with zero columns from p to
// bpad, and H^T as fp16 laid out against the K order [B columns 0 .. r-1 | P columns 0 .. bpad-1]: row q
// (an output column) holds H's entries for B columns l < k at l and for P columns c < p at r + c,
// zeros elsewhere and in every row q >= k'. B's columns k .. r-1 are cleared (they are zero after
// every fold and re-orthogonalisation; clearing them keeps a stray non-finite value there from
// reaching the products through a zero weight).
__global__ void __launch_bounds__(256) k_basis_prep(const FoldJob *jobs, FoldParams p) {
  const FoldJob &jb = jobs[blockIdx.y];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws + p.ws.scal);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], pp = sc[FS_P], kn = sc[FS_K_NEW];
  const int r = p.r, d = p.d, bpad = p.ws.bpad, kpad = p.ws.kpad, hs = p.ws.hs, pld = p.b;
  const float *P = reinterpret_cast<const float *>(jb.h.ws + p.ws.P);
  const float *Ht = reinterpret_cast<const float *>(jb.h.ws + p.ws.Ht);
  __half *Pb = reinterpret_cast<__half *>(jb.h.ws + p.ws.Pb);
  __half *Htb = reinterpret_cast<__half *>(jb.h.ws + p.ws.Htb);
  __nv_bfloat16 *B = static_cast<__nv_bfloat16 *>(jb.h.B);
  const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
  for (int e = tid; e < d * bpad; e += nth) {
    const int i = e / bpad, c = e % bpad;
    Pb[e] = __float2half_rn(c < pp ? P[(size_t)i * pld + c] : 0.f);
  }
  for (int e = tid; e < r * kpad; e += nth) {
    const int q = e / kpad, l = e % kpad;
    float v = 0.f;
    if (q < kn) {
      if (l < k) v = Ht[(size_t)q * hs + l];
      else if (l >= r && l - r < pp) v = Ht[(size_t)q * hs + k + (l - r)];
    }
    Htb[e] = __float2half_rn(v);
  }
  const int w = r - k;
  if (w > 0)
    for (int e = tid; e < d * w; e += nth) B[(size_t)(e / w) * r + k + e % w] = __float2bfloat16_rn(0.f);
}

cudaError_t launch_basis_prep(const FoldJob *jobs, const FoldParams &p, cudaStream_t s) {
  k_basis_prep<<<dim3(64, p.count), 256, 0, s>>>(jobs, p);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Coordinate rotation with CUDA cores: U[0:n] <- U[0:n] G[0:k] in place. A CTA owns 32 whole rows:
// it stages them in shared memory before writing any of them, so no other CTA reads what it
// overwrites.
constexpr int CRM = 32;

template <typename TS>
__global__ void __launch_bounds__(256) k_rotate_coords_ffma(const char *jobs, RotParams p) {
  const JobHead &jh = job_head(jobs, p.job_stride, blockIdx.y);
  const int32_t *sc = reinterpret_cast<const int32_t *>(jh.ws);
  if (sc[FS_SKIP]) return;
  const int k = sc[FS_K_OLD], kn = sc[FS_K_NEW], n = sc[FS_N_OLD];
  const int r = p.r;
  const int i0 = blockIdx.x * CRM;
  if (i0 >= n || k == 0) return;
  extern __shared__ float sm[];
  float *As = sm;  // [CRM][r + 1]
  __shared__ float Bs[16][64 + 4];
  TS *U = static_cast<TS *>(jh.U);
  const float *Gt = reinterpret_cast<const float *>(jh.ws + p.gt);
  const int tid = threadIdx.x, ld = r + 1;
  for (int e = tid; e < CRM * k; e += 256) {
    const int i = e / k, l = e % k;
    As[i * ld + l] = (i0 + i < n) ? to_f<TS>(U[(size_t)(i0 + i) * r + l]) : 0.f;
  }
  __syncthreads();
  const int tr = tid / 16, tc = tid % 16;
  for (int q0 = 0; q0 < kn; q0 += 64) {
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int l0 = 0; l0 < k; l0 += 16) {
      for (int e = tid; e < 16 * 64; e += 256) {
        const int qq = e / 16, ll = e % 16;
        const int q = q0 + qq, l = l0 + ll;
        Bs[ll][qq] = (q < kn && l < k) ? Gt[(size_t)q * r + l] : 0.f;
      }
      __syncthreads();
      const int lmax = min(16, k - l0);
      for (int ll = 0; ll < lmax; ++ll) {
        const float a0 = As[tr * ld + l0 + ll], a1 = As[(tr + 16) * ld + l0 + ll];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float bv = Bs[ll][tc + 16 * j];
          acc[0][j] = fmaf(a0, bv, acc[0][j]);
          acc[1][j] = fmaf(a1, bv, acc[1][j]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = i0 + tr + 16 * i, q = q0 + tc + 16 * j;
        if (row < n && q < kn) store_checked(&U[(size_t)row * r + q], acc[i][j], jh.meta);
      }
  }
}

cudaError_t launch_rotate_coords_ffma(const char *jobs, const RotParams &p, int64_t n_cap_max,
                                      cudaStream_t s) {
  const dim3 g((unsigned)((n_cap_max + CRM - 1) / CRM), p.count);
  const size_t smem = sizeof(float) * CRM * (p.r + 1);
  cudaError_t e = cudaSuccess;
  with_dtype(p.storage, [&](auto ts) {
    using TS = decltype(ts);
    e = cudaFuncSetAttribute(k_rotate_coords_ffma<TS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e == cudaSuccess) k_rotate_coords_ffma<TS><<<g, 256, smem, s>>>(jobs, p);
  });
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Steps 8-9 write-back: B <- Bn (unless B was rotated in place), U[n:n+b] <- G[k:], pos[n:n+b] <- f_pos, sigma <- sigma+, meta.
template <typename TS>
__global__ void k_fold_finalize(const FoldJob *jobs, FoldParams p) {
  const FoldJob &jb = jobs[blockIdx.y];
  const int32_t *sc = reinterpret_cast<const int32_t *>(jb.h.ws + p.ws.scal);
  const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
  if (sc[FS_SKIP]) {
    if (tid == 0) record_status(jb.h.meta, ISKV_ERR_CAPACITY);
    return;
  }
  const int kn = sc[FS_K_NEW];
  const int64_t n = sc[FS_N_OLD];
  const int r = p.r, d = p.d, b = p.b;
  TS *B = static_cast<TS *>(jb.h.B);
  TS *U = static_cast<TS *>(jb.h.U);
  const float *Bn = reinterpret_cast<const float *>(jb.h.ws + p.ws.Bn);
  const float *Gbot = reinterpret_cast<const float *>(jb.h.ws + p.ws.Gbot);
  const float *sig = reinterpret_cast<const float *>(jb.h.ws + p.ws.sig);
  if (!p.tc_basis)  // the tensor-core basis rotation wrote B in place
    for (int e = tid; e < d * r; e += nth) {
      const int q = e % r;
      store_checked(&B[e], q < kn ? Bn[e] : 0.f, jb.h.meta);
    }
  for (int e = tid; e < b * r; e += nth) {
    const int i = e / r, q = e % r;
    store_checked(&U[(size_t)(n + i) * r + q], q < kn ? Gbot[e] : 0.f, jb.h.meta);
  }
  for (int e = tid; e < b; e += nth) jb.h.pos[n + e] = jb.f_pos[e];
  for (int e = tid; e < r; e += nth) jb.h.sigma[e] = e < kn ? sig[e] : 0.f;
  if (tid == 0) {
    jb.h.meta[ISKV_META_K] = kn;
    jb.h.meta[ISKV_META_N] = n + b;
    jb.h.meta[ISKV_META_FOLDS] += 1;
  }
}

cudaError_t launch_fold_finalize(const FoldJob *jobs, const FoldParams &p, cudaStream_t s) {
  const dim3 g(32, p.count);
  with_dtype(p.storage, [&](auto ts) { k_fold_finalize<decltype(ts)><<<g, 256, 0, s>>>(jobs, p); });
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace iskv
