// Host-side launchers shared between the translation units of libiskv.
#pragma once

#include "common.cuh"

namespace iskv {

// Uniform parameters of a (batched) fold.
struct FoldParams {
  int d, r, b;          // feature width, rank budget (row stride of U and B), block rows
  int f_dtype, storage; // iskv_dtype of F and of U/B
  int count;            // number of jobs
  float tau_rel;        // residual threshold floor (relative)
  FoldWsLayout ws;      // per-job workspace layout
  int tc_basis;         // 1: the basis rotation ran on the tensor cores and wrote B in place
};

// Operands of the two rotations, as byte offsets into each job's workspace. The job's scalars
// (FS_*) give n, k before, k after, and the residual count p.
struct RotParams {
  int d, r, storage, count, job_stride;
  size_t gt, gtb;   // coordinate rotation: row q holds G[0:k, q] (float32 / fp16), row stride r
  size_t ht;        // basis rotation: row q holds H[0:k+p, q], row stride hs
  size_t pmat;      // residual basis P (d x p), row stride pld (unused when p = 0)
  size_t bn;        // basis rotation output (d x r float32)
  int hs, pld;
};

// One-sided Jacobi core SVD.
struct CoreParams {
  int r, b, count, job_stride;
  int mode;         // 0: fold core [[diag sigma, 0], [C, F P]]; 1: dense k x k matrix M
  size_t C, FP, M;  // inputs (mode 0: C [b][r], FP [b][b]; mode 1: M [k][ldm])
  size_t Gt, Gtb, Gbot, Ht, sig;  // outputs
  int hs, ldm, max_sweeps;
  int dd;           // 1: inner products accumulated in float64 (tighter tolerance), 0: float32
  float tol_floor;  // smallest cosine tolerance (see core_tol_floor)
};

// Floor of the core SVD's cosine tolerance for factors stored as `storage`. The rotations G and H
// a fold's core returns reach the two-byte factors through that storage's rounding (relative
// 2^-9 for bf16, 2^-11 for fp16; the tensor-core rotation also takes G as bf16), so column pairs
// whose cosine is already a sixteenth of it are left alone: the kept singular values move by the
// square of such a cosine (below 1e-8), the represented rows by less than the storage rounding.
// The re-orthogonalisation's core exists to make the factors orthonormal again, so its floor is
// a sixty-fourth of the bf16 rounding and none for fp16 (whose rounding is four times finer).
// float32 factors keep the float32 tolerance (no floor).
__host__ __device__ inline float core_tol_floor(int storage, bool reorth) {
  if (reorth) return storage == ISKV_BF16 ? 0x1p-15f : 0.f;
  return storage == ISKV_BF16 ? 0x1p-13f : (storage == ISKV_F16 ? 0x1p-15f : 0.f);
}

struct JacobiCfg {
  int cj;         // CTAs per cluster
  int w;          // columns per block (two blocks per CTA)
  int ne;         // column elements per lane (column buffer = 32 * ne floats)
  bool dbuf;      // double-buffered block exchange (one cluster barrier per round)
  size_t smem;    // dynamic shared memory bytes
};

JacobiCfg jacobi_cfg(int ncols_max, int col_len_max);
// Configuration of the core SVD for r_max = r and block b (fold) or of the dense r x r core
// (re-orthogonalisation); false when no cluster shape fits.
bool core_cfg(int r, int b, bool dense, JacobiCfg &c);
size_t fold_residual_smem(int d, int b);

cudaError_t launch_fold_prepare(const FoldJob *jobs, const FoldParams &p, cudaStream_t s);
cudaError_t launch_fold_project(const FoldJob *jobs, const FoldParams &p, cudaStream_t s);
cudaError_t launch_fold_residual(const FoldJob *jobs, const FoldParams &p, cudaStream_t s);
cudaError_t launch_fold_finalize(const FoldJob *jobs, const FoldParams &p, cudaStream_t s);
// Operands of the tensor-core basis rotation: P and H as bf16 in the padded layout of
// FoldWsLayout (Pb, Htb), and B's columns from k on zeroed.
cudaError_t launch_basis_prep(const FoldJob *jobs, const FoldParams &p, cudaStream_t s);

cudaError_t launch_core(const char *jobs, const CoreParams &p, cudaStream_t s);
// Core SVD work counters: CORE_STATS values per mode (see jacobi_core.cu), synchronous read.
constexpr int CORE_STATS = 6;
cudaError_t core_stats(long long *out, bool reset);
cudaError_t launch_rotate_basis(const char *jobs, const RotParams &p, cudaStream_t s);
cudaError_t launch_rotate_coords_ffma(const char *jobs, const RotParams &p, int64_t n_cap_max,
                                      cudaStream_t s);

// Upload a host array of job descriptors into device memory at `dst` with plain kernel launches
// (no pageable memcpy), so that the call stays stream-ordered.
cudaError_t upload_jobs(void *dst, const void *src, size_t bytes, cudaStream_t s);

RotParams fold_rot_params(const FoldParams &p);
CoreParams fold_core_params(const FoldParams &p);

}  // namespace iskv
