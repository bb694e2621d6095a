// Reconstruction job descriptors and launchers (shared by the API and the kernels).
#pragma once

#include "common.cuh"

namespace iskv {

struct ReconJob {
  const void *U;
  const float *sigma;
  const void *B;
  const int32_t *pos;
  int64_t *meta;
  const void *exact_rows;
  const int32_t *exact_pos;
  void *out;
  void *bsig;          // workspace: sigma-scaled basis for the tensor-core path
  int64_t n_exact;
  int64_t n_total;
  int32_t apply_rope;
  int32_t pad_;
};

struct ReconParams {
  int d, r, storage, exact_dtype, out_dtype, n_heads, head_dim, count;
  int exact_vec;  // exact rows move as 16-byte vectors (head_dim % 16 == 0, 16-byte aligned rows)
  double theta;
  int64_t n_cap_max;
};

cudaError_t launch_recon_compressed_ffma(const ReconJob *jobs, const ReconParams &p,
                                         cudaStream_t s);
cudaError_t launch_recon_compressed(const ReconJob *jobs, const ReconParams &p, cudaStream_t s);
cudaError_t launch_recon_exact(const ReconJob *jobs, const ReconParams &p, int64_t max_exact,
                               cudaStream_t s);

}  // namespace iskv
