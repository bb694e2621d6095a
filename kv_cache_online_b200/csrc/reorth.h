// Re-orthogonalisation: workspace layout and launcher.
#pragma once

#include "kernels.h"
#include "tc.h"

namespace iskv {

constexpr int REORTH_SPLIT = 2048;  // rows per Gram partial
constexpr int NS_ITERS = 5;         // coupled Newton-Schulz iterations

struct ReorthWsLayout {
  size_t scal, gpart_u, gpart_b, G[2], Y[2], Z[2], T[2], Y2[2], Z2[2], M, Gt, Gtb, Ht, sig, TUt,
      TUtb, TBt, TBtb, Bn, total;
  int nsplit_u, nsplit_b;
};

ReorthWsLayout reorth_ws_layout(int d, int r, int64_t n_cap);

struct ReorthParams {
  int d, r, storage, count;
  int64_t n_cap;
  ReorthWsLayout ws;
  const TcJob *tc_host;    // tensor-core coordinate rotation jobs (host copy) or null
  TcJob *tc_dev;           // their device table
  const TcJob *gram_host;  // tensor-core Gram jobs (host copy) or null
  TcJob *gram_dev;         // their device table
  int gram_nsu;            // tensor-core Gram: U chunks per job (balanced); 0: REORTH_SPLIT rows
  int tc_basis;            // 1: B <- B T_B on the tensor cores, in place (jobs in basis_dev)
  TcJob *basis_dev;
};

cudaError_t launch_reorth(const ReorthJob *jobs, const ReorthParams &p, cudaStream_t s);

// Diagnostics (iS-KV reading notes, Section 5.1 eq. 12 and the orthogonality the re-
// orthogonalisation restores): ||U^T U - I||_F and ||B^T B - I||_F over the current rank from the
// same Gram kernels, and the persistent bytes s_f (n k + d k + k) + s_e n_exact d of each history.
cudaError_t launch_diagnostics(const ReorthJob *jobs, const ReorthParams &p, int exact_bytes,
                               double *orth_u, double *orth_b, int64_t *pbytes, cudaStream_t s);

}  // namespace iskv
