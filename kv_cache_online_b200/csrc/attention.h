// Decode attention over the compressed cache: job table and launchers.
#pragma once

#include "kernels.h"

namespace iskv {

// One (sequence, layer) job: the K and V histories, the exact rows of both caches, the decode
// query and the output, plus this job's workspace slices.
struct AttnJob {
  const void *Uk;            // K history: U [n_cap][rk], sigma [rk], B [d][rk], pos [n_cap], meta
  const float *sk;
  const void *Bk;
  const int32_t *posk;
  int64_t *metak;
  const void *Uv;            // V history: U [n_cap][rv], sigma [rv], B [d][rv], pos, meta
  const float *sv;
  const void *Bv;
  const int32_t *posv;
  int64_t *metav;
  const void *kex;           // exact keys [n_kex][d] (pre-RoPE) at kexpos
  const int32_t *kexpos;
  const void *vex;           // exact values [n_vex][d] at vexpos
  const int32_t *vexpos;
  const float *q;            // [n_q][head_dim] float32, already rotated for the query position
  float *out;                // [n_q][head_dim] float32
  float *S;                  // workspace [n_q][n_total]: scores by position (-inf where no key)
  float *stats;              // workspace [n_q][2]: max score, sum of exp(score - max)
  float *wpart;              // workspace [nchunk][n_q][rv]: partial sums of p * U_v rows
  float *mpart;              // workspace [nchunk][n_q]: partial probability mass on V rows
  float *P;                  // workspace [n_q][n_cap]: probabilities at the compressed V rows
  void *Pb;                  // the same workspace as bf16 [n_cap][64] (tensor-core value mixing)
  float *opart;              // workspace [AO_SPLIT][n_q][head_dim]: partial outputs
  float *omass;              // workspace [AO_SPLIT][n_q]: partial probability mass
  void *bsig;                // workspace: sigma-scaled K basis (tensor-core scores)
  int64_t n_kex, n_vex, n_total;
};

struct AttnParams {
  int d, storage, exact_dtype, n_kv, n_q, head_dim, count, nchunk;
  int rk, rv;      // rank budgets (row strides of U and B) of the K and of the V histories
  int nblk;        // probability-mass partials: blocks of 256 * ATTN_PROB_ROWS value rows
  int tc_values;   // value mixing on the tensor cores (partials [chunk][rv][64])
  double theta;
  float scale;
  int64_t n_cap_max, n_total_max;
};

constexpr int ATTN_CHUNK = 2048;  // V rows per value-mixing block
constexpr int ATTN_MAX_Q = 64;   // query heads
constexpr int ATTN_PROB_ROWS = 8;  // value rows per thread in the probability kernel
constexpr int AO_SPLIT = 8;        // output parts per (KV head, job)

cudaError_t launch_attn_init(const AttnJob *jobs, const AttnParams &p, cudaStream_t s);
cudaError_t launch_attn_scores_ffma(const AttnJob *jobs, const AttnParams &p, cudaStream_t s);
cudaError_t launch_attn_scores_exact(const AttnJob *jobs, const AttnParams &p, int64_t max_kex,
                                     cudaStream_t s);
cudaError_t launch_attn_stats(const AttnJob *jobs, const AttnParams &p, cudaStream_t s);
cudaError_t launch_attn_probs(const AttnJob *jobs, const AttnParams &p, cudaStream_t s);
cudaError_t launch_attn_values(const AttnJob *jobs, const AttnParams &p, cudaStream_t s);
cudaError_t launch_attn_out(const AttnJob *jobs, const AttnParams &p, cudaStream_t s);

}  // namespace iskv
