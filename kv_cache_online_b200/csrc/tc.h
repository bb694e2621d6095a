// Tensor-core (tcgen05) path: job table and host launchers.
#pragma once

#include <cuda.h>

#include <vector>

#include "attention.h"
#include "kernels.h"
#include "recon.h"

namespace iskv {

// One tensor-core job: two TMA descriptors plus the pointers its epilogue needs. 64-byte aligned
// (TMA descriptors must be); lives in the caller's workspace.
struct alignas(64) TcJob {
  CUtensorMap mapA;      // U [n_cap][r] bf16 (basis rotation: B [d][r]), box {64, 128}
  CUtensorMap mapB;      // rotation: G^T [r][r] fp16 (basis: H^T [r][kpad]), box {64, r};
                         // reconstruction: sigma B [d][r]
  CUtensorMap mapO;      // reconstruction: out [n_total][d] bf16, box {64, 32} (tile stores);
                         // basis rotation: P [d][bpad] fp16, box {64, 128}
  CUtensorMap mapS;      // rotations: the output (U or B) bf16, box {64, 32} (tile stores)
  void *U;               // rotation output (in place)
  const int32_t *sc;     // rotation: the job's FS_* scalars
  void *out;             // reconstruction output [n_total][d] bf16
  const int32_t *pos;    // reconstruction: row positions
  int64_t *meta;         // status word target
  int64_t n_total;
  int32_t rope;
  int32_t tiles_ok;      // reconstruction: mapO is encoded (n_total >= 32), tile stores allowed
  float *S;              // attention scores: [n_q][n_total] float32 by position
  const float *q;        // attention scores: queries [n_q][128] float32
  float scale;           // attention scores: score scale
};

struct TcParams {
  int r, d, n_heads, count, tiles_per_job;
  int hp, stages;  // reconstruction: heads per CTA, U slab ring depth; rotations: A slab ring depth
  int kslabs;      // rotations: 64-wide K slabs per tile
  int mode;        // rotations: 0 coordinate (rows n of U), 1 basis (rows d of B)
  int stg;         // rotations: 1 = each epilogue warp stages 32 x 64 outputs for a tile store
  double theta;
};

// Gram partials for the re-orthogonalisation: `count` jobs, each with nsu splits of U rows and nsb
// splits of B rows (`split` rows each); outputs at byte offsets off_gu / off_gb of the job's
// workspace (TcJob::out), one r x r float32 matrix per split.
struct GramParams {
  int r, d, count;
  int nsu;    // U chunks per job: n rows in gram_chunk(n, nsu)-row chunks
  int nsb;    // B chunks per job of `split` rows
  int split;
  size_t off_gu, off_gb;
  size_t off_g1;  // with nsb == 1: B's Gram goes straight to this workspace offset (no partial)
};

// Rows per U chunk when n rows are split into nsu balanced chunks (whole 64-row stages).
__host__ __device__ inline int gram_chunk(int n, int nsu) {
  const int c = (n + nsu - 1) / nsu;
  return c < 64 ? 64 : (c + 63) / 64 * 64;
}

bool tc_gram_supported(int r, int storage);
int tc_sm_count();  // SMs of the current device
bool encode_gram_job(TcJob &tj, const void *U, int64_t n_cap, const void *B, int d, int r,
                     const int32_t *sc, int64_t *meta, void *ws);
// The launchers take job tables already uploaded to the device (upload_jobs).
cudaError_t launch_tc_gram(const TcJob *djobs, const GramParams &p, cudaStream_t s);

bool tc_rotation_supported(int r, int storage);

// Projection of the fold (Algorithm 2 steps 2-3) on the tensor cores: bf16 factors, bf16 block,
// b = 64, r = 128 or 256, d a multiple of 128 up to 1024; one CTA per history. Outputs C [b][r]
// and E [b][d] (float32) in the job's fold workspace; E1 [2b][d] bf16 is its scratch.
struct alignas(64) ProjJob {
  CUtensorMap mapBm;     // B [d][r] bf16, box {64, 64} (read MN-major: B^T as the A operand)
  CUtensorMap mapBk;     // B [d][r] bf16, box {64, 128} (read K-major)
  CUtensorMap mapF;      // F [b][d] bf16, box {64, 64}
  CUtensorMap mapE1;     // E1 [2b][d] bf16 (hi rows, then lo rows), box {64, 64}
  __nv_bfloat16 *B;
  const __nv_bfloat16 *F;
  float *C, *E;
  __nv_bfloat16 *E1;
  const int32_t *sc;     // the job's FS_* scalars
  int64_t *meta;
};
struct ProjParams {
  int r, d, count;
};
bool tc_project_supported(int d, int r, int b, int storage, int f_dtype);
bool encode_project_job(ProjJob &pj, void *B, int d, int r, const void *F, int b, float *C,
                        float *E, void *E1, const int32_t *sc, int64_t *meta);
cudaError_t launch_tc_project(const ProjJob *djobs, int count, int d, int r, cudaStream_t s);

// Basis rotation of the fold on the tensor cores: B[0:d] <- [B | P] H in place (bf16 factors,
// fp16 operands), with P (d x bpad) and H^T (r x kpad, kpad = r + bpad) as fp16 in the fold
// workspace. Job
// fields: mapA (B, d x r), mapO (Pb, d x bpad), mapB (Htb, r x kpad), U (= B, the output), sc.
// With bpad = 0 (no mapO) it is the re-orthogonalisation's B <- B T_B.
bool tc_basis_supported(int r, int bpad, int storage);
bool encode_basis_job(TcJob &tj, void *B, int d, int r, const void *Pb, int bpad,
                      const void *Htb, const int32_t *sc, int64_t *meta);
cudaError_t launch_tc_basis(const TcJob *djobs, int count, int d, int r, int kpad, cudaStream_t s);
bool tc_recon_supported(int r, int storage, int out_dtype, int head_dim);

bool encode_rotation_job(TcJob &tj, void *U, int64_t n_cap, int r, const void *gtb,
                         const int32_t *sc, int64_t *meta);
bool encode_recon_job(TcJob &tj, const void *U, int64_t n_cap, int r, const void *bsig, int d,
                      void *out, const int32_t *pos, int64_t *meta, int64_t n_total, int rope);

cudaError_t launch_tc_rotation(const TcJob *djobs, int count, int r, int64_t n_cap_max,
                               cudaStream_t s);
// Sigma-scaled basis for every job (the operand of launch_tc_recon); stage "reconstruct.prepare".
cudaError_t launch_recon_bsig(const ReconJob *djobs_recon, const ReconParams &p, cudaStream_t s);
cudaError_t launch_tc_recon(const TcJob *djobs, const ReconParams &p, cudaStream_t s);

// Decode-attention scores of compressed keys (the reconstruction kernel with a scores epilogue):
// bf16 factors, head_dim 128, r a multiple of 64 up to 256, 1, 2, 4 or 8 query heads per KV head.
bool tc_attn_supported(int r, int storage, int head_dim, int n_q, int n_kv);
bool encode_attn_job(TcJob &tj, const void *U, int64_t n_cap, int r, const void *bsig, int d,
                     float *S, const float *q, const int32_t *pos, int64_t *meta, int64_t n_total,
                     float scale);
cudaError_t launch_tc_attn_scores(const TcJob *djobs, const AttnParams &p, cudaStream_t s);

// Decode-attention value mixing: per split of ATTN_CHUNK rows, U^T P -> [split][r][64] float32.
struct PvParams {
  int r, count, nsplit;
};
bool tc_pv_supported(int r, int storage, int n_q);
bool encode_pv_job(TcJob &tj, const void *U, int64_t n_cap, int r, const void *Pb, float *wpart,
                   int64_t *meta);
cudaError_t launch_tc_pv(const TcJob *djobs, const PvParams &p, cudaStream_t s);

// One CTA waiting on a barrier nothing arrives at, bounded by limit_ns (failure-path self-test).
cudaError_t launch_wait_timeout(int64_t *meta, uint64_t limit_ns, cudaStream_t s);

inline size_t tc_table_bytes(int count) { return ((size_t)count * sizeof(TcJob) + 255) / 256 * 256; }

}  // namespace iskv
