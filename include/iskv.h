/*
 * iskv.h -- C ABI of libiskv, the B200 (sm_100a) hot path of iS-KV online low-rank KV-cache
 * compression.
 *
 * Sources: "iS-KV reading notes" (zhongzhuzhou.org notes on "iS-KV: Online Low-Rank KV Cache
 * Compression via Block-Incremental SVD"), cited by section / algorithm / equation.
 *
 * Conventions for every entry point
 *  - All array arguments are DEVICE pointers unless a comment says "host". The caller owns all
 *    memory: the library never allocates on these paths; every call that needs scratch takes a
 *    caller workspace sized by the matching *_workspace_size() query.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t passed as void*; NULL = the
 *    legacy default stream). The return value reports argument errors found on the host
 *    (ISKV_ERR_ARG / ISKV_ERR_SHAPE / ISKV_ERR_WORKSPACE) or a failed kernel launch
 *    (ISKV_ERR_CUDA); nothing is launched when an error is returned.
 *  - Conditions found on the device (capacity, non-finite values, an unconverged Jacobi sweep, a
 *    bounded wait that ran out) are OR-ed into the history's device status word
 *    (meta[ISKV_META_STATUS], bit (1 << code)) and read back with iskv_get_status(), which syncs.
 *  - Matrices are row-major. Element types are given by iskv_dtype values.
 */
#ifndef ISKV_H
#define ISKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ISKV_ABI_VERSION 1

typedef enum {
  ISKV_OK = 0,
  ISKV_ERR_ARG = 1,            /* null pointer, bad enum, misaligned pointer                  */
  ISKV_ERR_SHAPE = 2,          /* inconsistent or unsupported sizes                           */
  ISKV_ERR_CUDA = 3,           /* a CUDA runtime call or kernel launch failed                 */
  ISKV_ERR_CAPACITY = 4,       /* device: n + b > n_cap, the fold was skipped; host: a cache
                                  table or history has no room for the step                    */
  ISKV_ERR_NONFINITE = 5,      /* device: a non-finite singular value came out of a fold      */
  ISKV_ERR_NOT_CONVERGED = 6,  /* device: Jacobi / Newton-Schulz hit its iteration cap        */
  ISKV_ERR_TIMEOUT = 7,        /* device: a bounded cluster wait gave up                      */
  ISKV_ERR_WORKSPACE = 8       /* workspace pointer null, misaligned or too small             */
} iskv_status;

/*
 * Element types of factors, blocks, exact rows and reconstruction outputs. The tensor-core kernels
 * take bf16 factors (and bf16 reconstruction outputs); float32 and fp16 run on CUDA cores. fp16 has
 * a maximum finite value of 65504 (Section 7.3: fp16 factors overflowed on long generations): U and
 * B have orthonormal columns and sigma stays float32 here, so stored factors stay below 1, but a
 * reconstructed cache can exceed it -- every store of a finite value that overflows fp16 records
 * ISKV_ERR_NONFINITE in the history's status word. Prompt keys for the selection are float32 or
 * bf16.
 */
typedef enum { ISKV_F32 = 0, ISKV_BF16 = 1, ISKV_F16 = 2 } iskv_dtype;

/* Indices into the device meta word of a history. */
enum { ISKV_META_K = 0, ISKV_META_N = 1, ISKV_META_FOLDS = 2, ISKV_META_STATUS = 3 };

/*
 * One compressed history: one (sequence, layer, K|V) path, the factors U diag(sigma) B^T of
 * Section 2.2 ("iS-KV reading notes"), rank k <= r_max, n compressed rows.
 *   U      [n_cap][r_max]  storage dtype; row i = coordinates of compressed row i. Must be
 *                          zero-initialised: columns >= k and rows >= n are read as zero.
 *   sigma  [r_max]         float32, descending; entries >= k are zero.
 *   B      [d][r_max]      storage dtype; column j = basis vector j. Zero-initialised.
 *   pos    [n_cap]         int32 original token position of U row i (Section 3.2: K and V
 *                          histories index different tokens, so rows are scattered by position).
 *   meta   [4]             int64 {k, n, folds since last reorth, status bits}; zero at creation.
 * All five pointers are device pointers, 16-byte aligned. d must be a multiple of 16 and r_max a
 * multiple of 16, 16 <= r_max <= min(d, 512).
 */
typedef struct {
  int32_t d;
  int32_t r_max;
  int64_t n_cap;
  int32_t storage; /* iskv_dtype of U and B */
  int32_t reserved;
  void *U;
  float *sigma;
  void *B;
  int32_t *pos;
  int64_t *meta;
} iskv_lowrank;

/* ABI version (ISKV_ABI_VERSION) and a static string naming a status code. */
int32_t iskv_abi_version(void);
const char *iskv_status_string(int32_t status);

/* Detail of the last host-side error on the calling thread (empty string if none). */
const char *iskv_last_error(void);

/*
 * Block fold -- Algorithm 2 of Section 4 ("iS-KV reading notes"): merge the pending block F of b
 * exact rows into the history, rotating the basis and EVERY history coordinate row together:
 *   C = F B;  E = F - C B^T;  E <- E - (E B) B^T;  Householder QR  E^T = Q_R R_R;  SVD of R_R;
 *   P = kept residual directions (rho_i > tol, tol = max(tau_rel, 2^-23 max(b,d)) * max(sigma_1,
 *   rho_1));  Z = [[diag sigma, 0], [F B, F P]];  Z = G diag(sigma+) H^T truncated to
 *   k' = min(r_max, k + p);  U[0:n] <- U[0:n] G[0:k];  U[n:n+b] <- G[k:];  B <- [B, P] H;
 *   pos[n:n+b] <- f_pos;  k <- k';  n <- n + b;  folds += 1.
 * F      [b][d] f_dtype (device). f_pos [b] int32 (device).
 * Sizes: 1 <= b <= min(d, 128), b % 8 == 0.
 * ws     caller workspace of at least iskv_fold_workspace_size(1, d, r_max, b) bytes, 256-byte
 *        aligned; its contents need no initialisation and are scratch after the call returns.
 * Device errors: n + b > n_cap -> the fold is a no-op and ISKV_ERR_CAPACITY is recorded;
 * non-finite new singular values -> ISKV_ERR_NONFINITE; Jacobi sweep cap -> ISKV_ERR_NOT_CONVERGED
 * (best-so-far result is kept).
 */
size_t iskv_fold_workspace_size(int32_t count, int32_t d, int32_t r_max, int32_t b);
iskv_status iskv_fold_block(const iskv_lowrank *h, const void *F, int32_t f_dtype, int32_t b,
                            const int32_t *f_pos, float tau_rel, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * The same fold for `count` independent histories in one set of launches (e.g. every layer's K
 * and V path when their pending queues fill on the same decode step, Algorithm 3 step 4).
 * hs, F, f_pos are HOST arrays of `count` entries (F[i], f_pos[i] are device pointers). All
 * histories share d, r_max, storage; all blocks share b and f_dtype. 1 <= count <= 4096.
 */
iskv_status iskv_fold_block_batched(const iskv_lowrank *hs, int32_t count, const void *const *F,
                                    int32_t f_dtype, int32_t b, const int32_t *const *f_pos,
                                    float tau_rel, void *ws, size_t ws_bytes, void *stream);

/*
 * The batched fold, pipelined behind readers of the current factors (no counterpart on the
 * pages; Algorithm 3 runs a step's reconstruction or attention between two folds). The stages
 * that only read the histories' factors (projection, residual QR and SVD, core SVD) start at once
 * on `stream`; the stages that change them (basis and coordinate rotations, write-back of U,
 * sigma, B, positions and meta) first wait for `factors_ready`, a cudaEvent_t the caller records
 * on the stream of its last reader of those factors (a reconstruction or decode attention issued
 * on another stream), or NULL. One exception: with bf16 factors and blocks the projection clears
 * B's columns k .. r_max-1 before the wait; this library leaves those columns zero, so their
 * values do not change. Arguments and errors otherwise as iskv_fold_block_batched.
 */
iskv_status iskv_fold_block_batched_after(const iskv_lowrank *hs, int32_t count,
                                          const void *const *F, int32_t f_dtype, int32_t b,
                                          const int32_t *const *f_pos, float tau_rel, void *ws,
                                          size_t ws_bytes, void *stream, void *factors_ready);

/*
 * Re-orthogonalisation -- Section 4.4: with orthonormal-basis factorisations U = Q_U R_U,
 * B = Q_B R_B, decompose R_U diag(sigma) R_B^T = X diag(sigma') Y^T and set U <- Q_U X,
 * sigma <- sigma', B <- Q_B Y. The product U diag(sigma) B^T is unchanged in exact arithmetic;
 * k and n are unchanged; meta[FOLDS] is reset to 0. hs is a HOST array of `count` handles sharing
 * d, r_max, storage and n_cap. Any r_max a history may have (<= 512) fits the dense r x r core
 * SVD's thread-block cluster.
 */
size_t iskv_reorth_workspace_size(int32_t count, int32_t d, int32_t r_max, int64_t n_cap);
iskv_status iskv_reorth(const iskv_lowrank *hs, int32_t count, void *ws, size_t ws_bytes,
                        void *stream);

/*
 * Reconstruction -- Algorithm 3 steps 7-8: out[pos[i], :] = (U[i] * sigma) B^T for the n
 * compressed rows, out[exact_pos[e], :] = exact_rows[e] for the n_exact exact rows; when
 * apply_rope != 0 every written row is then rotated by its own position with rotate-half RoPE
 * (pairs (j, j + head_dim/2) inside each head, angle pos * rope_theta^(-2j/head_dim)).
 * out          [n_total][d] out_dtype; rows not named by either set are left untouched. bf16 outputs
 *              that are 16-byte aligned take the tensor-core path; others a CUDA-core path.
 * exact_rows   [n_exact][d] exact_dtype (may be NULL when n_exact == 0); exact_pos [n_exact].
 * Positions must be distinct across both sets; a position outside [0, n_total) is not written and
 * ISKV_ERR_SHAPE is recorded in the history's status word.
 * d == n_heads * head_dim, head_dim even and <= 256.
 * ws           iskv_reconstruct_workspace_size(1, d, r_max) bytes (sigma-scaled basis).
 * hs and the per-job arrays of the batched form are HOST arrays of `count` entries.
 */
size_t iskv_reconstruct_workspace_size(int32_t count, int32_t d, int32_t r_max);
iskv_status iskv_reconstruct(const iskv_lowrank *h, const void *exact_rows, int32_t exact_dtype,
                             const int32_t *exact_pos, int64_t n_exact, int64_t n_total,
                             int32_t n_heads, int32_t head_dim, int32_t apply_rope,
                             double rope_theta, void *out, int32_t out_dtype, void *ws,
                             size_t ws_bytes, void *stream);
iskv_status iskv_reconstruct_batched(const iskv_lowrank *hs, int32_t count,
                                     const void *const *exact_rows, int32_t exact_dtype,
                                     const int32_t *const *exact_pos, const int64_t *n_exact,
                                     const int64_t *n_total, int32_t n_heads, int32_t head_dim,
                                     const int32_t *apply_rope, double rope_theta,
                                     void *const *out, int32_t out_dtype, void *ws,
                                     size_t ws_bytes, void *stream);

/*
 * Diagnostics -- Section 5.1 eq. (12) and the orthogonality Section 4.4 restores. For each history:
 *   orth_u[i] = ||U^T U - I||_F and orth_b[i] = ||B^T B - I||_F over the current rank k (float64
 *   from the Gram matrices the re-orthogonalisation computes, float32 accumulation; 0 for an empty
 *   history, NaN for an inconsistent one),
 *   persistent_bytes[i] = s_f (n k + d k + k) + exact_elem_bytes * n_exact[i] * d, s_f the factor
 *   element size (U, the shared basis and the diagonal of Sigma; the exact rows -- protected,
 *   recent, pending -- held beside the history; positions, reserved capacity, workspaces and any
 *   reconstructed cache are not counted).
 * orth_u, orth_b [count] float64 and persistent_bytes [count] int64 are DEVICE arrays; n_exact is a
 * HOST array of count entries or NULL (no exact rows). hs share d, r_max, storage and n_cap.
 * ws           iskv_diagnostics_workspace_size(count, d, r_max, n_cap) bytes, 256-byte aligned.
 */
size_t iskv_diagnostics_workspace_size(int32_t count, int32_t d, int32_t r_max, int64_t n_cap);
iskv_status iskv_diagnostics(const iskv_lowrank *hs, int32_t count, const int64_t *n_exact,
                             int32_t exact_elem_bytes, double *orth_u, double *orth_b,
                             int64_t *persistent_bytes, void *ws, size_t ws_bytes, void *stream);

/*
 * Decode attention over the compressed cache -- Algorithm 3 steps 7-9 without the dense cache
 * (Section 5.2 names this factor-aware form as the route to a speed-up). For one (sequence,
 * layer): the keys at every cached position are the compressed rows (U_k[i] sigma_k) B_k^T at
 * hk.pos[i] and the exact keys k_exact[e] at k_exact_pos[e], each rotated by its own position with
 * rotate-half RoPE (as iskv_reconstruct); the values are the compressed rows of hv at hv.pos and
 * the exact values at v_exact_pos (no rotation). For each query head j (KV head
 * h = j / (n_q_heads / n_kv_heads)):
 *   s_j(p) = scale * q[j] . key_p[h],  P_j = softmax over the key positions,
 *   out[j] = sum_p P_j(p) value_p[h],
 * where the compressed values are mixed in their r-dimensional coordinates and projected once:
 * sum_i P_j(pos_v[i]) (U_v[i] sigma_v) B_v,h^T. Scores are float32 from the stored factors (bf16
 * factors: the tensor-core kernel, keys never leave the SM); the softmax and mixing are float32.
 * q            [n_q_heads][head_dim] float32 device, already rotated for the query position.
 * out          [n_q_heads][head_dim] float32 device.
 * k_exact, v_exact  [n][d] exact_dtype device (NULL when n == 0); positions int32 device.
 * Positions must lie in [0, n_total); the K and V caches must cover the same positions: a key
 * position without a value leaves probability mass unaccounted (checked to 1e-3) and, like an
 * out-of-range position or a cache with no key at all, records ISKV_ERR_SHAPE in the status word
 * (hk for key-side conditions, hv for value-side ones). hk and hv share d, storage and n_cap;
 * their rank budgets may differ (the keys and values of a layer compressed at different ranks,
 * the separate K / V ranks of Section 8), but all hk of a batched call share one r_max and all hv
 * another. d == n_kv_heads * head_dim, head_dim even <= 256, n_q_heads a multiple of n_kv_heads,
 * <= 64 and at most 8 per KV head.
 * ws           iskv_attention_workspace_size(count, d, r_max, n_cap, max n_total, n_q_heads) bytes
 *              with r_max the larger of the K and V rank budgets, 256-byte aligned (scores by
 *              position, softmax statistics, partial value sums).
 * hk, hv and the per-job arrays of the batched form are HOST arrays of `count` entries.
 */
size_t iskv_attention_workspace_size(int32_t count, int32_t d, int32_t r_max, int64_t n_cap,
                                     int64_t n_total_max, int32_t n_q_heads);
iskv_status iskv_decode_attention(const iskv_lowrank *hk, const iskv_lowrank *hv,
                                  const void *k_exact, const int32_t *k_exact_pos,
                                  int64_t n_k_exact, const void *v_exact,
                                  const int32_t *v_exact_pos, int64_t n_v_exact,
                                  int32_t exact_dtype, int64_t n_total, int32_t n_q_heads,
                                  int32_t n_kv_heads, int32_t head_dim, double rope_theta,
                                  float scale, const float *q, float *out, void *ws,
                                  size_t ws_bytes, void *stream);
iskv_status iskv_decode_attention_batched(
    const iskv_lowrank *hk, const iskv_lowrank *hv, int32_t count, const void *const *k_exact,
    const int32_t *const *k_exact_pos, const int64_t *n_k_exact, const void *const *v_exact,
    const int32_t *const *v_exact_pos, const int64_t *n_v_exact, int32_t exact_dtype,
    const int64_t *n_total, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
    double rope_theta, float scale, const float *const *q, float *const *out, void *ws,
    size_t ws_bytes, void *stream);

/*
 * Prompt-block protection -- Section 3.1 and Algorithm 1 steps 2-4: blocks of `block` prompt
 * tokens; the last `suffix_blocks` full blocks and the partial tail are the local suffix; for each
 * KV head, score(block) = min over its tokens of cos(post-RoPE key, block-mean key) (float64,
 * cos = dot / max(|k||m|, 1e-30)); each head picks its `per_head` lowest (score, block index)
 * candidates (all if fewer); P_K = union over heads of the picked blocks' tokens plus the suffix;
 * P_V = every prompt position q with |p - q| <= v_radius for some p in P_K.
 * keys            [L][n_heads][head_dim] k_dtype, post-RoPE.
 * pk_out, pv_out  [L] int32: ascending positions (first n_pk / n_pv entries valid).
 * head_blocks_out [n_heads][per_head] int32: each head's picked blocks ascending, -1 padded.
 * counts_out      [2 + n_heads] int64: {n_pk, n_pv, n_picked[h]...}.
 * Limits: 1 <= L <= 2^24, n_heads <= 64, head_dim <= 256 and even, block in [1, 64],
 * per_head <= 4096.
 * Scores: once the call has run, the first n_heads * n_cand float64 values of ws hold the block
 * scores, head-major ([h][j], n_cand = max(L / block - suffix_blocks, 0) candidate blocks), for
 * callers that want to inspect them; the rest of ws is scratch.
 */
size_t iskv_select_workspace_size(int64_t L, int32_t n_heads, int32_t block);
iskv_status iskv_select_prompt_blocks(const void *keys, int32_t k_dtype, int64_t L,
                                      int32_t n_heads, int32_t head_dim, int32_t block,
                                      int32_t per_head, int32_t suffix_blocks, int32_t v_radius,
                                      int32_t *pk_out, int32_t *pv_out, int32_t *head_blocks_out,
                                      int64_t *counts_out, void *ws, size_t ws_bytes,
                                      void *stream);

/*
 * Prompt-block selection that allocates nothing and takes no workspace. No counterpart on the
 * pages: it exists for callers that cannot allocate device memory -- a plugin running inside a host
 * framework that owns all device memory and passes it only inputs and outputs, or a
 * latency-critical path where a cudaMalloc could synchronise the device. Same arguments, limits
 * and results as iskv_select_prompt_blocks() without ws / ws_bytes.
 *  - Scratch: a fixed device array of ISKV_NOALLOC_SCRATCH bytes inside the library, present on
 *    every GPU that loads it until the process exits. A size whose workspace
 *    (iskv_select_workspace_size) exceeds it is refused with ISKV_ERR_WORKSPACE; at 8 heads and
 *    8-token blocks that allows prompts up to about 230K tokens.
 *  - Calls no cudaMalloc, cudaFree or allocating library routine.
 *  - Every call looks up the array's device address (a host-side query) with the caller's
 *    device current, so the address stays right after the context is torn down and re-created
 *    (cudaDeviceReset). The first call on a device may load the library's device code there:
 *    make that first call before any stream capture on the device.
 *  - A refusal leaves its reason in iskv_last_error(), as for the other entry points.
 *  - All calls on a device share the array and it keeps the last call's contents (the parts that
 *    must start at zero are cleared by each call): calls that overlap on the GPU race and corrupt
 *    each other's results, so order them on one stream.
 */
#define ISKV_NOALLOC_SCRATCH (4u << 20)
iskv_status iskv_select_prompt_blocks_noalloc(const void *keys, int32_t k_dtype, int64_t L,
                                              int32_t n_heads, int32_t head_dim, int32_t block,
                                              int32_t per_head, int32_t suffix_blocks,
                                              int32_t v_radius, int32_t *pk_out, int32_t *pv_out,
                                              int32_t *head_blocks_out, int64_t *counts_out,
                                              void *stream);

/*
 * Cache policy: the exact rows of one side (K or V) of one (sequence, layer), and when its pending
 * rows are folded (Section 3.1, Section 3.2; Algorithm 1 steps 5-9, Algorithm 3 steps 1-6).
 *
 * A side keeps exact: its protected rows P_X (fixed at prefill), the rows at the `window` most recent
 * positions, and the pending FIFO (unprotected rows that have left the window and wait for a full
 * block of `block` rows). Readings: the window is the set of the W most recent positions; a
 * protected position inside it is stored once, as protected, and stays exact when it leaves; decode
 * rows are never protected; the window at prefill is no longer than W (empty for keys by
 * Algorithm 1 step 5, the last min(W, L) prompt positions for values), so at most one row joins
 * the FIFO per decode step. The value side's first refit (Algorithm 3 step 3; refit_rows = r_V > 0)
 * waits until refit_rows rows are pending and re-factors them, after the rows the history holds, by
 * a rank-r_V SVD; its rows do not count toward reorth_rows (Section 4.4). The device runs the refit
 * as ONE fold whose block is all refit_rows rows (Algorithm 2 on the history's rows followed by
 * them, truncated to r_max: exactly the refit) when the fold takes such a block (refit_rows <= 128,
 * r_max + refit_rows inside the core SVD cluster); otherwise, for an EMPTY history (the prompt's
 * values all protected, as with short prompts) and refit_rows <= r_max, as consecutive block folds
 * that never truncate, which is the same SVD. Other refits are refused.
 *
 * Exact-row table (device, caller-owned):
 *   rows [cap_e][d]  dtype; rows 0 .. n_prot-1 are the protected rows in ascending position, rows
 *                    n_prot .. n_prot+n_live-1 the live rows (FIFO, then the unprotected window
 *                    rows) in ascending position. 16-byte aligned; d * element size a multiple of
 *                    16 bytes.
 *   pos  [cap_e]     int32 positions of those rows. rows/pos are directly the exact_rows /
 *                    exact_pos arguments of iskv_reconstruct() and iskv_decode_attention(), with
 *                    n_exact = n_prot + n_live.
 * Host mirror (maintained by the library; the caller sets the first block of fields and live_host /
 * live_cap, then lets iskv_cache_prefill() fill the rest):
 *   live_host [live_cap]  HOST int32: positions of the live rows, ascending; live_cap >=
 *                         window + max(block, refit_rows).
 *   n_prot, n_live, last  counts and the last stored position (prompt length - 1 after prefill).
 *   fold_rows             rows merged by folds since the last re-orthogonalisation.
 *   hist_rows             rows of the side's history (prefill sets it to the compressed prompt
 *                         rows; each fold adds `block`); a fold that would pass the history's n_cap
 *                         is refused on the host before anything is launched.
 * The mirror lets the host decide, without reading the device, which tables fold in a step.
 */
typedef struct {
  int32_t d;
  int32_t window;      /* W: the most recent W positions stay exact                         */
  int32_t block;       /* b: rows per fold, as iskv_fold_block() accepts                    */
  int32_t reorth_rows; /* re-orthogonalise after this many folded rows; 0 = never           */
  int32_t dtype;       /* iskv_dtype of rows                                                */
  int32_t refit_rows;  /* r_V: rows of the value side's first refit; 0 = no refit           */
  int64_t cap_e;       /* row capacity of rows / pos                                        */
  void *rows;
  int32_t *pos;
  int32_t *live_host;  /* host */
  int64_t live_cap;
  int64_t n_prot;
  int64_t n_live;
  int64_t last;
  int64_t fold_rows;
  int64_t hist_rows;
  int64_t refit_done;  /* 1 once the first refit has run (or when refit_rows == 0)           */
} iskv_exact_table;

/*
 * Prefill partition (Algorithm 1 steps 5-9): split the L prompt rows X [L][d] (x_dtype) of one
 * side.
 *   protected_pos [n_protected]  int32, strictly ascending, inside [0, L): P_X (for keys the
 *                                selection's P_K, for values its P_V).
 *   init_window                  0 for keys, min(W, L) for values; 0 <= init_window <= t->window.
 * Writes the protected rows, then the unprotected rows among the last init_window positions, into
 * the exact-row table (converted to t->dtype), and every other row, in ascending position, into
 * comp_rows [L][d] (x_dtype) with comp_pos [L]: the rows the prompt's truncated SVD compresses
 * (Algorithm 1 step 7; iskv_compress_prompt() folds them into the side's history). Sets the host
 * mirror
 * (n_prot = n_protected, n_live, live_host, last = L - 1, fold_rows = 0, hist_rows = *n_comp,
 * refit_done = (refit_rows == 0)) and *n_comp (host). The caller then puts the compressed rows'
 * factors in the side's history, with their positions comp_pos in its position table.
 * SYNCHRONOUS: waits for the stream, because the mirror needs the live positions. Errors:
 * ISKV_ERR_ARG for null / misaligned pointers, bad dtypes, init_window out of range, or
 * protected_pos not strictly ascending inside [0, L) (found on the device, reported after the
 * wait; the table is then undefined); ISKV_ERR_CAPACITY when n_protected + init_window > cap_e;
 * ISKV_ERR_NONFINITE when a finite row value overflows an fp16 table.
 */
size_t iskv_cache_prefill_workspace_size(int32_t init_window);
iskv_status iskv_cache_prefill(iskv_exact_table *t, const void *X, int32_t x_dtype, int64_t L,
                               const int32_t *protected_pos, int64_t n_protected,
                               int32_t init_window, void *comp_rows, int32_t *comp_pos,
                               int64_t *n_comp, void *ws, size_t ws_bytes, void *stream);

/*
 * One decode step for `count` tables (Algorithm 3 steps 1-6): tables[i] (host pointer to a
 * host struct, updated in place) with its history hists[i] (host pointer) stores new_rows[i] (device
 * [count][d], row_dtype, converted to the table dtype) at position tables[i]->last + 1; when that
 * makes `block` rows pending, the oldest `block` of them are folded into hists[i]
 * (iskv_fold_block_batched over every table that folds, with tau_rel), their positions join the
 * history's position table and their exact copies leave the table; when a table's folded rows
 * reach reorth_rows, its history is re-orthogonalised (iskv_reorth) in the same step and the count
 * restarts. A table whose first refit is still to come waits for refit_rows pending rows instead,
 * then factors the history's rows followed by those rows at rank r_max (Section 3.2, Algorithm 3
 * step 3): as one fold of all of them when the fold takes such a block; for an empty history with
 * refit_rows <= r_max, as untruncated block folds; otherwise as block folds into a wide history of
 * rank r_max + refit_rows - block (rounded up to a multiple of 16, at most 512 and d) held in the
 * workspace, none of which truncates before the last, whose top r_max components come back -- in
 * every case the rank-r_max truncated SVD of those rows (Eckart-Young). All tables share
 * d, window, block and dtype; the histories share d, r_max, storage and n_cap, as the batched fold
 * and re-orthogonalisation require. folded / reorthed (host [count], may be NULL) receive 1 where a
 * table folded a block (2 where it ran its first refit) / re-orthogonalised. Stream-ordered; the
 * host mirror is updated at once. The workspace query takes the largest refit_rows of the tables
 * (0 when none refits). Errors (nothing launched, no table changed): ISKV_ERR_ARG,
 * ISKV_ERR_SHAPE (mixed table shapes, a history whose d differs, a block the fold does not take, a
 * refit that can be run none of these ways), ISKV_ERR_CAPACITY (a table without room for the new row, or
 * a history without room for the block or the refit: hist_rows + rows > n_cap),
 * ISKV_ERR_WORKSPACE; ISKV_ERR_CUDA when a launch fails.
 */
/*
 * Compression of the prompt rows on the device (Algorithm 1 step 7): for each history hs[i], the
 * n_rows[i] rows rows[i] ([n_rows[i]][d] dtype, device, ascending positions pos[i] [n_rows[i]]
 * int32 device -- the comp_rows / comp_pos of iskv_cache_prefill) are folded (Algorithm 2) in
 * blocks of `block` rows; a last block of t < block rows is folded as ceil(t / 8) * 8 rows, the
 * real ones followed by zero rows, whose coordinate rows (zero) are then dropped again, so the
 * history ends with exactly n_rows[i] more rows. Reading of the pages' "truncated SVD of the
 * compressed prompt rows": the block fold reaches that SVD exactly when no fold truncates before
 * the last, i.e. when the history's rank plus n_rows[i] - (last block) stays within r_max; a longer
 * prompt is compressed incrementally, as the long-prompt workload compresses its prompt (rank 512
 * by folds of 128 rows). Histories usually start empty; the batched fold's rules apply (shared d,
 * r_max, storage; 8 <= block <= 128, a multiple of 8). Stream-ordered, no host synchronisation.
 * ws: iskv_compress_prompt_workspace_size(count, d, r_max, block) bytes, 256-byte aligned.
 * Errors: as iskv_fold_block_batched (ISKV_ERR_CAPACITY in a status word when a history has no
 * room for its rows).
 */
size_t iskv_compress_prompt_workspace_size(int32_t count, int32_t d, int32_t r_max, int32_t block);
iskv_status iskv_compress_prompt(const iskv_lowrank *hs, int32_t count, const void *const *rows,
                                 const int32_t *const *pos, const int64_t *n_rows, int32_t dtype,
                                 int32_t block, float tau_rel, void *ws, size_t ws_bytes,
                                 void *stream);

size_t iskv_cache_step_workspace_size(int32_t count, int32_t d, int32_t r_max, int32_t block,
                                      int64_t n_cap, int32_t refit_rows);
iskv_status iskv_cache_step(iskv_exact_table *const *tables, const iskv_lowrank *const *hists,
                            int32_t count, const void *new_rows, int32_t row_dtype, float tau_rel,
                            int32_t *folded, int32_t *reorthed, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * Host-only dry run of iskv_cache_step()'s schedule (touches no device memory and launches
 * nothing): folded[i] / reorthed[i] (host [count], may be NULL) receive what the next
 * iskv_cache_step() would do to tables[i] -- 0, 1 (a block fold) or 2 (the first refit), and
 * whether a re-orthogonalisation follows -- for histories of the given r_max and n_cap. With
 * advance != 0 the host mirrors are then advanced exactly as that step would advance them. Lets a
 * caller see which tables fold before a step (to plan workspaces or overlap other work). Errors as
 * iskv_cache_step()'s host-side ones (ISKV_ERR_ARG, ISKV_ERR_SHAPE, ISKV_ERR_CAPACITY); on an error
 * no mirror is changed.
 */
iskv_status iskv_cache_plan(iskv_exact_table *const *tables, int32_t count, int32_t r_max,
                            int64_t n_cap, int32_t advance, int32_t *folded, int32_t *reorthed);

/* Empty a history: zero its meta word, sigma, U and B (stream-ordered). */
iskv_status iskv_reset(const iskv_lowrank *h, void *stream);

/*
 * Synchronously read a history's meta word (waits for all work on the device to finish).
 * Any output pointer may be NULL (host pointers).
 */
iskv_status iskv_get_status(const iskv_lowrank *h, int64_t *k, int64_t *n, int64_t *folds,
                            int64_t *status_bits);

/*
 * Instrumentation (no counterpart on the pages; measurement support). When stage timing is on,
 * every entry point records CUDA events on its own stream around each internal stage (fold:
 * projection, residual QR + SVD, core SVD, basis rotation, coordinate rotation, write-back;
 * reorth; reconstruction; selection; decode attention; cache step: append and eviction).
 * iskv_stage_read() waits for those events and returns the
 * accumulated milliseconds and call counts per stage (arrays of iskv_stage_count() entries, host
 * memory). iskv_stage_timing() returns the previous setting. iskv_launch_count() is the number of
 * kernels the library has launched in this process (always counted).
 */
int32_t iskv_stage_timing(int32_t enable);
int32_t iskv_stage_count(void);
const char *iskv_stage_name(int32_t i);
iskv_status iskv_stage_read(double *ms, int64_t *calls);
void iskv_stage_reset(void);
int64_t iskv_launch_count(void);

/*
 * Work counters of the one-sided Jacobi core SVD (no counterpart on the pages; measurement
 * support for the fold's Algorithm 2 step 6 and the Section 4.4 re-orthogonalisation), always
 * counted on the device and accumulated over every call since the last reset. out: host int64[12],
 * six values for the fold's cores, then six for the re-orthogonalisation's: {cores solved, sweeps
 * summed over cores, largest sweep count of one core, column-pair inner products, rotations
 * applied, float32 flops}. Flops charge 2 m per inner product over the m rows of a column and
 * 8 (m + v) per rotation of two columns holding m rows of A and v explicit rows of V (per-round
 * column norms are not counted). Synchronous: waits for the device. reset != 0 zeroes the
 * counters after reading them.
 */
iskv_status iskv_core_stats(int64_t *out, int32_t reset);

/*
 * Failure-path self-test (no counterpart on the pages; it lets failure detection be tested without
 * faulting a GPU). Launches one CTA that waits on a shared-memory barrier nothing ever arrives at,
 * through the same bounded wait the tensor-core kernels use, with a limit of `limit_ns`
 * nanoseconds (clamped to [1e5, 2e9]). When the wait gives up, the kernel records
 * ISKV_ERR_TIMEOUT in meta[3] (bit 1 << ISKV_ERR_TIMEOUT) as those kernels do, and returns; the
 * context stays usable. meta: device int64[4], 8-byte aligned. Stream-ordered.
 */
iskv_status iskv_selftest_wait_timeout(int64_t *meta, int64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ISKV_H */
