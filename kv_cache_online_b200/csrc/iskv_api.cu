// C ABI of libiskv: argument validation on the host, workspace carving and the launch sequence of
// each entry point. Every numerical step runs in the kernels of the other translation units.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "iskv.h"
#include "kernels.h"
#include "policy.h"
#include "profiling.h"
#include "recon.h"
#include "reorth.h"
#include "select.h"
#include "tc.h"
#include "api_error.h"

using namespace iskv;

namespace iskv {

thread_local std::string g_last_error;

void clear_last_error() { g_last_error.clear(); }

iskv_status fail(iskv_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

iskv_status cuda_fail(cudaError_t e, const char *where) {
  return fail(ISKV_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

}  // namespace iskv

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_dtype(int32_t t) { return t == ISKV_F32 || t == ISKV_BF16 || t == ISKV_F16; }

iskv_status check_handle(const iskv_lowrank *h, const char *who) {
  if (!h) return fail(ISKV_ERR_ARG, "%s: null history handle", who);
  if (!h->U || !h->sigma || !h->B || !h->pos || !h->meta)
    return fail(ISKV_ERR_ARG, "%s: null pointer in history handle", who);
  if (!aligned(h->U, 16) || !aligned(h->sigma, 16) || !aligned(h->B, 16) || !aligned(h->pos, 16) ||
      !aligned(h->meta, 16))
    return fail(ISKV_ERR_ARG, "%s: history pointers must be 16-byte aligned", who);
  if (!valid_dtype(h->storage)) return fail(ISKV_ERR_ARG, "%s: bad storage dtype", who);
  if (h->d <= 0 || h->d % 16 || h->r_max < 16 || h->r_max % 16 || h->r_max > 512 ||
      h->r_max > h->d)
    return fail(ISKV_ERR_SHAPE, "%s: need d %% 16 == 0, r_max %% 16 == 0, 16 <= r_max <= "
                "min(d, 512) (got d=%d r_max=%d)", who, h->d, h->r_max);
  if (h->n_cap < 0 || h->n_cap >= (int64_t)1 << 31)
    return fail(ISKV_ERR_SHAPE, "%s: n_cap out of range", who);
  return ISKV_OK;
}

iskv_status check_ws(const void *ws, size_t have, size_t need, const char *who) {
  if (need == 0) return ISKV_OK;
  if (!ws) return fail(ISKV_ERR_WORKSPACE, "%s: null workspace", who);
  if (!aligned(ws, 256)) return fail(ISKV_ERR_WORKSPACE, "%s: workspace must be 256-byte aligned", who);
  if (have < need)
    return fail(ISKV_ERR_WORKSPACE, "%s: workspace too small (%zu < %zu bytes)", who, have, need);
  return ISKV_OK;
}

size_t jobs_bytes(int32_t count, size_t each) { return align_up((size_t)count * each, 256); }

}  // namespace

namespace {

struct AttnWsLayout {
  size_t tc, tcpv, recon, slices, bsig, S, stats, wpart, mpart, P, opart, omass, per_job, total;
  int nchunk, nblk;
};

AttnWsLayout attn_ws_layout(int32_t count, int32_t d, int32_t r, int64_t n_cap, int64_t n_total_max,
                            int32_t n_q) {
  AttnWsLayout L;
  L.nchunk = (int)((n_cap + ATTN_CHUNK - 1) / ATTN_CHUNK);
  if (L.nchunk < 1) L.nchunk = 1;
  L.nblk = (int)((n_cap + 256 * ATTN_PROB_ROWS - 1) / (256 * ATTN_PROB_ROWS));
  if (L.nblk < 1) L.nblk = 1;
  L.tc = jobs_bytes(count, sizeof(AttnJob));
  L.tcpv = L.tc + tc_table_bytes(count);
  L.recon = L.tcpv + tc_table_bytes(count);
  L.slices = L.recon + jobs_bytes(count, sizeof(ReconJob));
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  L.bsig = take((size_t)d * r * 2);
  L.S = take((size_t)n_q * (size_t)n_total_max * 4);
  L.stats = take((size_t)n_q * 2 * 4);
  // Value-mixing partials and probabilities: the CUDA-core layouts ([chunk][n_q][r] and
  // [n_q][n_cap] float32) or the tensor-core ones ([chunk][r][64] float32, [n_cap][64] bf16).
  L.wpart = take((size_t)L.nchunk * r * (n_q > 64 ? n_q : 64) * 4);
  L.mpart = take((size_t)L.nblk * n_q * 4);
  L.P = take((size_t)n_cap * (4 * n_q > 128 ? 4 * n_q : 128));
  L.opart = take((size_t)AO_SPLIT * n_q * d * 4);  // head_dim <= d
  L.omass = take((size_t)AO_SPLIT * n_q * 4);
  L.per_job = o;
  L.total = L.slices + (size_t)count * L.per_job;
  return L;
}

}  // namespace

namespace {

size_t elem_size(int32_t dtype) { return dtype == ISKV_F32 ? 4 : 2; }

iskv_status check_table(const iskv_exact_table *t, const char *who) {
  if (!t) return fail(ISKV_ERR_ARG, "%s: null table", who);
  if (!t->rows || !t->pos || !t->live_host)
    return fail(ISKV_ERR_ARG, "%s: null pointer in exact-row table", who);
  if (!valid_dtype(t->dtype)) return fail(ISKV_ERR_ARG, "%s: bad table dtype", who);
  if (!aligned(t->rows, 16) || !aligned(t->pos, 4))
    return fail(ISKV_ERR_ARG, "%s: table rows must be 16-byte aligned", who);
  if (t->d <= 0 || ((size_t)t->d * elem_size(t->dtype)) % 16)
    return fail(ISKV_ERR_SHAPE, "%s: d * element size must be a multiple of 16 bytes", who);
  if (t->window < 0 || t->block < 1 || t->reorth_rows < 0 || t->refit_rows < 0)
    return fail(ISKV_ERR_SHAPE, "%s: need window >= 0, block >= 1, reorth_rows >= 0, "
                "refit_rows >= 0", who);
  if (t->refit_rows % t->block)
    return fail(ISKV_ERR_SHAPE, "%s: refit_rows must be a multiple of block", who);
  if (t->cap_e < 0 || t->cap_e >= (int64_t)1 << 31)
    return fail(ISKV_ERR_SHAPE, "%s: cap_e out of range", who);
  const int64_t fifo = t->block > t->refit_rows ? t->block : t->refit_rows;
  if (t->live_cap < (int64_t)t->window + fifo)
    return fail(ISKV_ERR_SHAPE, "%s: live_cap must be >= window + max(block, refit_rows)", who);
  return ISKV_OK;
}

// Rows of the FIFO once position t is stored: live rows at or before t - window (the live rows are
// ascending, so they are a prefix), counting t itself when the window is empty.
int64_t pending_after(const iskv_exact_table *t, int64_t pos) {
  const int64_t edge = pos - t->window;
  int64_t lo = 0, hi = t->n_live;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (t->live_host[mid] <= edge) lo = mid + 1;
    else hi = mid;
  }
  return lo + (pos <= edge ? 1 : 0);
}

static_assert(sizeof(AppendJob) <= 64 && sizeof(EvictJob) <= 64, "policy job sizes");

// A refit of `rows` rows can be one fold with a block of that many rows (any history: Algorithm 2
// on the history's rows followed by the block, truncated to r_max) when the fold takes the block.
bool refit_in_one_fold(int d, int r, int rows) {
  JacobiCfg jc;
  return rows >= 8 && rows % 8 == 0 && rows <= 128 && rows <= d &&
         fold_residual_smem(d, rows) <= 200 * 1024 && core_cfg(r, rows, false, jc);
}

// Rank budget of the wide history through which a refit of `rows` rows (b-row blocks) reaches an
// exact truncated SVD: r + rows - b (rounded up to a multiple of 16) holds every direction of the
// first rows / b - 1 folds, so only the last fold truncates, and its top r are the rank-r SVD of
// the history's rows followed by the refit rows (Eckart-Young). 0 when no such fold fits.
int32_t wide_refit_rank(int d, int r, int b, int rows) {
  int32_t rw = (r + rows - b + 15) / 16 * 16;
  if (rw < r) rw = r;
  JacobiCfg jc;
  if (rw > 512 || rw > d || !core_cfg(rw, b, false, jc) || fold_residual_smem(d, b) > 200 * 1024)
    return 0;
  return rw;
}

// Workspace of a wide refit: the fold workspace of the wide history, then its U, B, sigma,
// positions and meta word (U and B sized for float32 elements, the widest storage).
struct WideWs {
  size_t fold, U, B, sig, pos, meta, total;
};

WideWs wide_ws(int d, int rw, int b, int64_t n_cap) {
  WideWs w;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  w.fold = take(iskv_fold_workspace_size(1, d, rw, b));
  w.U = take(sizeof(float) * (size_t)(n_cap > 0 ? n_cap : 1) * rw);
  w.B = take(sizeof(float) * (size_t)d * rw);
  w.sig = take(sizeof(float) * (size_t)rw);
  w.pos = take(sizeof(int32_t) * (size_t)(n_cap > 0 ? n_cap : 1));
  w.meta = take(4 * sizeof(int64_t));
  w.total = o;
  return w;
}

// What the next decode step does to one table, decided from its host mirror alone: the rows it
// folds (0: none; `block`, or refit_rows for the first refit), the block size of those folds,
// whether they run through a wide history (rank rw), and whether a re-orthogonalisation follows.
struct TablePlan {
  int32_t rows = 0, blk = 0, rw = 0;
  bool refit = false, reorth = false;
};

iskv_status plan_table(const iskv_exact_table *T, int d, int r, int64_t ncap, int i,
                       const char *who, TablePlan &p) {
  p = TablePlan{};
  const int b = T->block;
  const bool refit = !T->refit_done && T->refit_rows > 0;  // a 0-row refit counts as done
  const int32_t rows = refit ? T->refit_rows : b;
  if (pending_after(T, T->last + 1) < rows) return ISKV_OK;
  if (T->hist_rows + rows > ncap)
    return fail(ISKV_ERR_CAPACITY, "%s: table %d: history has no room for a block (%lld + %d > "
                "%lld)", who, i, (long long)T->hist_rows, rows, (long long)ncap);
  // A refit is one fold of all its rows when the fold takes such a block; otherwise, for an empty
  // history and refit_rows <= r_max, consecutive b-row folds that never truncate; otherwise
  // b-row folds into a wide history of rank r + refit_rows - b, of which the top r are kept.
  int32_t blk = b, rw = 0;
  if (refit) {
    if (refit_in_one_fold(d, r, rows)) blk = rows;
    else if (T->hist_rows != 0 || rows > r) {
      rw = wide_refit_rank(d, r, b, rows);
      if (rw == 0)
        return fail(ISKV_ERR_SHAPE, "%s: table %d: a first refit of %d rows is carried out as one "
                    "fold (refit_rows <= 128 with r_max + refit_rows inside the core SVD cluster), "
                    "for an empty history as untruncated block folds (refit_rows <= r_max), or "
                    "through a wide history of rank r_max + refit_rows - block (at most 512 and "
                    "d); history rows %lld", who, i, rows, (long long)T->hist_rows);
    }
  }
  p.rows = rows;
  p.blk = blk;
  p.rw = rw;
  p.refit = refit;
  p.reorth = !refit && T->reorth_rows > 0 && T->fold_rows + b >= T->reorth_rows;
  return ISKV_OK;
}

// The host mirror after the step `p` describes: the new position is stored, the folded rows leave
// the live rows and join the history, and the counters move (the refit is outside reorth_rows).
void advance_table(iskv_exact_table *T, const TablePlan &p) {
  T->last += 1;
  T->live_host[T->n_live++] = (int32_t)T->last;
  if (p.rows > 0) {
    std::memmove(T->live_host, T->live_host + p.rows,
                 sizeof(int32_t) * (size_t)(T->n_live - p.rows));
    T->n_live -= p.rows;
    T->hist_rows += p.rows;
    if (p.refit) T->refit_done = 1;
    else T->fold_rows += p.rows;
    if (T->refit_rows == 0) T->refit_done = 1;
  }
  if (p.reorth) T->fold_rows = 0;
}

// Mirror checks shared by the step and its dry run: the table has room for the new row.
iskv_status check_room(const iskv_exact_table *T, int i, const char *who) {
  if (T->n_prot < 0 || T->n_live < 0 || T->hist_rows < 0 || T->last + 1 >= (int64_t)1 << 31)
    return fail(ISKV_ERR_SHAPE, "%s: table %d: inconsistent host mirror", who, i);
  if (T->n_prot + T->n_live + 1 > T->cap_e || T->n_live + 1 > T->live_cap)
    return fail(ISKV_ERR_CAPACITY, "%s: table %d has no room for the new row", who, i);
  return ISKV_OK;
}

}  // namespace

extern "C" {

int32_t iskv_abi_version(void) { return ISKV_ABI_VERSION; }

const char *iskv_status_string(int32_t st) {
  switch (st) {
    case ISKV_OK: return "ok";
    case ISKV_ERR_ARG: return "invalid argument";
    case ISKV_ERR_SHAPE: return "unsupported or inconsistent shape";
    case ISKV_ERR_CUDA: return "CUDA error";
    case ISKV_ERR_CAPACITY: return "history capacity exceeded";
    case ISKV_ERR_NONFINITE: return "non-finite singular value";
    case ISKV_ERR_NOT_CONVERGED: return "iteration did not converge";
    case ISKV_ERR_TIMEOUT: return "bounded wait timed out";
    case ISKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown status";
  }
}

const char *iskv_last_error(void) { return g_last_error.c_str(); }

iskv_status iskv_core_stats(int64_t *out, int32_t reset) {
  g_last_error.clear();
  if (!out) return fail(ISKV_ERR_ARG, "iskv_core_stats: null output");
  long long v[2 * CORE_STATS];
  cudaError_t e = core_stats(v, reset != 0);
  if (e != cudaSuccess) return cuda_fail(e, "iskv_core_stats");
  for (int i = 0; i < 2 * CORE_STATS; ++i) out[i] = v[i];
  return ISKV_OK;
}

// ------------------------------------------------------------------------------------------------
// Fold
size_t iskv_fold_workspace_size(int32_t count, int32_t d, int32_t r_max, int32_t b) {
  if (count < 1 || d < 1 || r_max < 1 || b < 1) return 0;
  const FoldWsLayout L = fold_ws_layout(d, r_max, b);
  return jobs_bytes(count, sizeof(FoldJob)) + 3 * tc_table_bytes(count) + (size_t)count * L.total;
}

static iskv_status fold_batched(const iskv_lowrank *hs, int32_t count, const void *const *F,
                                int32_t f_dtype, int32_t b, const int32_t *const *f_pos,
                                float tau_rel, void *ws, size_t ws_bytes, void *stream,
                                void *factors_ready) {
  const char *who = "iskv_fold_block";
  g_last_error.clear();
  if (!hs || !F || !f_pos) return fail(ISKV_ERR_ARG, "%s: null host array", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  if (!valid_dtype(f_dtype)) return fail(ISKV_ERR_ARG, "%s: bad F dtype", who);
  if (!(tau_rel >= 0.f)) return fail(ISKV_ERR_ARG, "%s: tau_rel must be >= 0", who);
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_handle(&hs[i], who);
    if (st != ISKV_OK) return st;
    if (hs[i].d != hs[0].d || hs[i].r_max != hs[0].r_max || hs[i].storage != hs[0].storage)
      return fail(ISKV_ERR_SHAPE, "%s: batched histories must share d, r_max, storage", who);
    if (!F[i] || !f_pos[i]) return fail(ISKV_ERR_ARG, "%s: null F or f_pos", who);
    if (!aligned(F[i], 16) || !aligned(f_pos[i], 4))
      return fail(ISKV_ERR_ARG, "%s: F must be 16-byte aligned", who);
  }
  const int d = hs[0].d, r = hs[0].r_max;
  if (b < 8 || b % 8 || b > 128 || b > d)
    return fail(ISKV_ERR_SHAPE, "%s: need 8 <= b <= min(d, 128), b %% 8 == 0 (got %d)", who, b);
  if (fold_residual_smem(d, b) > 200 * 1024)
    return fail(ISKV_ERR_SHAPE, "%s: d = %d with b = %d exceeds the residual QR cluster", who, d, b);
  {
    JacobiCfg jc;
    if (!core_cfg(r, b, false, jc))
      return fail(ISKV_ERR_SHAPE, "%s: r_max + b too large for the core SVD cluster", who);
  }
  const size_t need = iskv_fold_workspace_size(count, d, r, b);
  iskv_status st = check_ws(ws, ws_bytes, need, who);
  if (st != ISKV_OK) return st;

  FoldParams p;
  p.d = d;
  p.r = r;
  p.b = b;
  p.f_dtype = f_dtype;
  p.storage = hs[0].storage;
  p.count = count;
  p.tau_rel = tau_rel;
  p.ws = fold_ws_layout(d, r, b);
  p.tc_basis = tc_basis_supported(r, p.ws.bpad, p.storage) ? 1 : 0;
  char *base = static_cast<char *>(ws);
  TcJob *tc_dev = reinterpret_cast<TcJob *>(base + jobs_bytes(count, sizeof(FoldJob)));
  TcJob *basis_dev = reinterpret_cast<TcJob *>(base + jobs_bytes(count, sizeof(FoldJob)) +
                                               tc_table_bytes(count));
  ProjJob *proj_dev = reinterpret_cast<ProjJob *>(base + jobs_bytes(count, sizeof(FoldJob)) +
                                                  2 * tc_table_bytes(count));
  const size_t jb = jobs_bytes(count, sizeof(FoldJob)) + 3 * tc_table_bytes(count);
  std::vector<FoldJob> jobs(count);
  int64_t ncap_max = 0;
  for (int32_t i = 0; i < count; ++i) {
    FoldJob &j = jobs[i];
    j.h.U = hs[i].U;
    j.h.sigma = hs[i].sigma;
    j.h.B = hs[i].B;
    j.h.pos = hs[i].pos;
    j.h.meta = hs[i].meta;
    j.h.ws = base + jb + (size_t)i * p.ws.total;
    j.F = F[i];
    j.f_pos = f_pos[i];
    j.n_cap = hs[i].n_cap;
    j.pad_ = 0;
    if (hs[i].n_cap > ncap_max) ncap_max = hs[i].n_cap;
  }
  const bool tc_rot = tc_rotation_supported(r, p.storage);
  std::vector<TcJob> tj;
  if (tc_rot) {
    tj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_rotation_job(tj[i], hs[i].U, hs[i].n_cap, r, jobs[i].h.ws + p.ws.Gtb,
                               reinterpret_cast<const int32_t *>(jobs[i].h.ws + p.ws.scal),
                               hs[i].meta))
        return fail(ISKV_ERR_CUDA, "fold: tensor map encoding failed");
  }
  const bool tc_proj = tc_project_supported(d, r, b, p.storage, f_dtype);
  std::vector<ProjJob> pj;
  if (tc_proj) {
    pj.resize(count);
    for (int32_t i = 0; i < count; ++i) {
      char *w = jobs[i].h.ws;
      if (!encode_project_job(pj[i], hs[i].B, d, r, F[i], b, reinterpret_cast<float *>(w + p.ws.C),
                              reinterpret_cast<float *>(w + p.ws.E), w + p.ws.E1,
                              reinterpret_cast<const int32_t *>(w + p.ws.scal), hs[i].meta))
        return fail(ISKV_ERR_CUDA, "fold: tensor map encoding failed");
    }
  }
  std::vector<TcJob> bj;
  if (p.tc_basis) {
    bj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_basis_job(bj[i], hs[i].B, d, r, jobs[i].h.ws + p.ws.Pb, p.ws.bpad,
                            jobs[i].h.ws + p.ws.Htb,
                            reinterpret_cast<const int32_t *>(jobs[i].h.ws + p.ws.scal),
                            hs[i].meta))
        return fail(ISKV_ERR_CUDA, "fold: tensor map encoding failed");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FoldJob *djobs = reinterpret_cast<FoldJob *>(base);
  stage_begin(s);
  cudaError_t e = upload_jobs(djobs, jobs.data(), sizeof(FoldJob) * count, s);
  if (e == cudaSuccess && tc_rot) e = upload_jobs(tc_dev, tj.data(), sizeof(TcJob) * count, s);
  if (e == cudaSuccess && p.tc_basis)
    e = upload_jobs(basis_dev, bj.data(), sizeof(TcJob) * count, s);
  if (e == cudaSuccess && tc_proj) e = upload_jobs(proj_dev, pj.data(), sizeof(ProjJob) * count, s);
  if (e != cudaSuccess) return cuda_fail(e, "fold: upload");
  if ((e = launch_fold_prepare(djobs, p, s)) != cudaSuccess) return cuda_fail(e, "fold: prepare");
  stage_mark(s, ST_UPLOAD);
  e = tc_proj ? launch_tc_project(proj_dev, count, d, r, s) : launch_fold_project(djobs, p, s);
  if (e != cudaSuccess) return cuda_fail(e, "fold: project");
  stage_mark(s, ST_FOLD_PROJECT);
  if ((e = launch_fold_residual(djobs, p, s)) != cudaSuccess) return cuda_fail(e, "fold: residual");
  stage_mark(s, ST_FOLD_RESIDUAL);
  const char *cj = reinterpret_cast<const char *>(djobs);
  if ((e = launch_core(cj, fold_core_params(p), s)) != cudaSuccess)
    return cuda_fail(e, "fold: core svd");
  stage_mark(s, ST_FOLD_CORE);
  // The stages above only read the histories' factors; the rotations and the write-back below
  // change them, after the caller's readers of the current factors are done.
  if (factors_ready &&
      (e = cudaStreamWaitEvent(s, static_cast<cudaEvent_t>(factors_ready), 0)) != cudaSuccess)
    return cuda_fail(e, "fold: wait for factors_ready");
  const RotParams rp = fold_rot_params(p);
  if (p.tc_basis) {
    e = launch_basis_prep(djobs, p, s);
    if (e == cudaSuccess) e = launch_tc_basis(basis_dev, count, d, r, p.ws.kpad, s);
  } else {
    e = launch_rotate_basis(cj, rp, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "fold: basis rotation");
  stage_mark(s, ST_FOLD_BASIS);
  if (tc_rot) {
    e = launch_tc_rotation(tc_dev, count, r, ncap_max, s);
  } else {
    e = launch_rotate_coords_ffma(cj, rp, ncap_max, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "fold: coordinate rotation");
  stage_mark(s, ST_FOLD_COORDS);
  if ((e = launch_fold_finalize(djobs, p, s)) != cudaSuccess) return cuda_fail(e, "fold: finalize");
  stage_mark(s, ST_FOLD_FINALIZE);
  return ISKV_OK;
}

iskv_status iskv_fold_block_batched(const iskv_lowrank *hs, int32_t count, const void *const *F,
                                    int32_t f_dtype, int32_t b, const int32_t *const *f_pos,
                                    float tau_rel, void *ws, size_t ws_bytes, void *stream) {
  return fold_batched(hs, count, F, f_dtype, b, f_pos, tau_rel, ws, ws_bytes, stream, nullptr);
}

iskv_status iskv_fold_block_batched_after(const iskv_lowrank *hs, int32_t count,
                                          const void *const *F, int32_t f_dtype, int32_t b,
                                          const int32_t *const *f_pos, float tau_rel, void *ws,
                                          size_t ws_bytes, void *stream, void *factors_ready) {
  return fold_batched(hs, count, F, f_dtype, b, f_pos, tau_rel, ws, ws_bytes, stream,
                      factors_ready);
}

iskv_status iskv_fold_block(const iskv_lowrank *h, const void *F, int32_t f_dtype, int32_t b,
                            const int32_t *f_pos, float tau_rel, void *ws, size_t ws_bytes,
                            void *stream) {
  const void *Fs[1] = {F};
  const int32_t *ps[1] = {f_pos};
  if (!h) return fail(ISKV_ERR_ARG, "iskv_fold_block: null history handle");
  return iskv_fold_block_batched(h, 1, Fs, f_dtype, b, ps, tau_rel, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------------------------------------
// Re-orthogonalisation
size_t iskv_reorth_workspace_size(int32_t count, int32_t d, int32_t r_max, int64_t n_cap) {
  if (count < 1 || d < 1 || r_max < 1 || n_cap < 0) return 0;
  const ReorthWsLayout L = reorth_ws_layout(d, r_max, n_cap);
  return jobs_bytes(count, sizeof(ReorthJob)) + 3 * tc_table_bytes(count) + (size_t)count * L.total;
}

iskv_status iskv_reorth(const iskv_lowrank *hs, int32_t count, void *ws, size_t ws_bytes,
                        void *stream) {
  const char *who = "iskv_reorth";
  g_last_error.clear();
  if (!hs) return fail(ISKV_ERR_ARG, "%s: null host array", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_handle(&hs[i], who);
    if (st != ISKV_OK) return st;
    if (hs[i].d != hs[0].d || hs[i].r_max != hs[0].r_max || hs[i].storage != hs[0].storage ||
        hs[i].n_cap != hs[0].n_cap)
      return fail(ISKV_ERR_SHAPE, "%s: batched histories must share d, r_max, storage, n_cap", who);
  }
  const int d = hs[0].d, r = hs[0].r_max;
  const int64_t ncap = hs[0].n_cap;
  {
    JacobiCfg jc;
    if (!core_cfg(r, 0, true, jc))
      return fail(ISKV_ERR_SHAPE, "%s: r_max = %d too large for the dense core SVD",
                  who, r);
  }
  const size_t need = iskv_reorth_workspace_size(count, d, r, ncap);
  iskv_status st = check_ws(ws, ws_bytes, need, who);
  if (st != ISKV_OK) return st;
  ReorthParams p;
  p.d = d;
  p.r = r;
  p.storage = hs[0].storage;
  p.count = count;
  p.n_cap = ncap;
  p.ws = reorth_ws_layout(d, r, ncap);
  char *base = static_cast<char *>(ws);
  TcJob *tc_dev = reinterpret_cast<TcJob *>(base + jobs_bytes(count, sizeof(ReorthJob)));
  TcJob *gram_dev = reinterpret_cast<TcJob *>(base + jobs_bytes(count, sizeof(ReorthJob)) +
                                              tc_table_bytes(count));
  TcJob *basis_dev = reinterpret_cast<TcJob *>(base + jobs_bytes(count, sizeof(ReorthJob)) +
                                               2 * tc_table_bytes(count));
  const size_t jb = jobs_bytes(count, sizeof(ReorthJob)) + 3 * tc_table_bytes(count);
  std::vector<ReorthJob> jobs(count);
  for (int32_t i = 0; i < count; ++i) {
    ReorthJob &j = jobs[i];
    j.h.U = hs[i].U;
    j.h.sigma = hs[i].sigma;
    j.h.B = hs[i].B;
    j.h.pos = hs[i].pos;
    j.h.meta = hs[i].meta;
    j.h.ws = base + jb + (size_t)i * p.ws.total;
    j.n_cap = hs[i].n_cap;
    j.n_exact = 0;
  }
  std::vector<TcJob> tj, gj, bj;
  p.tc_host = nullptr;
  p.tc_dev = tc_dev;
  p.gram_host = nullptr;
  p.gram_nsu = 0;
  p.gram_dev = gram_dev;
  p.tc_basis = tc_basis_supported(r, 0, p.storage) ? 1 : 0;
  p.basis_dev = basis_dev;
  if (p.tc_basis) {
    bj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_basis_job(bj[i], hs[i].B, d, r, nullptr, 0, jobs[i].h.ws + p.ws.TBtb,
                            reinterpret_cast<const int32_t *>(jobs[i].h.ws + p.ws.scal),
                            hs[i].meta))
        return fail(ISKV_ERR_CUDA, "reorth: tensor map encoding failed");
  }
  if (tc_gram_supported(r, p.storage)) {
    gj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_gram_job(gj[i], hs[i].U, hs[i].n_cap, hs[i].B, d, r,
                           reinterpret_cast<const int32_t *>(jobs[i].h.ws + p.ws.scal), hs[i].meta,
                           jobs[i].h.ws))
        return fail(ISKV_ERR_CUDA, "reorth: tensor map encoding failed");
    p.gram_host = gj.data();
    // U chunks per job: about one chunk per SM over all jobs (the B chunks are short).
    int nsu = tc_sm_count() / count;
    p.gram_nsu = nsu < 1 ? 1 : (nsu > p.ws.nsplit_u ? p.ws.nsplit_u : nsu);
  }
  if (tc_rotation_supported(r, p.storage)) {
    tj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_rotation_job(tj[i], hs[i].U, hs[i].n_cap, r, jobs[i].h.ws + p.ws.TUtb,
                               reinterpret_cast<const int32_t *>(jobs[i].h.ws + p.ws.scal),
                               hs[i].meta))
        return fail(ISKV_ERR_CUDA, "reorth: tensor map encoding failed");
    p.tc_host = tj.data();
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ReorthJob *djobs = reinterpret_cast<ReorthJob *>(base);
  stage_begin(s);
  cudaError_t e = upload_jobs(djobs, jobs.data(), sizeof(ReorthJob) * count, s);
  if (e == cudaSuccess && p.gram_host) e = upload_jobs(gram_dev, gj.data(), sizeof(TcJob) * count, s);
  if (e == cudaSuccess && p.tc_host) e = upload_jobs(tc_dev, tj.data(), sizeof(TcJob) * count, s);
  if (e == cudaSuccess && p.tc_basis)
    e = upload_jobs(basis_dev, bj.data(), sizeof(TcJob) * count, s);
  if (e != cudaSuccess) return cuda_fail(e, "reorth: upload");
  stage_mark(s, ST_UPLOAD);
  if ((e = launch_reorth(djobs, p, s)) != cudaSuccess) return cuda_fail(e, "reorth");
  return ISKV_OK;
}

// ------------------------------------------------------------------------------------------------
// Reconstruction
size_t iskv_reconstruct_workspace_size(int32_t count, int32_t d, int32_t r_max) {
  if (count < 1 || d < 1 || r_max < 1) return 0;
  return jobs_bytes(count, sizeof(ReconJob)) + tc_table_bytes(count) +
         (size_t)count * align_up((size_t)d * r_max * 2, 256);
}

iskv_status iskv_reconstruct_batched(const iskv_lowrank *hs, int32_t count,
                                     const void *const *exact_rows, int32_t exact_dtype,
                                     const int32_t *const *exact_pos, const int64_t *n_exact,
                                     const int64_t *n_total, int32_t n_heads, int32_t head_dim,
                                     const int32_t *apply_rope, double rope_theta,
                                     void *const *out, int32_t out_dtype, void *ws,
                                     size_t ws_bytes, void *stream) {
  const char *who = "iskv_reconstruct";
  g_last_error.clear();
  if (!hs || !exact_rows || !exact_pos || !n_exact || !n_total || !apply_rope || !out)
    return fail(ISKV_ERR_ARG, "%s: null host array", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  if (!valid_dtype(exact_dtype) || !valid_dtype(out_dtype))
    return fail(ISKV_ERR_ARG, "%s: bad dtype", who);
  if (n_heads < 1 || head_dim < 2 || head_dim % 2 || head_dim > 256)
    return fail(ISKV_ERR_SHAPE, "%s: need even head_dim <= 256", who);
  if (!(rope_theta > 0.0)) return fail(ISKV_ERR_ARG, "%s: rope_theta must be > 0", who);
  int64_t max_exact = 0, ncap_max = 0;
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_handle(&hs[i], who);
    if (st != ISKV_OK) return st;
    if (hs[i].d != hs[0].d || hs[i].r_max != hs[0].r_max || hs[i].storage != hs[0].storage)
      return fail(ISKV_ERR_SHAPE, "%s: batched histories must share d, r_max, storage", who);
    if (hs[i].d != n_heads * head_dim)
      return fail(ISKV_ERR_SHAPE, "%s: d must equal n_heads * head_dim", who);
    if (!out[i]) return fail(ISKV_ERR_ARG, "%s: null output", who);
    if (n_exact[i] < 0 || n_total[i] < 0) return fail(ISKV_ERR_SHAPE, "%s: negative size", who);
    if (n_exact[i] > 0 && (!exact_rows[i] || !exact_pos[i]))
      return fail(ISKV_ERR_ARG, "%s: null exact rows", who);
    if (n_exact[i] > max_exact) max_exact = n_exact[i];
    if (hs[i].n_cap > ncap_max) ncap_max = hs[i].n_cap;
  }
  const int d = hs[0].d, r = hs[0].r_max;
  const size_t need = iskv_reconstruct_workspace_size(count, d, r);
  iskv_status st = check_ws(ws, ws_bytes, need, who);
  if (st != ISKV_OK) return st;
  ReconParams p;
  p.d = d;
  p.r = r;
  p.storage = hs[0].storage;
  p.exact_dtype = exact_dtype;
  p.out_dtype = out_dtype;
  p.n_heads = n_heads;
  p.head_dim = head_dim;
  p.count = count;
  p.theta = rope_theta;
  p.n_cap_max = ncap_max;
  // Exact rows move as 16-byte vectors when every row starts on a 16-byte boundary.
  p.exact_vec = head_dim % 16 == 0;
  for (int32_t i = 0; i < count; ++i)
    if (n_exact[i] > 0 && (!aligned(exact_rows[i], 16) || !aligned(out[i], 16))) p.exact_vec = 0;
  char *base = static_cast<char *>(ws);
  TcJob *tc_dev = reinterpret_cast<TcJob *>(base + jobs_bytes(count, sizeof(ReconJob)));
  const size_t jb = jobs_bytes(count, sizeof(ReconJob)) + tc_table_bytes(count);
  std::vector<ReconJob> jobs(count);
  for (int32_t i = 0; i < count; ++i) {
    ReconJob &j = jobs[i];
    j.U = hs[i].U;
    j.sigma = hs[i].sigma;
    j.B = hs[i].B;
    j.pos = hs[i].pos;
    j.meta = hs[i].meta;
    j.exact_rows = exact_rows[i];
    j.exact_pos = exact_pos[i];
    j.out = out[i];
    j.bsig = base + jb + (size_t)i * align_up((size_t)d * r * 2, 256);
    j.n_exact = n_exact[i];
    j.n_total = n_total[i];
    j.apply_rope = apply_rope[i];
    j.pad_ = 0;
  }
  // The tensor-core path writes 16-byte vectors and tiles: every output must be 16-byte aligned.
  bool outs_aligned = true;
  for (int32_t i = 0; i < count; ++i) outs_aligned = outs_aligned && aligned(out[i], 16);
  const bool tc = outs_aligned && tc_recon_supported(r, p.storage, out_dtype, head_dim);
  std::vector<TcJob> tj;
  if (tc) {
    tj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_recon_job(tj[i], hs[i].U, hs[i].n_cap, r, jobs[i].bsig, d, out[i], hs[i].pos,
                            hs[i].meta, n_total[i], apply_rope[i]))
        return fail(ISKV_ERR_CUDA, "reconstruct: tensor map encoding failed");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ReconJob *djobs = reinterpret_cast<ReconJob *>(base);
  stage_begin(s);
  cudaError_t e = upload_jobs(djobs, jobs.data(), sizeof(ReconJob) * count, s);
  if (e == cudaSuccess && tc) e = upload_jobs(tc_dev, tj.data(), sizeof(TcJob) * count, s);
  if (e != cudaSuccess) return cuda_fail(e, "reconstruct: upload");
  stage_mark(s, ST_UPLOAD);
  if (tc) {
    if ((e = launch_recon_bsig(djobs, p, s)) != cudaSuccess)
      return cuda_fail(e, "reconstruct: scaled basis");
    stage_mark(s, ST_RECON_PREPARE);
    e = launch_tc_recon(tc_dev, p, s);
  } else {
    stage_mark(s, ST_RECON_PREPARE);
    e = launch_recon_compressed(djobs, p, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "reconstruct: compressed rows");
  stage_mark(s, ST_RECON_COMPRESSED);
  if ((e = launch_recon_exact(djobs, p, max_exact, s)) != cudaSuccess)
    return cuda_fail(e, "reconstruct: exact rows");
  stage_mark(s, ST_RECON_EXACT);
  return ISKV_OK;
}

iskv_status iskv_reconstruct(const iskv_lowrank *h, const void *exact_rows, int32_t exact_dtype,
                             const int32_t *exact_pos, int64_t n_exact, int64_t n_total,
                             int32_t n_heads, int32_t head_dim, int32_t apply_rope,
                             double rope_theta, void *out, int32_t out_dtype, void *ws,
                             size_t ws_bytes, void *stream) {
  if (!h) return fail(ISKV_ERR_ARG, "iskv_reconstruct: null history handle");
  const void *er[1] = {exact_rows};
  const int32_t *ep[1] = {exact_pos};
  const int64_t ne[1] = {n_exact};
  const int64_t nt[1] = {n_total};
  const int32_t ar[1] = {apply_rope};
  void *o[1] = {out};
  return iskv_reconstruct_batched(h, 1, er, exact_dtype, ep, ne, nt, n_heads, head_dim, ar,
                                  rope_theta, o, out_dtype, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------------------------------------
// Diagnostics: orthogonality of the factors and persistent bytes (eq. 12)
size_t iskv_diagnostics_workspace_size(int32_t count, int32_t d, int32_t r_max, int64_t n_cap) {
  return iskv_reorth_workspace_size(count, d, r_max, n_cap);
}

iskv_status iskv_diagnostics(const iskv_lowrank *hs, int32_t count, const int64_t *n_exact,
                             int32_t exact_elem_bytes, double *orth_u, double *orth_b,
                             int64_t *persistent_bytes, void *ws, size_t ws_bytes, void *stream) {
  const char *who = "iskv_diagnostics";
  g_last_error.clear();
  if (!hs || !orth_u || !orth_b || !persistent_bytes)
    return fail(ISKV_ERR_ARG, "%s: null argument", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  if (exact_elem_bytes < 0 || exact_elem_bytes > 8)
    return fail(ISKV_ERR_ARG, "%s: exact_elem_bytes must be in [0, 8]", who);
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_handle(&hs[i], who);
    if (st != ISKV_OK) return st;
    if (hs[i].d != hs[0].d || hs[i].r_max != hs[0].r_max || hs[i].storage != hs[0].storage ||
        hs[i].n_cap != hs[0].n_cap)
      return fail(ISKV_ERR_SHAPE, "%s: batched histories must share d, r_max, storage, n_cap", who);
    if (n_exact && n_exact[i] < 0) return fail(ISKV_ERR_SHAPE, "%s: negative n_exact", who);
  }
  const int d = hs[0].d, r = hs[0].r_max;
  const int64_t ncap = hs[0].n_cap;
  const size_t need = iskv_diagnostics_workspace_size(count, d, r, ncap);
  iskv_status st = check_ws(ws, ws_bytes, need, who);
  if (st != ISKV_OK) return st;
  ReorthParams p;
  p.d = d;
  p.r = r;
  p.storage = hs[0].storage;
  p.count = count;
  p.n_cap = ncap;
  p.ws = reorth_ws_layout(d, r, ncap);
  char *base = static_cast<char *>(ws);
  TcJob *gram_dev = reinterpret_cast<TcJob *>(base + jobs_bytes(count, sizeof(ReorthJob)) +
                                              tc_table_bytes(count));
  const size_t jb = jobs_bytes(count, sizeof(ReorthJob)) + 2 * tc_table_bytes(count);
  std::vector<ReorthJob> jobs(count);
  for (int32_t i = 0; i < count; ++i) {
    ReorthJob &j = jobs[i];
    j.h.U = hs[i].U;
    j.h.sigma = hs[i].sigma;
    j.h.B = hs[i].B;
    j.h.pos = hs[i].pos;
    j.h.meta = hs[i].meta;
    j.h.ws = base + jb + (size_t)i * p.ws.total;
    j.n_cap = hs[i].n_cap;
    j.n_exact = n_exact ? n_exact[i] : 0;
  }
  std::vector<TcJob> gj;
  p.tc_host = nullptr;
  p.tc_dev = nullptr;
  p.gram_host = nullptr;
  p.gram_nsu = 0;
  p.gram_dev = gram_dev;
  p.tc_basis = 0;
  p.basis_dev = nullptr;
  if (tc_gram_supported(r, p.storage)) {
    gj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_gram_job(gj[i], hs[i].U, hs[i].n_cap, hs[i].B, d, r,
                           reinterpret_cast<const int32_t *>(jobs[i].h.ws + p.ws.scal), hs[i].meta,
                           jobs[i].h.ws))
        return fail(ISKV_ERR_CUDA, "%s: tensor map encoding failed", who);
    p.gram_host = gj.data();
    // U chunks per job: about one chunk per SM over all jobs (the B chunks are short).
    int nsu = tc_sm_count() / count;
    p.gram_nsu = nsu < 1 ? 1 : (nsu > p.ws.nsplit_u ? p.ws.nsplit_u : nsu);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ReorthJob *djobs = reinterpret_cast<ReorthJob *>(base);
  cudaError_t e = upload_jobs(djobs, jobs.data(), sizeof(ReorthJob) * count, s);
  if (e == cudaSuccess && p.gram_host) e = upload_jobs(gram_dev, gj.data(), sizeof(TcJob) * count, s);
  if (e != cudaSuccess) return cuda_fail(e, "diagnostics: upload");
  if ((e = launch_diagnostics(djobs, p, exact_elem_bytes, orth_u, orth_b, persistent_bytes, s)) !=
      cudaSuccess)
    return cuda_fail(e, "diagnostics");
  return ISKV_OK;
}

// ------------------------------------------------------------------------------------------------
// Decode attention over the compressed cache
size_t iskv_attention_workspace_size(int32_t count, int32_t d, int32_t r_max, int64_t n_cap,
                                     int64_t n_total_max, int32_t n_q_heads) {
  if (count < 1 || d < 1 || r_max < 1 || n_cap < 0 || n_total_max < 0 || n_q_heads < 1) return 0;
  return attn_ws_layout(count, d, r_max, n_cap, n_total_max, n_q_heads).total;
}

iskv_status iskv_decode_attention_batched(
    const iskv_lowrank *hk, const iskv_lowrank *hv, int32_t count, const void *const *k_exact,
    const int32_t *const *k_exact_pos, const int64_t *n_k_exact, const void *const *v_exact,
    const int32_t *const *v_exact_pos, const int64_t *n_v_exact, int32_t exact_dtype,
    const int64_t *n_total, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
    double rope_theta, float scale, const float *const *q, float *const *out, void *ws,
    size_t ws_bytes, void *stream) {
  const char *who = "iskv_decode_attention";
  g_last_error.clear();
  if (!hk || !hv || !k_exact || !k_exact_pos || !n_k_exact || !v_exact || !v_exact_pos ||
      !n_v_exact || !n_total || !q || !out)
    return fail(ISKV_ERR_ARG, "%s: null host array", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  if (!valid_dtype(exact_dtype)) return fail(ISKV_ERR_ARG, "%s: bad dtype", who);
  if (head_dim < 2 || head_dim % 2 || head_dim > 256)
    return fail(ISKV_ERR_SHAPE, "%s: need even head_dim <= 256", who);
  if (n_kv_heads < 1 || n_q_heads < 1 || n_q_heads > ATTN_MAX_Q || n_q_heads % n_kv_heads ||
      n_q_heads / n_kv_heads > 8)
    return fail(ISKV_ERR_SHAPE,
                "%s: need n_q_heads a multiple of n_kv_heads, <= %d, at most 8 per KV head", who,
                ATTN_MAX_Q);
  if (!(rope_theta > 0.0)) return fail(ISKV_ERR_ARG, "%s: rope_theta must be > 0", who);
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
    return fail(ISKV_ERR_ARG, "%s: scale must be finite", who);
  int64_t max_kex = 0, ntot_max = 0;
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_handle(&hk[i], who);
    if (st == ISKV_OK) st = check_handle(&hv[i], who);
    if (st != ISKV_OK) return st;
    for (const iskv_lowrank *h : {&hk[i], &hv[i]})
      if (h->d != hk[0].d || h->storage != hk[0].storage || h->n_cap != hk[0].n_cap)
        return fail(ISKV_ERR_SHAPE, "%s: K and V histories must share d, storage, n_cap", who);
    if (hk[i].r_max != hk[0].r_max || hv[i].r_max != hv[0].r_max)
      return fail(ISKV_ERR_SHAPE, "%s: batched K histories must share r_max, and so must the V "
                  "histories", who);
    if (hk[i].d != n_kv_heads * head_dim)
      return fail(ISKV_ERR_SHAPE, "%s: d must equal n_kv_heads * head_dim", who);
    if (!q[i] || !out[i]) return fail(ISKV_ERR_ARG, "%s: null query or output", who);
    if (n_k_exact[i] < 0 || n_v_exact[i] < 0 || n_total[i] < 1)
      return fail(ISKV_ERR_SHAPE, "%s: bad sizes", who);
    if ((n_k_exact[i] > 0 && (!k_exact[i] || !k_exact_pos[i])) ||
        (n_v_exact[i] > 0 && (!v_exact[i] || !v_exact_pos[i])))
      return fail(ISKV_ERR_ARG, "%s: null exact rows", who);
    if (n_k_exact[i] > max_kex) max_kex = n_k_exact[i];
    if (n_total[i] > ntot_max) ntot_max = n_total[i];
  }
  const int d = hk[0].d, rk = hk[0].r_max, rv = hv[0].r_max, r = rk > rv ? rk : rv;
  const int64_t ncap = hk[0].n_cap;
  const AttnWsLayout L = attn_ws_layout(count, d, r, ncap, ntot_max, n_q_heads);
  iskv_status st = check_ws(ws, ws_bytes, L.total, who);
  if (st != ISKV_OK) return st;
  AttnParams p;
  p.d = d;
  p.rk = rk;
  p.rv = rv;
  p.storage = hk[0].storage;
  p.exact_dtype = exact_dtype;
  p.n_kv = n_kv_heads;
  p.n_q = n_q_heads;
  p.head_dim = head_dim;
  p.count = count;
  p.nchunk = L.nchunk;
  p.nblk = L.nblk;
  p.tc_values = tc_pv_supported(rv, p.storage, n_q_heads) ? 1 : 0;
  p.theta = rope_theta;
  p.scale = scale;
  p.n_cap_max = ncap;
  p.n_total_max = ntot_max;
  char *base = static_cast<char *>(ws);
  std::vector<AttnJob> jobs(count);
  for (int32_t i = 0; i < count; ++i) {
    AttnJob &j = jobs[i];
    char *slice = base + L.slices + (size_t)i * L.per_job;
    j.Uk = hk[i].U;
    j.sk = hk[i].sigma;
    j.Bk = hk[i].B;
    j.posk = hk[i].pos;
    j.metak = hk[i].meta;
    j.Uv = hv[i].U;
    j.sv = hv[i].sigma;
    j.Bv = hv[i].B;
    j.posv = hv[i].pos;
    j.metav = hv[i].meta;
    j.kex = k_exact[i];
    j.kexpos = k_exact_pos[i];
    j.vex = v_exact[i];
    j.vexpos = v_exact_pos[i];
    j.q = q[i];
    j.out = out[i];
    j.S = reinterpret_cast<float *>(slice + L.S);
    j.stats = reinterpret_cast<float *>(slice + L.stats);
    j.wpart = reinterpret_cast<float *>(slice + L.wpart);
    j.mpart = reinterpret_cast<float *>(slice + L.mpart);
    j.P = reinterpret_cast<float *>(slice + L.P);
    j.Pb = slice + L.P;
    j.opart = reinterpret_cast<float *>(slice + L.opart);
    j.omass = reinterpret_cast<float *>(slice + L.omass);
    j.bsig = slice + L.bsig;
    j.n_kex = n_k_exact[i];
    j.n_vex = n_v_exact[i];
    j.n_total = n_total[i];
  }
  const bool tc = tc_attn_supported(rk, p.storage, head_dim, n_q_heads, n_kv_heads);
  std::vector<TcJob> tj;
  std::vector<ReconJob> rj;
  ReconParams rp;
  if (tc) {
    tj.resize(count);
    rj.resize(count);
    for (int32_t i = 0; i < count; ++i) {
      std::memset(&rj[i], 0, sizeof(ReconJob));
      rj[i].U = hk[i].U;
      rj[i].sigma = hk[i].sigma;
      rj[i].B = hk[i].B;
      rj[i].pos = hk[i].pos;
      rj[i].meta = hk[i].meta;
      rj[i].bsig = jobs[i].bsig;
      if (!encode_attn_job(tj[i], hk[i].U, ncap, rk, jobs[i].bsig, d, jobs[i].S, q[i], hk[i].pos,
                           hk[i].meta, n_total[i], scale))
        return fail(ISKV_ERR_CUDA, "%s: tensor map encoding failed", who);
    }
    rp.d = d;
    rp.r = rk;
    rp.storage = p.storage;
    rp.exact_dtype = exact_dtype;
    rp.out_dtype = ISKV_BF16;
    rp.n_heads = n_kv_heads;
    rp.head_dim = head_dim;
    rp.count = count;
    rp.exact_vec = 0;
    rp.theta = rope_theta;
    rp.n_cap_max = ncap;
  }
  std::vector<TcJob> pj;
  if (p.tc_values) {
    pj.resize(count);
    for (int32_t i = 0; i < count; ++i)
      if (!encode_pv_job(pj[i], hv[i].U, ncap, rv, jobs[i].Pb, jobs[i].wpart, hv[i].meta))
        return fail(ISKV_ERR_CUDA, "%s: tensor map encoding failed", who);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  AttnJob *djobs = reinterpret_cast<AttnJob *>(base);
  TcJob *pv_dev = reinterpret_cast<TcJob *>(base + L.tcpv);
  TcJob *tc_dev = reinterpret_cast<TcJob *>(base + L.tc);
  ReconJob *recon_dev = reinterpret_cast<ReconJob *>(base + L.recon);
  stage_begin(s);
  cudaError_t e = upload_jobs(djobs, jobs.data(), sizeof(AttnJob) * count, s);
  if (e == cudaSuccess && tc) e = upload_jobs(tc_dev, tj.data(), sizeof(TcJob) * count, s);
  if (e == cudaSuccess && tc) e = upload_jobs(recon_dev, rj.data(), sizeof(ReconJob) * count, s);
  if (e == cudaSuccess && p.tc_values) e = upload_jobs(pv_dev, pj.data(), sizeof(TcJob) * count, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention: upload");
  stage_mark(s, ST_UPLOAD);
  if ((e = launch_attn_init(djobs, p, s)) != cudaSuccess) return cuda_fail(e, "attention: init");
  if (tc && (e = launch_recon_bsig(recon_dev, rp, s)) != cudaSuccess)
    return cuda_fail(e, "attention: scaled basis");
  stage_mark(s, ST_ATTN_PREPARE);
  e = tc ? launch_tc_attn_scores(tc_dev, p, s) : launch_attn_scores_ffma(djobs, p, s);
  if (e == cudaSuccess) e = launch_attn_scores_exact(djobs, p, max_kex, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention: scores");
  stage_mark(s, ST_ATTN_SCORES);
  if ((e = launch_attn_stats(djobs, p, s)) != cudaSuccess) return cuda_fail(e, "attention: softmax");
  stage_mark(s, ST_ATTN_SOFTMAX);
  e = launch_attn_probs(djobs, p, s);
  if (e == cudaSuccess) {
    if (p.tc_values) {
      PvParams pv;
      pv.r = rv;
      pv.count = count;
      pv.nsplit = L.nchunk;
      e = launch_tc_pv(pv_dev, pv, s);
    } else {
      e = launch_attn_values(djobs, p, s);
    }
  }
  if (e == cudaSuccess) e = launch_attn_out(djobs, p, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention: values");
  stage_mark(s, ST_ATTN_VALUES);
  return ISKV_OK;
}

iskv_status iskv_decode_attention(const iskv_lowrank *hk, const iskv_lowrank *hv,
                                  const void *k_exact, const int32_t *k_exact_pos,
                                  int64_t n_k_exact, const void *v_exact,
                                  const int32_t *v_exact_pos, int64_t n_v_exact,
                                  int32_t exact_dtype, int64_t n_total, int32_t n_q_heads,
                                  int32_t n_kv_heads, int32_t head_dim, double rope_theta,
                                  float scale, const float *q, float *out, void *ws,
                                  size_t ws_bytes, void *stream) {
  if (!hk || !hv) return fail(ISKV_ERR_ARG, "iskv_decode_attention: null history handle");
  const void *ke[1] = {k_exact};
  const int32_t *kp[1] = {k_exact_pos};
  const int64_t nk[1] = {n_k_exact};
  const void *ve[1] = {v_exact};
  const int32_t *vp[1] = {v_exact_pos};
  const int64_t nv[1] = {n_v_exact};
  const int64_t nt[1] = {n_total};
  const float *qq[1] = {q};
  float *oo[1] = {out};
  return iskv_decode_attention_batched(hk, hv, 1, ke, kp, nk, ve, vp, nv, exact_dtype, nt,
                                       n_q_heads, n_kv_heads, head_dim, rope_theta, scale, qq, oo,
                                       ws, ws_bytes, stream);
}

// ------------------------------------------------------------------------------------------------
// Prompt-block selection
size_t iskv_select_workspace_size(int64_t L, int32_t n_heads, int32_t block) {
  if (L < 1 || n_heads < 1 || block < 1) return 0;
  return select_ws_layout(L, n_heads, block).total;
}

iskv_status iskv_select_prompt_blocks(const void *keys, int32_t k_dtype, int64_t L,
                                      int32_t n_heads, int32_t head_dim, int32_t block,
                                      int32_t per_head, int32_t suffix_blocks, int32_t v_radius,
                                      int32_t *pk_out, int32_t *pv_out, int32_t *head_blocks_out,
                                      int64_t *counts_out, void *ws, size_t ws_bytes,
                                      void *stream) {
  const char *who = "iskv_select_prompt_blocks";
  g_last_error.clear();
  if (!keys || !pk_out || !pv_out || !head_blocks_out || !counts_out)
    return fail(ISKV_ERR_ARG, "%s: null pointer", who);
  if (k_dtype != ISKV_F32 && k_dtype != ISKV_BF16)
    return fail(ISKV_ERR_ARG, "%s: keys must be float32 or bf16", who);
  if (L < 1 || L > ((int64_t)1 << 24)) return fail(ISKV_ERR_SHAPE, "%s: need 1 <= L <= 2^24", who);
  if (n_heads < 1 || n_heads > 64 || head_dim < 2 || head_dim > 256 || head_dim % 2)
    return fail(ISKV_ERR_SHAPE, "%s: need n_heads <= 64, even head_dim <= 256", who);
  if (block < 1 || block > 64 || per_head < 0 || per_head > 4096 || suffix_blocks < 0 ||
      v_radius < 0)
    return fail(ISKV_ERR_SHAPE, "%s: bad block / per_head / suffix / radius", who);
  const size_t need = iskv_select_workspace_size(L, n_heads, block);
  iskv_status st = check_ws(ws, ws_bytes, need, who);
  if (st != ISKV_OK) return st;
  SelectArgs a;
  a.keys = keys;
  a.k_dtype = k_dtype;
  a.L = L;
  a.H = n_heads;
  a.hd = head_dim;
  a.block = block;
  a.per_head = per_head;
  a.suffix_blocks = suffix_blocks;
  a.v_radius = v_radius;
  a.pk_out = pk_out;
  a.pv_out = pv_out;
  a.head_blocks = head_blocks_out;
  a.counts = counts_out;
  a.ws = ws;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  stage_begin(s);
  cudaError_t e = launch_select(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "select");
  stage_mark(s, ST_SELECT);
  return ISKV_OK;
}

// ------------------------------------------------------------------------------------------------
// Cache policy
size_t iskv_cache_prefill_workspace_size(int32_t init_window) {
  (void)init_window;
  return 256;  // an int64[4] scratch word: live-row count and error bits
}

iskv_status iskv_cache_prefill(iskv_exact_table *t, const void *X, int32_t x_dtype, int64_t L,
                               const int32_t *protected_pos, int64_t n_protected,
                               int32_t init_window, void *comp_rows, int32_t *comp_pos,
                               int64_t *n_comp, void *ws, size_t ws_bytes, void *stream) {
  const char *who = "iskv_cache_prefill";
  g_last_error.clear();
  iskv_status st = check_table(t, who);
  if (st != ISKV_OK) return st;
  if (!valid_dtype(x_dtype)) return fail(ISKV_ERR_ARG, "%s: bad X dtype", who);
  if (!n_comp) return fail(ISKV_ERR_ARG, "%s: null n_comp", who);
  if (L < 0 || L >= (int64_t)1 << 31) return fail(ISKV_ERR_SHAPE, "%s: L out of range", who);
  if (L > 0 && (!X || !comp_rows || !comp_pos))
    return fail(ISKV_ERR_ARG, "%s: null X / comp_rows / comp_pos", who);
  if (!aligned(X, elem_size(x_dtype)) || !aligned(comp_rows, elem_size(x_dtype)) ||
      !aligned(comp_pos, 4) || !aligned(protected_pos, 4))
    return fail(ISKV_ERR_ARG, "%s: misaligned X / comp_rows / positions", who);
  if (n_protected < 0 || n_protected > L)
    return fail(ISKV_ERR_SHAPE, "%s: need 0 <= n_protected <= L", who);
  if (n_protected > 0 && !protected_pos) return fail(ISKV_ERR_ARG, "%s: null protected_pos", who);
  if (init_window < 0 || init_window > t->window)
    return fail(ISKV_ERR_ARG, "%s: need 0 <= init_window <= window", who);
  const int64_t w = init_window < L ? init_window : L;
  if (n_protected + w > t->cap_e)
    return fail(ISKV_ERR_CAPACITY, "%s: %lld protected + %lld window rows exceed cap_e = %lld", who,
                (long long)n_protected, (long long)w, (long long)t->cap_e);
  st = check_ws(ws, ws_bytes, iskv_cache_prefill_workspace_size(init_window), who);
  if (st != ISKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int64_t *scal = static_cast<int64_t *>(ws);
  PrefillArgs a;
  a.X = X;
  a.P = protected_pos;
  a.rows = t->rows;
  a.pos = t->pos;
  a.comp = comp_rows;
  a.comp_pos = comp_pos;
  a.st = scal;
  a.L = L;
  a.n_p = n_protected;
  a.w = w;
  a.d = t->d;
  a.x_dtype = x_dtype;
  a.t_dtype = t->dtype;
  int64_t hst[4] = {0, 0, 0, 0};
  cudaError_t e = cudaMemsetAsync(scal, 0, sizeof hst, s);
  if (e == cudaSuccess) e = launch_prefill_partition(a, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(hst, scal, sizeof hst, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && w > 0)
    e = cudaMemcpyAsync(t->live_host, t->pos + n_protected, sizeof(int32_t) * (size_t)w,
                        cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cache prefill");
  const int64_t n_live = hst[0];
  if ((hst[ISKV_META_STATUS] >> ISKV_ERR_ARG) & 1 || n_live < 0 || n_live > w)
    return fail(ISKV_ERR_ARG, "%s: protected positions must be strictly ascending inside [0, L)",
                who);
  t->n_prot = n_protected;
  t->n_live = n_live;
  t->last = L - 1;
  t->fold_rows = 0;
  t->hist_rows = L - n_protected - n_live;
  t->refit_done = t->refit_rows > 0 ? 0 : 1;
  *n_comp = t->hist_rows;
  if ((hst[ISKV_META_STATUS] >> ISKV_ERR_NONFINITE) & 1)
    return fail(ISKV_ERR_NONFINITE, "%s: a finite row value overflows the fp16 table", who);
  return ISKV_OK;
}

size_t iskv_cache_step_workspace_size(int32_t count, int32_t d, int32_t r_max, int32_t block,
                                      int64_t n_cap, int32_t refit_rows) {
  if (count < 1 || d < 1 || r_max < 1 || block < 1 || n_cap < 0 || refit_rows < 0) return 0;
  size_t need = jobs_bytes(count, sizeof(AppendJob));
  const size_t ev = jobs_bytes(count, sizeof(EvictJob));
  const size_t fw = iskv_fold_workspace_size(count, d, r_max, block);
  const size_t rw = iskv_reorth_workspace_size(count, d, r_max, n_cap);
  if (ev > need) need = ev;
  if (fw > need) need = fw;
  if (rw > need) need = rw;
  if (refit_rows > 0 && refit_in_one_fold(d, r_max, refit_rows)) {
    const size_t fr = iskv_fold_workspace_size(count, d, r_max, refit_rows);
    if (fr > need) need = fr;
  } else if (refit_rows > 0) {
    const int32_t rw = wide_refit_rank(d, r_max, block, refit_rows);
    if (rw > 0) {
      const size_t wr = wide_ws(d, rw, block, n_cap).total;
      if (wr > need) need = wr;
    }
  }
  return need;
}

iskv_status iskv_cache_step(iskv_exact_table *const *tables, const iskv_lowrank *const *hists,
                            int32_t count, const void *new_rows, int32_t row_dtype, float tau_rel,
                            int32_t *folded, int32_t *reorthed, void *ws, size_t ws_bytes,
                            void *stream) {
  const char *who = "iskv_cache_step";
  g_last_error.clear();
  if (!tables || !hists || !new_rows) return fail(ISKV_ERR_ARG, "%s: null argument", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  if (!valid_dtype(row_dtype)) return fail(ISKV_ERR_ARG, "%s: bad row dtype", who);
  if (!(tau_rel >= 0.f)) return fail(ISKV_ERR_ARG, "%s: tau_rel must be >= 0", who);
  if (!aligned(new_rows, elem_size(row_dtype))) return fail(ISKV_ERR_ARG, "%s: misaligned rows", who);
  bool any_reorth = false;
  int32_t refit_max = 0;
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_table(tables[i], who);
    if (st != ISKV_OK) return st;
    if ((st = check_handle(hists[i], who)) != ISKV_OK) return st;
    const iskv_exact_table *T = tables[i], *T0 = tables[0];
    if (T->d != T0->d || T->window != T0->window || T->block != T0->block || T->dtype != T0->dtype)
      return fail(ISKV_ERR_SHAPE, "%s: tables must share d, window, block and dtype", who);
    const iskv_lowrank *H = hists[i], *H0 = hists[0];
    if (H->d != T0->d || H->r_max != H0->r_max || H->storage != H0->storage || H->n_cap != H0->n_cap)
      return fail(ISKV_ERR_SHAPE, "%s: histories must have the tables' d and share r_max, storage, "
                  "n_cap", who);
    if ((st = check_room(T, i, who)) != ISKV_OK) return st;
    if (T->reorth_rows > 0) any_reorth = true;
    if (!T->refit_done && T->refit_rows > refit_max) refit_max = T->refit_rows;
  }
  const iskv_exact_table *T0 = tables[0];
  const int d = T0->d, b = T0->block, r = hists[0]->r_max;
  const int64_t ncap = hists[0]->n_cap;
  // The fold's and re-orthogonalisation's own argument checks, made before anything is launched.
  if (b < 8 || b % 8 || b > 128 || b > d)
    return fail(ISKV_ERR_SHAPE, "%s: need 8 <= block <= min(d, 128), block %% 8 == 0", who);
  if (fold_residual_smem(d, b) > 200 * 1024)
    return fail(ISKV_ERR_SHAPE, "%s: d = %d with block = %d exceeds the residual QR cluster", who,
                d, b);
  {
    JacobiCfg jc;
    if (!core_cfg(r, b, false, jc))
      return fail(ISKV_ERR_SHAPE, "%s: r_max + block too large for the core SVD cluster", who);
    if (any_reorth && !core_cfg(r, 0, true, jc))
      return fail(ISKV_ERR_SHAPE, "%s: r_max too large for the dense core SVD", who);
  }
  const size_t need = iskv_cache_step_workspace_size(count, d, r, b, ncap, refit_max);
  iskv_status st = check_ws(ws, ws_bytes, need, who);
  if (st != ISKV_OK) return st;

  // The plan of the step, from the host mirror alone.
  const size_t esz = elem_size(T0->dtype), rsz = elem_size(row_dtype);
  std::vector<AppendJob> aj(count);
  std::vector<int32_t> fold_idx, reorth_idx;
  std::vector<TablePlan> plan(count);
  std::vector<int32_t> fold_rows(count, 0);  // rows this step folds per table (b, or refit_rows)
  std::vector<int32_t> fold_blk(count, 0);   // block size of those folds (b, or refit_rows)
  for (int32_t i = 0; i < count; ++i) {
    const iskv_exact_table *T = tables[i];
    const int64_t t = T->last + 1, slot = T->n_prot + T->n_live;
    AppendJob &j = aj[i];
    j.src = static_cast<const char *>(new_rows) + (size_t)i * d * rsz;
    j.dst = static_cast<char *>(T->rows) + (size_t)slot * d * esz;
    j.dst_pos = T->pos + slot;
    j.meta = hists[i]->meta;
    j.position = (int32_t)t;
    j.pad_ = 0;
    if ((st = plan_table(T, d, r, ncap, i, who, plan[i])) != ISKV_OK) return st;
    if (plan[i].rows > 0) {
      fold_idx.push_back(i);
      fold_rows[i] = plan[i].rows;
      fold_blk[i] = plan[i].rw > 0 ? 0 : plan[i].blk;  // wide refits fold on their own below
    }
    if (plan[i].reorth) reorth_idx.push_back(i);
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char *base = static_cast<char *>(ws);
  AppendJob *daj = reinterpret_cast<AppendJob *>(base);
  stage_begin(s);
  cudaError_t e = upload_jobs(daj, aj.data(), sizeof(AppendJob) * count, s);
  if (e == cudaSuccess) e = launch_cache_append(daj, count, d, row_dtype, T0->dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "cache step: append");
  stage_mark(s, ST_CACHE_APPEND);
  const int nf = (int)fold_idx.size();
  if (nf > 0) {
    std::vector<EvictJob> ej(nf);
    for (int k = 0; k < nf; ++k) {
      const iskv_exact_table *T = tables[fold_idx[k]];
      ej[k].rows = static_cast<char *>(T->rows) + (size_t)T->n_prot * d * esz;
      ej[k].pos = T->pos + T->n_prot;
      ej[k].keep = T->n_live + 1 - fold_rows[fold_idx[k]];
      ej[k].row_bytes = (int64_t)d * esz;
      ej[k].shift = fold_rows[fold_idx[k]];
      ej[k].pad_ = 0;
    }
    // Batched folds per block size; pass j of a block size folds the j-th block of the FIFO of
    // every table with that block size that folds more than j blocks (regular folds and one-fold
    // refits take pass 0 only, a refit by b-row folds passes 0 .. refit_rows / b - 1).
    std::vector<int32_t> sizes;
    for (int32_t i : fold_idx)
      if (fold_blk[i] > 0 && std::find(sizes.begin(), sizes.end(), fold_blk[i]) == sizes.end())
        sizes.push_back(fold_blk[i]);
    std::sort(sizes.begin(), sizes.end());
    for (int32_t fb : sizes) {
      int32_t passes = 0;
      for (int32_t i : fold_idx)
        if (fold_blk[i] == fb && fold_rows[i] / fb > passes) passes = fold_rows[i] / fb;
      for (int32_t j = 0; j < passes; ++j) {
        std::vector<iskv_lowrank> fh;
        std::vector<const void *> F;
        std::vector<const int32_t *> fp;
        for (int32_t i : fold_idx) {
          if (fold_blk[i] != fb || fold_rows[i] / fb <= j) continue;
          const iskv_exact_table *T = tables[i];
          const int64_t row0 = T->n_prot + (int64_t)j * fb;
          fh.push_back(*hists[i]);
          F.push_back(static_cast<const char *>(T->rows) + (size_t)row0 * d * esz);
          fp.push_back(T->pos + row0);
        }
        st = iskv_fold_block_batched(fh.data(), (int32_t)fh.size(), F.data(), T0->dtype, fb,
                                     fp.data(), tau_rel, ws, ws_bytes, stream);
        if (st != ISKV_OK) return st;
      }
    }
    // Wide refits, one table at a time (a first refit happens once per side): the history is
    // copied into a wide one of rank rw inside the workspace, the refit rows are folded into it
    // in b-row blocks (none truncates before the last), and its top r components come back.
    for (int32_t i : fold_idx) {
      if (plan[i].rw == 0) continue;
      const iskv_exact_table *T = tables[i];
      const iskv_lowrank *H = hists[i];
      const int32_t rw = plan[i].rw;
      const WideWs W = wide_ws(d, rw, b, ncap);
      WidenArgs wa;
      wa.U = H->U;
      wa.B = H->B;
      wa.sigma = H->sigma;
      wa.pos = H->pos;
      wa.meta = H->meta;
      wa.Uw = base + W.U;
      wa.Bw = base + W.B;
      wa.sigw = reinterpret_cast<float *>(base + W.sig);
      wa.posw = reinterpret_cast<int32_t *>(base + W.pos);
      wa.metaw = reinterpret_cast<int64_t *>(base + W.meta);
      wa.n_cap = ncap;
      wa.d = d;
      wa.r = r;
      wa.rw = rw;
      wa.esz = (int)elem_size(H->storage);
      if ((e = launch_history_widen(wa, s)) != cudaSuccess) return cuda_fail(e, "refit: widen");
      iskv_lowrank hw = *H;
      hw.r_max = rw;
      hw.U = wa.Uw;
      hw.B = wa.Bw;
      hw.sigma = wa.sigw;
      hw.pos = wa.posw;
      hw.meta = wa.metaw;
      for (int32_t j = 0; j < plan[i].rows / b; ++j) {
        const int64_t row0 = T->n_prot + (int64_t)j * b;
        const void *Fj = static_cast<const char *>(T->rows) + (size_t)row0 * d * esz;
        const int32_t *pj = T->pos + row0;
        st = iskv_fold_block_batched(&hw, 1, &Fj, T0->dtype, b, &pj, tau_rel, base + W.fold,
                                     iskv_fold_workspace_size(1, d, rw, b), stream);
        if (st != ISKV_OK) return st;
      }
      if ((e = launch_history_narrow(wa, s)) != cudaSuccess) return cuda_fail(e, "refit: narrow");
    }
    EvictJob *dej = reinterpret_cast<EvictJob *>(base);
    stage_begin(s);
    e = upload_jobs(dej, ej.data(), sizeof(EvictJob) * nf, s);
    if (e == cudaSuccess) e = launch_cache_evict(dej, nf, s);
    if (e != cudaSuccess) return cuda_fail(e, "cache step: evict");
    stage_mark(s, ST_CACHE_EVICT);
  }
  const int nr = (int)reorth_idx.size();
  if (nr > 0) {
    std::vector<iskv_lowrank> rh(nr);
    for (int k = 0; k < nr; ++k) rh[k] = *hists[reorth_idx[k]];
    st = iskv_reorth(rh.data(), nr, ws, ws_bytes, stream);
    if (st != ISKV_OK) return st;
  }

  // Host mirror.
  for (int32_t i = 0; i < count; ++i) {
    advance_table(tables[i], plan[i]);
    if (folded) folded[i] = plan[i].rows > 0 ? (plan[i].refit ? 2 : 1) : 0;
    if (reorthed) reorthed[i] = plan[i].reorth ? 1 : 0;
  }
  return ISKV_OK;
}

// ------------------------------------------------------------------------------------------------
// Prompt compression (Algorithm 1 step 7) by block folds.
size_t iskv_compress_prompt_workspace_size(int32_t count, int32_t d, int32_t r_max, int32_t block) {
  if (count < 1 || d < 1 || r_max < 1 || block < 1) return 0;
  size_t need = align_up(iskv_fold_workspace_size(count, d, r_max, block), 256);
  need += jobs_bytes(count, sizeof(TailJob));
  need += (size_t)count * align_up((size_t)block * d * sizeof(float), 256);
  need += (size_t)count * align_up((size_t)block * sizeof(int32_t), 256);
  return need;
}

iskv_status iskv_compress_prompt(const iskv_lowrank *hs, int32_t count, const void *const *rows,
                                 const int32_t *const *pos, const int64_t *n_rows, int32_t dtype,
                                 int32_t block, float tau_rel, void *ws, size_t ws_bytes,
                                 void *stream) {
  const char *who = "iskv_compress_prompt";
  g_last_error.clear();
  if (!hs || !rows || !pos || !n_rows) return fail(ISKV_ERR_ARG, "%s: null host array", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  if (!valid_dtype(dtype)) return fail(ISKV_ERR_ARG, "%s: bad dtype", who);
  if (!(tau_rel >= 0.f)) return fail(ISKV_ERR_ARG, "%s: tau_rel must be >= 0", who);
  int64_t nb_max = 0;
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_handle(&hs[i], who);
    if (st != ISKV_OK) return st;
    if (hs[i].d != hs[0].d || hs[i].r_max != hs[0].r_max || hs[i].storage != hs[0].storage)
      return fail(ISKV_ERR_SHAPE, "%s: histories must share d, r_max, storage", who);
    if (n_rows[i] < 0) return fail(ISKV_ERR_SHAPE, "%s: negative row count", who);
    if (n_rows[i] > 0 && (!rows[i] || !pos[i]))
      return fail(ISKV_ERR_ARG, "%s: null rows or positions", who);
    if (n_rows[i] > 0 && (!aligned(rows[i], 16) || !aligned(pos[i], 4)))
      return fail(ISKV_ERR_ARG, "%s: rows must be 16-byte aligned", who);
    if (n_rows[i] / block > nb_max) nb_max = n_rows[i] / block;
  }
  const int d = hs[0].d, r = hs[0].r_max;
  if (block < 8 || block % 8 || block > 128 || block > d)
    return fail(ISKV_ERR_SHAPE, "%s: need 8 <= block <= min(d, 128), block %% 8 == 0", who);
  const size_t need = iskv_compress_prompt_workspace_size(count, d, r, block);
  iskv_status st = check_ws(ws, ws_bytes, need, who);
  if (st != ISKV_OK) return st;
  const size_t esz = elem_size(dtype), fw = align_up(iskv_fold_workspace_size(count, d, r, block), 256);
  char *base = static_cast<char *>(ws);
  TailJob *tjobs = reinterpret_cast<TailJob *>(base + fw);
  char *tbuf = base + fw + jobs_bytes(count, sizeof(TailJob));
  const size_t rowbuf = align_up((size_t)block * d * sizeof(float), 256);
  char *pbuf = tbuf + (size_t)count * rowbuf;
  const size_t posbuf = align_up((size_t)block * sizeof(int32_t), 256);
  // Full blocks: pass j folds block j of every history that has more than j of them.
  for (int64_t j = 0; j < nb_max; ++j) {
    std::vector<iskv_lowrank> fh;
    std::vector<const void *> F;
    std::vector<const int32_t *> fp;
    for (int32_t i = 0; i < count; ++i) {
      if (n_rows[i] / block <= j) continue;
      fh.push_back(hs[i]);
      F.push_back(static_cast<const char *>(rows[i]) + (size_t)j * block * d * esz);
      fp.push_back(pos[i] + j * block);
    }
    st = iskv_fold_block_batched(fh.data(), (int32_t)fh.size(), F.data(), dtype, block, fp.data(),
                                 tau_rel, ws, fw, stream);
    if (st != ISKV_OK) return st;
  }
  // Short last blocks, one batched fold per padded size.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int32_t t8 = 8; t8 <= block; t8 += 8) {
    std::vector<TailJob> tj;
    std::vector<iskv_lowrank> fh;
    std::vector<const void *> F;
    std::vector<const int32_t *> fp;
    for (int32_t i = 0; i < count; ++i) {
      const int32_t t = (int32_t)(n_rows[i] % block);
      if (t == 0 || (t + 7) / 8 * 8 != t8) continue;
      const int64_t row0 = n_rows[i] - t;
      const int k = (int)tj.size();
      TailJob j;
      j.src = static_cast<const char *>(rows[i]) + (size_t)row0 * d * esz;
      j.src_pos = pos[i] + row0;
      j.dst = tbuf + (size_t)k * rowbuf;
      j.dst_pos = reinterpret_cast<int32_t *>(pbuf + (size_t)k * posbuf);
      j.meta = hs[i].meta;
      j.row_bytes = (int64_t)d * (int64_t)esz;
      j.n0 = 0;
      j.t = t;
      j.t8 = t8;
      tj.push_back(j);
      fh.push_back(hs[i]);
      F.push_back(j.dst);
      fp.push_back(j.dst_pos);
    }
    if (tj.empty()) continue;
    const int nt = (int)tj.size();
    cudaError_t e = upload_jobs(tjobs, tj.data(), sizeof(TailJob) * nt, s);
    if (e == cudaSuccess) e = launch_tail_pad(tjobs, nt, s);
    if (e != cudaSuccess) return cuda_fail(e, "compress prompt: pad");
    st = iskv_fold_block_batched(fh.data(), nt, F.data(), dtype, t8, fp.data(), tau_rel, ws, fw,
                                 stream);
    if (st != ISKV_OK) return st;
    if ((e = launch_tail_drop(tjobs, nt, s)) != cudaSuccess)
      return cuda_fail(e, "compress prompt: drop");
  }
  return ISKV_OK;
}

iskv_status iskv_cache_plan(iskv_exact_table *const *tables, int32_t count, int32_t r_max,
                            int64_t n_cap, int32_t advance, int32_t *folded, int32_t *reorthed) {
  const char *who = "iskv_cache_plan";
  g_last_error.clear();
  if (!tables) return fail(ISKV_ERR_ARG, "%s: null tables", who);
  if (count < 1 || count > 4096) return fail(ISKV_ERR_SHAPE, "%s: count must be in [1, 4096]", who);
  if (r_max < 1 || n_cap < 0) return fail(ISKV_ERR_SHAPE, "%s: bad r_max / n_cap", who);
  std::vector<TablePlan> plan(count);
  for (int32_t i = 0; i < count; ++i) {
    iskv_status st = check_table(tables[i], who);
    if (st != ISKV_OK) return st;
    if ((st = check_room(tables[i], i, who)) != ISKV_OK) return st;
    if ((st = plan_table(tables[i], tables[i]->d, r_max, n_cap, i, who, plan[i])) != ISKV_OK)
      return st;
  }
  for (int32_t i = 0; i < count; ++i) {
    if (folded) folded[i] = plan[i].rows > 0 ? (plan[i].refit ? 2 : 1) : 0;
    if (reorthed) reorthed[i] = plan[i].reorth ? 1 : 0;
    if (advance) advance_table(tables[i], plan[i]);
  }
  return ISKV_OK;
}

// ------------------------------------------------------------------------------------------------
iskv_status iskv_reset(const iskv_lowrank *h, void *stream) {
  g_last_error.clear();
  iskv_status st = check_handle(h, "iskv_reset");
  if (st != ISKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t es = h->storage == ISKV_F32 ? 4 : 2;
  cudaError_t e = cudaMemsetAsync(h->meta, 0, 4 * sizeof(int64_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->sigma, 0, sizeof(float) * h->r_max, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->U, 0, es * (size_t)h->n_cap * h->r_max, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->B, 0, es * (size_t)h->d * h->r_max, s);
  if (e != cudaSuccess) return cuda_fail(e, "iskv_reset");
  return ISKV_OK;
}

iskv_status iskv_get_status(const iskv_lowrank *h, int64_t *k, int64_t *n, int64_t *folds,
                            int64_t *status_bits) {
  g_last_error.clear();
  iskv_status st = check_handle(h, "iskv_get_status");
  if (st != ISKV_OK) return st;
  int64_t m[4];
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(m, h->meta, sizeof m, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "iskv_get_status");
  if (k) *k = m[ISKV_META_K];
  if (n) *n = m[ISKV_META_N];
  if (folds) *folds = m[ISKV_META_FOLDS];
  if (status_bits) *status_bits = m[ISKV_META_STATUS];
  return ISKV_OK;
}

}  // extern "C"

extern "C" iskv_status iskv_selftest_wait_timeout(int64_t *meta, int64_t limit_ns, void *stream) {
  g_last_error.clear();
  if (!meta || !aligned(meta, 8)) return fail(ISKV_ERR_ARG, "selftest: meta must be 8-byte aligned");
  int64_t ns = limit_ns < 100000 ? 100000 : (limit_ns > 2000000000 ? 2000000000 : limit_ns);
  cudaError_t e = launch_wait_timeout(meta, (uint64_t)ns, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest: launch");
  return ISKV_OK;
}
