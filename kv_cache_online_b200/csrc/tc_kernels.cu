// Tensor-core (tcgen05) kernels for the two dense contractions that sweep every history row:
//
//  * coordinate rotation (iS-KV reading notes, Algorithm 2 step 7; Section 4.4):
//      U[0:n] <- U[0:n] G,  in place, bf16 factors, fp32 accumulation in tensor memory;
//  * reconstruction (Algorithm 3 steps 7-8):
//      out[pos_i] = RoPE_pos_i( U_i (diag(sigma) B^T) ),  bf16 out, RoPE fused into the epilogue.
//
// Both are persistent kernels over 128-row tiles of U. Roles: warp 0 issues TMA loads (U tiles,
// and the small right-hand operand), warp 1 owns tensor memory and issues tcgen05.mma from one
// thread, warps 2-9 drain the fp32 accumulators from tensor memory (each warp reads the 32 TMEM
// lanes it may access, i.e. 32 rows) and write the results. The U tile is held as r/64 K-slabs of
// 16 KB; each slab is released to the producer as soon as the last MMA reading it completes, so the
// next tile's loads overlap the current tile's MMAs. Two TMEM accumulator buffers let the epilogue
// of one tile (or head) overlap the MMAs of the next.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "profiling.h"
#include "recon.h"
#include "tc.h"
#include "tc_sm100.cuh"

namespace iskv {

using namespace tc;

constexpr int TC_THREADS = 320;        // 10 warps
constexpr int TC_M = 128;              // rows per tile
constexpr int SLAB_BYTES = 128 * 128;  // 128 rows x 64 bf16
constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait

struct TcCtl {
  uint64_t a_full[4], a_empty[4];
  uint64_t b_full[2], b_empty[2];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t done;
  uint32_t tmem;
  int abort;
};

// ------------------------------------------------------------------------------------------------
// Tile iteration shared by all roles: contiguous ranges of (job, 128-row tile) per CTA.
struct TileRange {
  int begin, end, tiles_per_job;
};

ISKV_DEV TileRange my_tiles(int count, int tiles_per_job) {
  const int total = count * tiles_per_job;
  const int per = (total + gridDim.x - 1) / gridDim.x;
  TileRange t;
  t.begin = blockIdx.x * per;
  t.end = min(total, t.begin + per);
  t.tiles_per_job = tiles_per_job;
  return t;
}

template <class Ctl>
ISKV_DEV void fail_timeout(Ctl *c, int64_t *meta) {
  c->abort = 1;
  if (meta) record_status(meta, ISKV_ERR_TIMEOUT);
}

// Two bf16 values (low half first) as two fp16 values, each rounded to nearest: exact for
// magnitudes in fp16's normal range [2^-14, 65504].
ISKV_DEV uint32_t bf16x2_to_f16x2(uint32_t x) {
  const __half2 h = __floats2half2_rn(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
  return *reinterpret_cast<const uint32_t *>(&h);
}

// ================================================================================================
// In-place rotations of a factor's rows on the tensor cores (bf16 factors):
//   mode 0, coordinate rotation (Algorithm 2 step 7; the re-orthogonalisation's U <- U T_U):
//     U[0:n] <- U[0:n] G, mapA = U, mapB = G^T (r x r);
//   mode 1, basis rotation (Algorithm 2 step 8; the re-orthogonalisation's B <- B T_B):
//     B[0:d] <- [B | P] H, mapA = B, mapO = P (d x bpad fp16), mapB = H^T (r x (r + bpad)).
// The operands are fp16 (11-bit significand): the rotations' entries lie in [-1, 1] and the
// factors' columns have unit norm, so nothing leaves fp16's range, while bf16 operands (8 bits)
// would scale every output column by the rounding of its near-one entry: one coherent 2^-9 error
// per column and rotation, which a trajectory of folds accumulates. A tile is 128 rows; its K
// slabs 0 .. r/64 - 1 come from mapA as bf16 and are converted to fp16 in shared memory, the
// rest from mapO as fp16. The rotation's transpose stays resident per history while the A slabs
// stream through a ring of p.stages 16 KB stages. Warp 0 loads, warp 1 issues the MMAs (M = 128,
// N = r, accumulators double-buffered in TMEM), warps 2-9 write bf16 rows in place (a tile's rows
// are read only by that tile), warps 10-13 convert.
constexpr int ROT_MAX_STAGES = 8;
constexpr int ROT_THREADS = 448;        // 14 warps
constexpr int ROT_STG_BYTES = 32 * 128;  // one epilogue warp's staged rows

struct RotCtl {
  uint64_t a_full[ROT_MAX_STAGES], a_conv[ROT_MAX_STAGES], a_empty[ROT_MAX_STAGES];
  uint64_t b_full, b_empty;
  uint64_t acc_full[2], acc_empty[2];
  uint64_t done;
  uint32_t tmem;
  int abort;
};

__global__ void __launch_bounds__(ROT_THREADS, 1) k_rotate_tc(const TcJob *jobs, TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int R = p.r, KS = p.kslabs, KB = R / 64, N = R, NS = p.stages;
  uint8_t *sB = smem;                        // KS slabs x (N x 128 B)
  uint8_t *sA = smem + KS * N * 128;         // NS x 16 KB
  uint8_t *sStg = sA + NS * SLAB_BYTES;      // p.stg: 8 warps x (32 rows x 128 B), SW128
  RotCtl *ctl = reinterpret_cast<RotCtl *>(sStg + (p.stg ? 8 * ROT_STG_BYTES : 0));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = N <= 64 ? 128 : (N <= 128 ? 256 : 512);
  const uint32_t idesc = idesc_f16_f32(TC_M, N);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&ctl->a_full[s], 1);
      mbar_init(&ctl->a_conv[s], 4);
      mbar_init(&ctl->a_empty[s], 1);
    }
    mbar_init(&ctl->b_full, 1);
    mbar_init(&ctl->b_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->acc_full[i], 1);
      mbar_init(&ctl->acc_empty[i], 8);
    }
    mbar_init(&ctl->done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&ctl->tmem, ncols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int *abort = &ctl->abort;
  const TileRange tr = my_tiles(p.count, p.tiles_per_job);
  // Per-thread cache of the current history's row count: every role tests every tile, and the
  // scalars change only with the history, so they are read from global memory once per history.
  int cache_j = -1, cache_n = 0;
  auto rows_of = [&](int j) -> int {
    if (j != cache_j) {
      const int32_t *sc = jobs[j].sc;
      cache_j = j;
      cache_n = sc[FS_SKIP] ? 0 : (p.mode ? p.d : (sc[FS_K_OLD] == 0 ? 0 : sc[FS_N_OLD]));
    }
    return cache_n;
  };

  if (warp == 0 && lane == 0) {
    // ---------------- producer
    int cur = -1, nb = 0;
    uint32_t gsl = 0;  // A slabs issued so far
    bool ok = true;
    for (int t = tr.begin; t < tr.end && ok && !*abort; ++t) {
      const int j = t / tr.tiles_per_job, row0 = (t % tr.tiles_per_job) * TC_M;
      const TcJob &jb = jobs[j];
      if (row0 >= rows_of(j)) continue;
      if (j != cur) {
        if (nb > 0 && !mbar_wait(&ctl->b_empty, (nb - 1) & 1, abort, WAIT_NS)) {
          fail_timeout(ctl, jb.meta);
          break;
        }
        tensormap_acquire(&jb.mapA);
        if (KS > KB) tensormap_acquire(&jb.mapO);
        tensormap_acquire(&jb.mapB);
        mbar_arrive_expect_tx(&ctl->b_full, KS * N * 128);
        for (int s = 0; s < KS; ++s) tma_load_2d(sB + s * N * 128, &jb.mapB, s * 64, 0, &ctl->b_full);
        cur = j;
        ++nb;
      }
      for (int s = 0; s < KS; ++s, ++gsl) {
        const uint32_t st = gsl % NS, use = gsl / NS;
        if (use > 0 && !mbar_wait(&ctl->a_empty[st], (use - 1) & 1, abort, WAIT_NS)) {
          fail_timeout(ctl, jb.meta);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&ctl->a_full[st], SLAB_BYTES);
        if (s < KB) tma_load_2d(sA + st * SLAB_BYTES, &jb.mapA, s * 64, row0, &ctl->a_full[st]);
        else tma_load_2d(sA + st * SLAB_BYTES, &jb.mapO, (s - KB) * 64, row0, &ctl->a_full[st]);
      }
    }
    // Let every load this thread issued land before the CTA can exit.
    for (uint32_t i = gsl > (uint32_t)NS ? gsl - NS : 0; i < gsl; ++i)
      mbar_wait(&ctl->a_full[i % NS], (i / NS) & 1, abort, WAIT_NS / 4);
    if (nb > 0) mbar_wait(&ctl->b_full, (nb - 1) & 1, abort, WAIT_NS / 4);
  } else if (warp >= 10) {
    // ---------------- converters: bf16 slabs to fp16 in place (elementwise, so the swizzled
    // layout is kept); mapO's slabs arrive as fp16.
    const int ct = threadIdx.x - 10 * 32;  // 0 .. 127
    uint32_t gsl = 0;
    for (int t = tr.begin; t < tr.end && !__any_sync(~0u, *abort != 0); ++t) {
      const int j = t / tr.tiles_per_job, row0 = (t % tr.tiles_per_job) * TC_M;
      const TcJob &jb = jobs[j];
      if (row0 >= rows_of(j)) continue;
      bool ok = true;
      for (int s = 0; s < KS; ++s, ++gsl) {
        const uint32_t st = gsl % NS;
        if (!__all_sync(~0u, mbar_wait(&ctl->a_full[st], (gsl / NS) & 1, abort, WAIT_NS))) {
          ok = false;
          break;
        }
        if (s < KB) {
          uint4 *w = reinterpret_cast<uint4 *>(sA + st * SLAB_BYTES);
#pragma unroll
          for (int i = 0; i < SLAB_BYTES / 16 / 128; ++i) {
            uint4 v = w[ct + 128 * i];
            v.x = bf16x2_to_f16x2(v.x);
            v.y = bf16x2_to_f16x2(v.y);
            v.z = bf16x2_to_f16x2(v.z);
            v.w = bf16x2_to_f16x2(v.w);
            w[ct + 128 * i] = v;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->a_conv[st]);
      }
      if (!ok) { fail_timeout(ctl, jb.meta); break; }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int cur = -1, nb = 0, na = 0;
    RingPos rp;
    const uint64_t da0 = sw128_desc(smem_u32(sA)), db0 = sw128_desc(smem_u32(sB));
    for (int t = tr.begin; t < tr.end && !*abort; ++t) {
      const int j = t / tr.tiles_per_job, row0 = (t % tr.tiles_per_job) * TC_M;
      const TcJob &jb = jobs[j];
      if (row0 >= rows_of(j)) continue;
      if (j != cur) {
        if (cur >= 0) mma_commit(&ctl->b_empty);
        if (!mbar_wait(&ctl->b_full, nb & 1, abort, WAIT_NS)) { fail_timeout(ctl, jb.meta); break; }
        cur = j;
        ++nb;
      }
      const int buf = na & 1, use = na >> 1;
      if (use > 0 && !mbar_wait(&ctl->acc_empty[buf], (use - 1) & 1, abort, WAIT_NS)) {
        fail_timeout(ctl, jb.meta);
        break;
      }
      fence_after_sync();
      const uint32_t d = tmem + buf * N;
      bool ok = true;
      for (int s = 0; s < KS; ++s) {
        if (!mbar_wait(&ctl->a_conv[rp.slot], rp.phase, abort, WAIT_NS)) {
          ok = false;
          break;
        }
        fence_after_sync();
        const uint64_t da = desc_add(da0, rp.slot * SLAB_BYTES), db = desc_add(db0, s * N * 128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(d, desc_add(da, kk * 32), desc_add(db, kk * 32), idesc, (s | kk) != 0);
        mma_commit(&ctl->a_empty[rp.slot]);
        rp.next(NS);
      }
      if (!ok) { fail_timeout(ctl, jb.meta); break; }
      mma_commit(&ctl->acc_full[buf]);
      ++na;
    }
    mma_commit(&ctl->done);
    mbar_wait(&ctl->done, 0, abort, WAIT_NS / 4);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> bf16 -> rows (in place). With p.stg each warp stages
    // its 32 rows x 64 columns in shared memory (128-byte swizzled) and lane 0 writes them with
    // one tile store; the last, partial tile of a coordinate rotation keeps per-row stores so
    // that no row at or beyond n is written.
    const int q = warp & 3, half = (warp - 2) >> 2;
    const int cols = N / 2, c0 = half * cols;
    uint8_t *stg = sStg + (warp - 2) * ROT_STG_BYTES;
    bool pending = false;
    int acq = -1, na = 0;
    // Lanes of a warp take every exit together: tcgen05.ld is a warp-wide instruction.
    for (int t = tr.begin; t < tr.end && !__any_sync(~0u, *abort != 0); ++t) {
      const int j = t / tr.tiles_per_job, row0 = (t % tr.tiles_per_job) * TC_M;
      const TcJob &jb = jobs[j];
      const int n = rows_of(j);
      if (row0 >= n) continue;
      const int buf = na & 1, use = na >> 1;
      if (!__all_sync(~0u, mbar_wait(&ctl->acc_full[buf], use & 1, abort, WAIT_NS))) {
        fail_timeout(ctl, jb.meta);
        break;
      }
      fence_after_sync();
      const int rbase = row0 + q * 32, row = rbase + lane;
      const uint32_t tbase = tmem + buf * N + ((uint32_t)(q * 32) << 16) + c0;
      if (p.stg && (p.mode || rbase + 32 <= n)) {
        if (lane == 0 && acq != j) {
          tensormap_acquire(&jb.mapS);
          acq = j;
        }
        for (int cb = 0; cb < cols; cb += 64) {
          // The staged rows are free once the previous tile store has read them.
          if (pending) {
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
          }
#pragma unroll
          for (int cc = 0; cc < 64; cc += 16) {
            float v[16];
            tmem_ld16(tbase + cb + cc, v);
            tmem_ld_wait();
            uint4 w0, w1;
            w0.x = pack_bf16(v[0], v[1]);   w0.y = pack_bf16(v[2], v[3]);
            w0.z = pack_bf16(v[4], v[5]);   w0.w = pack_bf16(v[6], v[7]);
            w1.x = pack_bf16(v[8], v[9]);   w1.y = pack_bf16(v[10], v[11]);
            w1.z = pack_bf16(v[12], v[13]); w1.w = pack_bf16(v[14], v[15]);
            // 16-byte chunk c of a 128-byte staged row sits at chunk c ^ (row & 7).
            const int ck = cc / 8, sw = lane & 7;
            *reinterpret_cast<uint4 *>(stg + lane * 128 + 16 * (ck ^ sw)) = w0;
            *reinterpret_cast<uint4 *>(stg + lane * 128 + 16 * ((ck + 1) ^ sw)) = w1;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&jb.mapS, c0 + cb, rbase, stg);
            bulk_commit();
          }
          pending = true;
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->acc_empty[buf]);
        ++na;
        continue;
      }
      __nv_bfloat16 *U = static_cast<__nv_bfloat16 *>(jb.U) + (size_t)row * R;
      for (int cc = 0; cc < cols; cc += 16) {
        float v[16];
        tmem_ld16(tmem + buf * N + ((uint32_t)(q * 32) << 16) + c0 + cc, v);
        tmem_ld_wait();
        if (row < n) {
          uint4 w0, w1;
          w0.x = pack_bf16(v[0], v[1]);   w0.y = pack_bf16(v[2], v[3]);
          w0.z = pack_bf16(v[4], v[5]);   w0.w = pack_bf16(v[6], v[7]);
          w1.x = pack_bf16(v[8], v[9]);   w1.y = pack_bf16(v[10], v[11]);
          w1.z = pack_bf16(v[12], v[13]); w1.w = pack_bf16(v[14], v[15]);
          uint4 *dst = reinterpret_cast<uint4 *>(U + c0 + cc);
          dst[0] = w0;
          dst[1] = w1;
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->acc_empty[buf]);
      ++na;
    }
    if (lane == 0 && pending) bulk_wait0();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

// ================================================================================================
// Projection of the fold (Algorithm 2 steps 2-3) for bf16 factors and a bf16 block F with b = 64:
// one CTA per history runs four contractions with B, each streaming B from L2 through a ring of
// 64 KB stages (C^T, C2^T: M = k in 128-row tiles, K = d, B read MN-major; E1, E: M = d in 128-row
// tiles, K = k, B read K-major; N = b throughout, accumulators in TMEM):
//   1. C^T  = B^T F^T           F exact in bf16;
//   2. E1   = F - C B^T         C rounded to bf16 (kept as the MMA operand in shared memory);
//   3. C2^T = B^T E1^T          E1 as two bf16 terms hi + lo (E1 to about 2^-17);
//   4. E    = E1 - C2 B^T       C2 rounded to bf16.
// With B^T B = I, C2 = -(the rounding of C in step 2), so step 4 removes it; what remains in E is
// the rounding of E1 (2^-17 relative) and of C2 (2^-9 of that rounding), far below the bf16
// storage of the factors. C (float32, for the core) and E (float32, for the residual QR) go to the
// workspace; E1's bf16 pair sits in the workspace between steps 2 and 3 (the TMA reads it back).
constexpr int PROJ_STAGES = 3;
constexpr int PROJ_STAGE_BYTES = 64 * 1024;
constexpr int PROJ_B = 64;  // rows of the block

struct ProjCtl {
  uint64_t full[PROJ_STAGES], empty[PROJ_STAGES];
  uint64_t pacc;      // steps 1 and 3: accumulators complete
  uint64_t tacc[8];   // steps 2 and 4: accumulator of d-tile t complete
  uint64_t c_ready;   // C (step 1) / C2 (step 3) staged as bf16 in shared memory (8 warps)
  uint64_t e1_ready;  // E1 written to the workspace (8 warps)
  uint64_t done;
  uint32_t tmem;
  int abort;
};

ISKV_DEV void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__global__ void __launch_bounds__(TC_THREADS, 1) k_project_tc(const ProjJob *jobs, ProjParams p) {
  const ProjJob &jb = jobs[blockIdx.x];
  if (jb.sc[FS_SKIP]) return;  // uniform over the CTA
  // The job's pointers, read once: the stores through them could otherwise alias the job table
  // in the compiler's view and force a reload of each pointer after every store.
  float *__restrict__ const Cw = jb.C;
  float *__restrict__ const Ew = jb.E;
  __nv_bfloat16 *__restrict__ const E1w = jb.E1;
  const __nv_bfloat16 *__restrict__ const Fr = jb.F;
  int64_t *const meta = jb.meta;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int R = p.r, D = p.d, KB = R / 64, MH = R / 128, NT = D / 128, ND = D / 64;
  const int k_old = jb.sc[FS_K_OLD];
  uint8_t *ring = smem;                                     // PROJ_STAGES x 64 KB
  uint8_t *sC = smem + PROJ_STAGES * PROJ_STAGE_BYTES;      // KB slabs x (64 rows x 128 B)
  ProjCtl *ctl = reinterpret_cast<ProjCtl *>(sC + KB * PROJ_B * 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tcols = (NT > MH ? NT : MH) * PROJ_B;
  const uint32_t ncols = tcols <= 32 ? 32 : tcols <= 64 ? 64 : tcols <= 128 ? 128 : tcols <= 256 ? 256 : 512;
  // bf16 A and B, fp32 D; steps 1/3: A (B^T) MN-major, B operand K-major; steps 2/4: both K-major.
  const uint32_t idesc_t = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                           ((uint32_t)(PROJ_B >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
  const uint32_t idesc_n = idesc_bf16_f32(128, PROJ_B);

  // B's columns k_old .. r-1 are cleared (zero after every fold and re-orthogonalisation): the
  // contractions run over all r columns.
  if (k_old < R) {
    __nv_bfloat16 *__restrict__ B = jb.B;
    const int w = R - k_old;
    for (int e = threadIdx.x; e < D * w; e += blockDim.x)
      B[(size_t)(e / w) * R + k_old + e % w] = __float2bfloat16_rn(0.f);
    fence_proxy_async_global();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < PROJ_STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->pacc, 1);
    for (int t = 0; t < 8; ++t) mbar_init(&ctl->tacc[t], 1);
    mbar_init(&ctl->c_ready, 8);
    mbar_init(&ctl->e1_ready, 8);
    mbar_init(&ctl->done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&ctl->tmem, ncols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int *abort = &ctl->abort;

  if (warp == 0 && lane == 0) {
    // ---------------- producer: stages of steps 1-4 in order, one ring
    tensormap_acquire(&jb.mapBm);
    tensormap_acquire(&jb.mapBk);
    tensormap_acquire(&jb.mapF);
    tensormap_acquire(&jb.mapE1);
    uint32_t g = 0;
    bool ok = true;
    for (int step = 0; step < 4 && ok; ++step) {
      if (step == 2 && !mbar_wait(&ctl->e1_ready, 0, abort, WAIT_NS)) { ok = false; break; }
      const bool tstep = (step & 1) == 0;  // steps 1 and 3 (K = d)
      const int n = tstep ? ND : NT;
      for (int i = 0; i < n; ++i, ++g) {
        const uint32_t st = g % PROJ_STAGES, use = g / PROJ_STAGES;
        if (use > 0 && !mbar_wait(&ctl->empty[st], (use - 1) & 1, abort, WAIT_NS)) {
          ok = false;
          break;
        }
        uint8_t *dst = ring + st * PROJ_STAGE_BYTES;
        if (tstep) {
          // B rows [64 i, 64 i + 64) as KB MN-major boxes of 64 columns, then the block's 64
          // columns [64 i, 64 i + 64): F (step 1) or E1 hi and lo (step 3).
          const int nb = step == 0 ? 1 : 2;
          mbar_arrive_expect_tx(&ctl->full[st], KB * 8192 + nb * 8192);
          for (int sl = 0; sl < KB; ++sl)
            tma_load_2d(dst + sl * 8192, &jb.mapBm, sl * 64, i * 64, &ctl->full[st]);
          if (step == 0) {
            tma_load_2d(dst + 32768, &jb.mapF, i * 64, 0, &ctl->full[st]);
          } else {
            tma_load_2d(dst + 32768, &jb.mapE1, i * 64, 0, &ctl->full[st]);
            tma_load_2d(dst + 40960, &jb.mapE1, i * 64, PROJ_B, &ctl->full[st]);
          }
        } else {
          // B rows [128 i, 128 i + 128) as KB K-major boxes of 64 columns.
          mbar_arrive_expect_tx(&ctl->full[st], KB * 16384);
          for (int s = 0; s < KB; ++s)
            tma_load_2d(dst + s * 16384, &jb.mapBk, s * 64, i * 128, &ctl->full[st]);
        }
      }
    }
    if (!ok) fail_timeout(ctl, meta);
    // Let every load this thread issued land before the CTA can exit.
    for (uint32_t i = g > PROJ_STAGES ? g - PROJ_STAGES : 0; i < g; ++i)
      mbar_wait(&ctl->full[i % PROJ_STAGES], (i / PROJ_STAGES) & 1, abort, WAIT_NS / 4);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    uint32_t g = 0;
    bool ok = true;
    for (int step = 0; step < 4 && ok && !*abort; ++step) {
      const bool tstep = (step & 1) == 0;
      // Step 2 needs C staged; step 3 needs TMEM columns of step 2 read out (E1 written);
      // step 4 needs C2 staged.
      if (step == 1 && !mbar_wait(&ctl->c_ready, 0, abort, WAIT_NS)) { ok = false; break; }
      if (step == 2 && !mbar_wait(&ctl->e1_ready, 0, abort, WAIT_NS)) { ok = false; break; }
      if (step == 3 && !mbar_wait(&ctl->c_ready, 1, abort, WAIT_NS)) { ok = false; break; }
      fence_after_sync();
      const int n = tstep ? ND : NT;
      for (int i = 0; i < n; ++i, ++g) {
        const uint32_t st = g % PROJ_STAGES;
        if (!mbar_wait(&ctl->full[st], (g / PROJ_STAGES) & 1, abort, WAIT_NS)) {
          ok = false;
          break;
        }
        fence_after_sync();
        const uint32_t base = smem_u32(ring + st * PROJ_STAGE_BYTES);
        if (tstep) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            for (int h = 0; h < MH; ++h) {
              const uint64_t adesc = sw128_mn_desc(base + h * 16384 + kk * 2048, 8192);
              mma_bf16(tmem + h * PROJ_B, adesc, sw128_desc(base + 32768 + kk * 32), idesc_t,
                       (i | kk) != 0);
              if (step == 2)
                mma_bf16(tmem + h * PROJ_B, adesc, sw128_desc(base + 40960 + kk * 32), idesc_t,
                         true);
            }
          }
        } else {
          const uint32_t c0 = smem_u32(sC);
          for (int s = 0; s < KB; ++s)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmem + i * PROJ_B, sw128_desc(base + s * 16384 + kk * 32),
                       sw128_desc(c0 + s * 8192 + kk * 32), idesc_n, (s | kk) != 0);
          mma_commit(&ctl->tacc[i]);
        }
        mma_commit(&ctl->empty[st]);
      }
      if (ok && tstep) mma_commit(&ctl->pacc);
    }
    if (!ok) fail_timeout(ctl, meta);
    mma_commit(&ctl->done);
    mbar_wait(&ctl->done, 0, abort, WAIT_NS / 4);
  } else if (warp >= 2) {
    // ---------------- epilogue: 8 warps; TMEM lane quarter q = warp & 3
    const int q = warp & 3, half = (warp - 2) >> 2;
    const uint32_t lanes = (uint32_t)(q * 32) << 16;
    bool ok = true;
    for (int step = 0; step < 4 && ok; ++step) {
      if ((step & 1) == 0) {
        // C^T (step 1) or C2^T (step 3) of M-tile `half`: thread = column kc of C.
        if (half < MH) {
          ok = __all_sync(~0u, mbar_wait(&ctl->pacc, step >> 1, abort, WAIT_NS));
          if (!ok) break;
          fence_after_sync();
          const int kc = half * 128 + q * 32 + lane;
          const bool keep = kc < k_old;
          uint8_t *col = sC + (kc / 64) * 8192 + (kc & 7) * 2;
          const int ck = (kc & 63) >> 3;
          for (int c = 0; c < PROJ_B; c += 16) {
            float v[16];
            tmem_ld16(tmem + lanes + half * PROJ_B + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const int i = c + u;
              const float x = keep ? v[u] : 0.f;
              if (step == 0) Cw[(size_t)i * R + kc] = x;
              *reinterpret_cast<__nv_bfloat16 *>(col + i * 128 + ((ck ^ (i & 7)) << 4)) =
                  __float2bfloat16_rn(x);
            }
          }
          fence_proxy_async_smem();
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->c_ready);
      } else {
        // Steps 2 and 4: d-tiles half, half + 2, ...: thread = row dr of B (column of E).
        for (int t = half; t < NT; t += 2) {
          ok = __all_sync(~0u, mbar_wait(&ctl->tacc[t], step >> 1, abort, WAIT_NS));
          if (!ok) break;
          fence_after_sync();
          const int dr = t * 128 + q * 32 + lane;
          // All 64 global loads of the column are issued before any use (one latency per tile).
          float x[PROJ_B];
          if (step == 1) {
#pragma unroll
            for (int i = 0; i < PROJ_B; ++i) x[i] = __bfloat162float(Fr[(size_t)i * D + dr]);
          } else {
#pragma unroll
            for (int i = 0; i < PROJ_B; ++i) x[i] = Ew[(size_t)i * D + dr];
          }
#pragma unroll
          for (int c = 0; c < PROJ_B; c += 16) {
            float v[16];
            tmem_ld16(tmem + lanes + t * PROJ_B + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const size_t at = (size_t)(c + u) * D + dr;
              const float e = x[c + u] - v[u];
              Ew[at] = e;
              if (step == 1) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(e);
                E1w[at] = hi;
                E1w[(size_t)PROJ_B * D + at] = __float2bfloat16_rn(e - __bfloat162float(hi));
              }
            }
          }
        }
        if (!ok) break;
        if (step == 1) {
          // E1 is read back by the tensor-memory-access unit (the async proxy) in step 3.
          fence_proxy_async_global();
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->e1_ready);
        }
      }
    }
    if (!ok) fail_timeout(ctl, meta);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

// ================================================================================================
// Reconstruction. Job fields: mapA (U), mapB (sigma-scaled basis, d x r bf16), out, pos, meta.
//
// Basis-stationary schedule. Each CTA owns `hp` heads (two when the head count is even) and keeps
// their rows of sigma*B^T resident in shared memory while it streams U through a ring of 16 KB
// K-slabs (128 rows x 64 coordinates). The n_heads/hp CTAs that own the other heads of the same
// rows form a group and walk the same row tiles in step, so each U tile is read from HBM once and
// served from L2 to the rest of the group. One MMA of N = hp x 128 covers all of the CTA's heads,
// so the tensor core reads each A slab once per K step.
//
// Output rows go to their positions pos_i. Each epilogue warp holds 32 rows and 32 RoPE pairs
// (columns j and j + 64) of a head; it stages them in shared memory as two 32-column boxes in the
// 64-byte swizzled layout (bank-conflict-free writes) and, when the 32 rows' positions are
// consecutive -- rows stored in position order, the usual case -- writes them with two TMA tile
// stores of its own (no barrier with the warp that holds the other columns). Groups with gaps or
// invalid rows are written from registers. Tensor memory is released as soon as the unit's last
// accumulators are in registers, before the staging.
constexpr int REC_MAX_STAGES = 8;
// Epilogue warps: two per TMEM lane quarter, 32 RoPE pairs each. (Sixteen warps with 16 pairs
// each and 32-byte tile stores measured slower.)
constexpr int REC_EPW = 8;
constexpr int REC_THREADS = 64 + 32 * REC_EPW;
constexpr int REC_STG_BYTES = 2 * TC_M * 128;  // lo and hi column halves of one head

// RoPE tables (head_dim 128, 64 frequencies omega_j = theta^(-2j/128)). Angles are reduced in
// exact integer arithmetic: W_j = omega_j / (2 pi) is held as a 0.64 fixed-point fraction
// (wh, wl), and for a position p < 2^31 the top 32 bits of frac(p W_j) are
// p * wh + umulhi(p, wl) (mod 2^32) -- the signed turn count in [-1/2, 1/2) at resolution
// 2^-32, with error below 2^-22 turns from W_j's float64 rounding. The angle in [-pi, pi) then goes
// to the hardware sine/cosine (absolute error ~1e-6 there, far below the bf16 output's rounding).
struct RopeTab {
  uint32_t wh[64], wl[64];
};

// Host-side table for rope_theta (float64 arithmetic; the kernel only copies it).
RopeTab make_rope_tab(double theta) {
  RopeTab t;
  const double two_pi = 6.283185307179586476925286766559;
  for (int j = 0; j < 64; ++j) {
    const double w = std::exp(-2.0 * j / 128.0 * std::log(theta)) / two_pi;  // turns per position
    const double hi = std::floor(std::ldexp(w, 32));
    t.wh[j] = (uint32_t)hi;
    t.wl[j] = (uint32_t)std::floor(std::ldexp(std::ldexp(w, 32) - hi, 32));
  }
  return t;
}

ISKV_DEV void rope_angle(const RopeTab *t, int j, uint32_t p, float &c, float &s) {
  const uint32_t top = p * t->wh[j] + __umulhi(p, t->wl[j]);
  const float ang = (float)(int32_t)top * 1.46291807926715968e-09f;  // 2 pi / 2^32
  __sincosf(ang, &s, &c);
}

struct RecCtl {
  uint64_t a_full[REC_MAX_STAGES], a_empty[REC_MAX_STAGES];
  uint64_t b_full, b_empty;
  uint64_t acc_full[2], acc_empty[2];
  uint64_t done;
  uint32_t tmem;
  int abort;
};

// Reconstruction: rows U (sigma B)^T, RoPE'd at their positions, written to out[pos].
__global__ void __launch_bounds__(REC_THREADS, 1) k_rec_tc(const TcJob *jobs, TcParams p,
                                                      const __grid_constant__ RopeTab rt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int R = p.r, KS = R / 64, D = p.d, HP = p.hp, NA = p.stages;
  constexpr int HN = 128;                        // columns per head
  uint8_t *sB = smem;                            // KS slabs x (HP x 128 rows) x 128 B, resident
  uint8_t *sA = sB + KS * HP * SLAB_BYTES;       // NA slabs x 16 KB
  uint8_t *sStg = sA + NA * SLAB_BYTES;          // 2 x (128 rows x 128 B), SW128
  RecCtl *ctl = reinterpret_cast<RecCtl *>(sStg + REC_STG_BYTES);
  RopeTab *rope_tab = reinterpret_cast<RopeTab *>(ctl + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Epilogue warps: WPQ per TMEM lane quarter, each holding NP of a head's 64 RoPE pairs.
  constexpr int EPW = REC_EPW, WPQ = EPW / 4, NP = 64 / WPQ;
  const int NN = HP * HN;                        // MMA N
  const uint32_t ncols = HP == 2 ? 512 : 256;    // two accumulator buffers of NN columns
  const uint32_t idesc = idesc_bf16_f32(TC_M, NN);
  // Group and member: CTAs g*G .. g*G+G-1 cover the heads of the same row tiles.
  const int G = p.n_heads / HP, group = blockIdx.x / G, member = blockIdx.x % G;
  const int ngroups = gridDim.x / G;
  const int total = p.count * p.tiles_per_job;
  const int per = (total + ngroups - 1) / ngroups;
  const int t_begin = group * per, t_end = min(total, t_begin + per);
  const int tpj = p.tiles_per_job;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) {
      mbar_init(&ctl->a_full[i], 1);
      mbar_init(&ctl->a_empty[i], 1);
    }
    mbar_init(&ctl->b_full, 1);
    mbar_init(&ctl->b_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->acc_full[i], 1);
      mbar_init(&ctl->acc_empty[i], EPW);
    }
    mbar_init(&ctl->done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 64) {
    rope_tab->wh[threadIdx.x] = rt.wh[threadIdx.x];
    rope_tab->wl[threadIdx.x] = rt.wl[threadIdx.x];
  }
  if (warp == 1) tmem_alloc(&ctl->tmem, ncols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int *abort = &ctl->abort;
  // Per-thread cache of the current history's row count: every role tests every tile, and the
  // count changes only with the history, so it is read from global memory once per history.
  int cache_j = -1;
  int64_t cache_n = 0;
  auto rows_of = [&](int j) -> int64_t {
    if (j != cache_j) {
      cache_j = j;
      cache_n = jobs[j].meta[ISKV_META_N];
    }
    return cache_n;
  };
  // Tile cursor: linear tile t = j * tpj + k (history j, row tile k). Every role walks the same
  // sequence of valid tiles (rows below the history's current length, a prefix of its tiles),
  // advancing incrementally so that no division sits on a unit's critical path.
  struct Cur {
    int t, j, k;
  };
  auto seek = [&](Cur c) -> Cur {  // first valid tile at or after c; t = -1 when none is left
    while (c.t < t_end) {
      if (c.k * TC_M < rows_of(c.j)) return c;
      c.t += tpj - c.k;  // the rest of this history is past its length
      ++c.j;
      c.k = 0;
    }
    c.t = -1;
    return c;
  };
  auto advance = [&](Cur c) -> Cur {
    ++c.t;
    if (++c.k == tpj) {
      c.k = 0;
      ++c.j;
    }
    return seek(c);
  };
  Cur c_first;
  c_first.t = t_begin;
  c_first.j = t_begin / tpj;
  c_first.k = t_begin - c_first.j * tpj;
  c_first = seek(c_first);

  if (warp == 0 && lane == 0) {
    // ---------------- producer: basis rows of this CTA's heads once per history, U slabs per tile
    int na = 0, nb = 0, cur = -1;
    RingPos rp;
    int64_t *fm = nullptr;  // meta of the history being loaded: where a timeout is recorded
    bool ok = true;
    for (Cur c = c_first; c.t >= 0 && ok && !*abort; c = advance(c)) {
      const int j = c.j, row0 = c.k * TC_M;
      const TcJob &jb = jobs[j];
      fm = jb.meta;
      if (j != cur) {
        if (nb > 0 && !mbar_wait(&ctl->b_empty, (nb - 1) & 1, abort, WAIT_NS)) { ok = false; break; }
        tensormap_acquire(&jb.mapA);
        tensormap_acquire(&jb.mapB);
        mbar_arrive_expect_tx(&ctl->b_full, KS * HP * SLAB_BYTES);
        for (int s = 0; s < KS; ++s)
          for (int h = 0; h < HP; ++h)
            tma_load_2d(sB + (s * HP + h) * SLAB_BYTES, &jb.mapB, s * 64, (member * HP + h) * HN,
                        &ctl->b_full);
        cur = j;
        ++nb;
      }
      for (int s = 0; s < KS; ++s) {
        // The slot's previous use (one lap back) must have been consumed.
        if (na >= NA && !mbar_wait(&ctl->a_empty[rp.slot], rp.phase ^ 1u, abort, WAIT_NS)) { ok = false; break; }
        mbar_arrive_expect_tx(&ctl->a_full[rp.slot], SLAB_BYTES);
        tma_load_2d(sA + rp.slot * SLAB_BYTES, &jb.mapA, s * 64, row0, &ctl->a_full[rp.slot]);
        rp.next(NA);
        ++na;
      }
    }
    if (!ok) fail_timeout(ctl, fm);
    // Let every copy issued land before the CTA exits.
    if (nb > 0) mbar_wait(&ctl->b_full, (nb - 1) & 1, abort, WAIT_NS / 4);
    for (int k = 1; k <= NA && na - k >= 0; ++k)
      mbar_wait(&ctl->a_full[(na - k) % NA], ((na - k) / NA) & 1, abort, WAIT_NS / 4);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int nb = 0, nc = 0, cur = -1;
    int64_t *fm = nullptr;
    bool ok = true;
    RingPos rp;
    const uint64_t da0 = sw128_desc(smem_u32(sA)), db0 = sw128_desc(smem_u32(sB));
    for (Cur c = c_first; c.t >= 0 && ok && !*abort; c = advance(c)) {
      const int j = c.j;
      fm = jobs[j].meta;
      if (j != cur) {
        // The resident basis may be replaced once every MMA reading it has completed.
        if (nb > 0) mma_commit(&ctl->b_empty);
        if (!mbar_wait(&ctl->b_full, nb & 1, abort, WAIT_NS)) { ok = false; break; }
        cur = j;
        ++nb;
      }
      const int buf = nc & 1, use = nc >> 1;
      if (use > 0 && !mbar_wait(&ctl->acc_empty[buf], (use - 1) & 1, abort, WAIT_NS)) { ok = false; break; }
      fence_after_sync();
      const uint32_t d0 = tmem + buf * NN;
      for (int s = 0; s < KS; ++s) {
        if (!mbar_wait(&ctl->a_full[rp.slot], rp.phase, abort, WAIT_NS)) { ok = false; break; }
        fence_after_sync();
        const uint64_t da = desc_add(da0, rp.slot * SLAB_BYTES);
        const uint64_t db = desc_add(db0, s * HP * SLAB_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(d0, desc_add(da, kk * 32), desc_add(db, kk * 32), idesc, (s | kk) != 0);
        mma_commit(&ctl->a_empty[rp.slot]);
        rp.next(NA);
      }
      if (!ok) break;
      mma_commit(&ctl->acc_full[buf]);
      ++nc;
    }
    if (!ok) fail_timeout(ctl, fm);
    mma_commit(&ctl->done);
    mbar_wait(&ctl->done, 0, abort, WAIT_NS / 4);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> RoPE -> bf16 -> staged rows -> bulk copies to out[pos]
    const int q = warp & 3, half = (warp - 2) >> 2;
    const int j0 = half * NP;  // this thread's head-local pairs j0 .. j0 + NP - 1 (cols j, j + 64)
    const int srow = q * 32 + lane;
    // This warp's staged rows (reconstruction): its 32 rows x NP columns of the lo half and of the
    // hi half, each a box of 2 NP-byte rows in the matching swizzled layout; lane 0 issues the
    // warp's tile stores.
    uint8_t *stg = sStg + (warp - 2) * (2 * 32 * NP * 2);
    const bool issuer = lane == 0;
    bool pending = false;  // a tile store of this warp may still be reading the staged rows
    int nc = 0;
    // The warps that share rows (the WPQ warps of lane quarter q) take every decision together
    // through an AND-reducing named barrier, and tcgen05.ld is warp-wide.
    const int pair_bar = 1 + q;
    constexpr int PB = 32 * WPQ;  // threads at the quarter's barrier
    float cs[NP], sn[NP];
    // Fields of the history being written, read from global memory once per history rather than
    // once per unit (each read is a dependent global load on the unit's critical path).
    int hj = -1;
    const int32_t *h_pos = nullptr;
    __nv_bfloat16 *h_out = nullptr;
    int64_t h_rows = 0, h_total = 0;
    bool h_rope = false, h_tiles = false;
    auto hist = [&](int j) {
      if (j != hj) {
        hj = j;
        const TcJob &jb = jobs[j];
        h_pos = jb.pos;
        h_out = static_cast<__nv_bfloat16 *>(jb.out);
        h_rows = rows_of(j);
        h_total = jb.n_total;
        h_rope = jb.rope != 0;
        h_tiles = jb.tiles_ok != 0;
      }
    };
    // Position of this thread's row in a unit, loaded one unit ahead. The raw 32-bit value is
    // carried to the next unit unconverted, so nothing waits on the load until then.
    auto row_pos = [&](const Cur &c) -> int32_t {
      if (c.t < 0) return 0;
      hist(c.j);
      const int64_t row = (int64_t)c.k * TC_M + srow;
      return row < h_rows ? __ldg(h_pos + row) : 0;
    };
    int acq_j = -1;  // history whose output tensor map this thread last acquired
    Cur c = c_first;
    int32_t ps_next = row_pos(c);
    for (;;) {
      if (!named_and(pair_bar, PB, c.t >= 0 && !*abort)) break;
      const int jj = c.j;
      const int32_t ps_raw = ps_next;
      hist(jj);
      bool valid = c.k * TC_M + srow < h_rows;
      const bool rope = h_rope, tiles_ok = h_tiles;
      __nv_bfloat16 *const out = h_out;
      const int64_t n_total = h_total;
      const Cur cn = advance(c);
      ps_next = row_pos(cn);  // consumed by the next unit: its latency hides behind this one
      const int64_t ps = valid ? (int64_t)ps_raw : 0;
      if (valid && (ps < 0 || ps >= n_total)) {
        record_status(jobs[jj].meta, ISKV_ERR_SHAPE);
        valid = false;
      }
      if (rope && valid) {
#pragma unroll
        for (int i = 0; i < NP; ++i) rope_angle(rope_tab, j0 + i, (uint32_t)ps, cs[i], sn[i]);
      }
      __nv_bfloat16 *orow = out + (size_t)(valid ? ps : 0) * D + (size_t)member * HP * HN;
      // This lane quarter's 32 rows go out as tiles when their positions are consecutive (the
      // same answer in both warps of the pair: they hold the same rows).
      const int64_t first = __shfl_sync(~0u, ps, 0);
      const bool tiles = tiles_ok && __all_sync(~0u, valid && ps == first + lane);
      const TcJob &jb = jobs[jj];
      if (tiles && issuer && acq_j != jj) {
        tensormap_acquire(&jb.mapO);
        acq_j = jj;
      }
      const int buf = nc & 1, use = nc >> 1;
      if (!named_and(pair_bar, PB, mbar_wait(&ctl->acc_full[buf], use & 1, abort, WAIT_NS))) {
        fail_timeout(ctl, jb.meta);
        break;
      }
      fence_after_sync();
      const uint32_t base = tmem + buf * NN + ((uint32_t)(q * 32) << 16);
      for (int h = 0; h < HP; ++h) {
        // The head's 32 RoPE pairs go to packed registers first, so the TMEM loads and the math
        // overlap the previous tile stores still reading the staged rows.
        uint32_t wl[NP / 2], wh[NP / 2];
#pragma unroll
        for (int jb16 = 0; jb16 < NP; jb16 += 16) {
          float lo[16], hi[16];
          tmem_ld16(base + h * HN + j0 + jb16, lo);
          tmem_ld16(base + h * HN + 64 + j0 + jb16, hi);
          tmem_ld_wait();
          if (rope) {
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              const float c0 = cs[jb16 + i], s0 = sn[jb16 + i];
              const float c1 = cs[jb16 + i + 1], s1 = sn[jb16 + i + 1];
              wl[(jb16 + i) / 2] =
                  pack_bf16(lo[i] * c0 - hi[i] * s0, lo[i + 1] * c1 - hi[i + 1] * s1);
              wh[(jb16 + i) / 2] =
                  pack_bf16(hi[i] * c0 + lo[i] * s0, hi[i + 1] * c1 + lo[i + 1] * s1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              wl[(jb16 + i) / 2] = pack_bf16(lo[i], lo[i + 1]);
              wh[(jb16 + i) / 2] = pack_bf16(hi[i], hi[i + 1]);
            }
          }
        }
        if (h == HP - 1) {
          // Every accumulator of the unit is in registers: tensor memory can take the next unit
          // while this warp stages and stores.
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->acc_empty[buf]);
        }
        if (tiles) {
          // The staged rows are free once this warp's previous tile stores have read them.
          if (pending) {
            if (issuer) bulk_wait_read0();
            __syncwarp();
          }
          // Row = lane, 64-byte staged rows: 16-byte chunk u sits at chunk u ^ ((row >> 1) & 3)
          // (the 64-byte swizzle: address bits 7-8 into bits 4-5).
          static_assert(NP == 32, "staging is laid out for 32 pairs per warp");
          const int sw = (lane >> 1) & 3;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            *reinterpret_cast<uint4 *>(stg + lane * 64 + 16 * (u ^ sw)) =
                make_uint4(wl[4 * u], wl[4 * u + 1], wl[4 * u + 2], wl[4 * u + 3]);
            *reinterpret_cast<uint4 *>(stg + 2048 + lane * 64 + 16 * (u ^ sw)) =
                make_uint4(wh[4 * u], wh[4 * u + 1], wh[4 * u + 2], wh[4 * u + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (issuer) {
            const int x = (member * HP + h) * HN + j0;
            tma_store_2d(&jb.mapO, x, (int)first, stg);
            tma_store_2d(&jb.mapO, x + 64, (int)first, stg + 2048);
            bulk_commit();
          }
          pending = true;
        } else if (valid) {
          uint4 *dl = reinterpret_cast<uint4 *>(orow + h * HN + j0);
          uint4 *dh = reinterpret_cast<uint4 *>(orow + h * HN + 64 + j0);
#pragma unroll
          for (int u = 0; u < NP / 8; ++u) {
            dl[u] = make_uint4(wl[4 * u], wl[4 * u + 1], wl[4 * u + 2], wl[4 * u + 3]);
            dh[u] = make_uint4(wh[4 * u], wh[4 * u + 1], wh[4 * u + 2], wh[4 * u + 3]);
          }
        }
      }
      ++nc;
      c = cn;
    }
    if (issuer && pending) bulk_wait0();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

// ================================================================================================
// Decode-attention scores of compressed keys on the tensor cores (bf16 factors, head_dim 128).
// A first MMA per 128-row tile forms the keys of the CTA's heads, U (sigma B_h)^T, in tensor
// memory, as in the reconstruction. The epilogue applies RoPE at each row's position and writes
// the rotated keys back into the same tensor memory as bf16, pair j of a head as one 32-bit
// column (rotated low component, rotated high component). A second MMA with A in tensor memory
// contracts them with the head's query group: B = [q_hi; q_lo], N = 16 rows of bf16, the queries
// split into a bf16 head and a bf16 remainder, so the queries enter with about 16 significant bits
// and the keys with the bf16 rounding of a reconstructed bf16 cache. Only the scores
// S[query head][pos] leave the SM.
struct ScoCtl {
  uint64_t a_full[REC_MAX_STAGES], a_empty[REC_MAX_STAGES];
  uint64_t b_full, b_empty;
  uint64_t acc_full[2], acc_empty[2];
  uint64_t kst_full[2], s_full[2];  // rotated keys written back / query contraction done
  uint64_t done;
  uint32_t tmem;
  int abort;
};
constexpr int SCO_EPW = 8;                     // epilogue warps, two per TMEM lane quarter
constexpr int SCO_THREADS = 64 + 32 * SCO_EPW;
constexpr int SCO_QN = 16;                     // MMA N of the query contraction
constexpr int SCO_Q_BYTES = 2 * SCO_QN * 128;  // one head's query operand: two 64-wide K slabs

// Resident basis rows for hp heads, the U slab ring, the query operands, the warps' base angles,
// barriers, RoPE table.
size_t tc_sco_smem(int r, int hp, int stages) {
  return 1024 + (size_t)hp * (r / 64) * SLAB_BYTES + (size_t)stages * SLAB_BYTES +
         (size_t)hp * SCO_Q_BYTES + SCO_EPW * 32 * sizeof(float2) + sizeof(ScoCtl) +
         sizeof(RopeTab);
}

template <int QPK>
__global__ void __launch_bounds__(SCO_THREADS, 1) k_scores_tc(const TcJob *jobs, TcParams p,
                                                          const __grid_constant__ RopeTab rt) {
  static_assert(2 * QPK <= SCO_QN, "query group wider than the contraction");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int R = p.r, KS = R / 64, HP = p.hp, NA = p.stages;
  constexpr int HN = 128;                   // columns per head
  uint8_t *sB = smem;                       // KS slabs x (HP x 128 rows) x 128 B, resident
  uint8_t *sA = sB + KS * HP * SLAB_BYTES;  // NA slabs x 16 KB
  uint8_t *sQ = sA + NA * SLAB_BYTES;       // HP x [2 K slabs][16 rows][128 B], SW128
  float2 *sBase = reinterpret_cast<float2 *>(sQ + HP * SCO_Q_BYTES);  // per epilogue warp: 32
  ScoCtl *ctl = reinterpret_cast<ScoCtl *>(sBase + SCO_EPW * 32);
  RopeTab *rope_tab = reinterpret_cast<RopeTab *>(ctl + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NN = HP * HN;                      // MMA N of the keys
  const uint32_t ncols = HP == 2 ? 512 : 256;  // two accumulator buffers of NN columns
  const uint32_t idesc = idesc_bf16_f32(TC_M, NN);
  const uint32_t idesc_q = idesc_bf16_f32(TC_M, SCO_QN);
  const int G = p.n_heads / HP, group = blockIdx.x / G, member = blockIdx.x % G;
  const int ngroups = gridDim.x / G;
  const int total = p.count * p.tiles_per_job;
  const int per = (total + ngroups - 1) / ngroups;
  const int t_begin = group * per, t_end = min(total, t_begin + per);
  const int tpj = p.tiles_per_job;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) {
      mbar_init(&ctl->a_full[i], 1);
      mbar_init(&ctl->a_empty[i], 1);
    }
    mbar_init(&ctl->b_full, 1);
    mbar_init(&ctl->b_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->acc_full[i], 1);
      mbar_init(&ctl->acc_empty[i], SCO_EPW);
      mbar_init(&ctl->kst_full[i], SCO_EPW);
      mbar_init(&ctl->s_full[i], 1);
    }
    mbar_init(&ctl->done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 64) {
    rope_tab->wh[threadIdx.x] = rt.wh[threadIdx.x];
    rope_tab->wl[threadIdx.x] = rt.wl[threadIdx.x];
  }
  if (warp == 1) tmem_alloc(&ctl->tmem, ncols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int *abort = &ctl->abort;
  // Tile walk: linear tile t = j * tpj + k (history j, row tile k); every role visits the same
  // valid tiles (a prefix of each history's tiles, below its current length) in the same order.
  int cache_j = -1;
  int64_t cache_n = 0;
  auto rows_of = [&](int j) -> int64_t {
    if (j != cache_j) {
      cache_j = j;
      cache_n = jobs[j].meta[ISKV_META_N];
    }
    return cache_n;
  };
  struct Cur {
    int t, j, k;
  };
  auto seek = [&](Cur c) -> Cur {
    while (c.t < t_end) {
      if (c.k * TC_M < rows_of(c.j)) return c;
      c.t += tpj - c.k;
      ++c.j;
      c.k = 0;
    }
    c.t = -1;
    return c;
  };
  auto advance = [&](Cur c) -> Cur {
    ++c.t;
    if (++c.k == tpj) {
      c.k = 0;
      ++c.j;
    }
    return seek(c);
  };
  Cur c_first;
  c_first.t = t_begin;
  c_first.j = t_begin / tpj;
  c_first.k = t_begin - c_first.j * tpj;
  c_first = seek(c_first);

  if (warp == 0 && lane == 0) {
    // ---------------- producer: basis rows of this CTA's heads once per history, U slabs per tile
    int na = 0, nb = 0, cur = -1;
    RingPos rp;
    int64_t *fm = nullptr;
    bool ok = true;
    for (Cur c = c_first; c.t >= 0 && ok && !*abort; c = advance(c)) {
      const int j = c.j, row0 = c.k * TC_M;
      const TcJob &jb = jobs[j];
      fm = jb.meta;
      if (j != cur) {
        if (nb > 0 && !mbar_wait(&ctl->b_empty, (nb - 1) & 1, abort, WAIT_NS)) { ok = false; break; }
        tensormap_acquire(&jb.mapA);
        tensormap_acquire(&jb.mapB);
        mbar_arrive_expect_tx(&ctl->b_full, KS * HP * SLAB_BYTES);
        for (int s = 0; s < KS; ++s)
          for (int h = 0; h < HP; ++h)
            tma_load_2d(sB + (s * HP + h) * SLAB_BYTES, &jb.mapB, s * 64, (member * HP + h) * HN,
                        &ctl->b_full);
        cur = j;
        ++nb;
      }
      for (int s = 0; s < KS; ++s) {
        // The slot's previous use (one lap back) must have been consumed.
        if (na >= NA && !mbar_wait(&ctl->a_empty[rp.slot], rp.phase ^ 1u, abort, WAIT_NS)) { ok = false; break; }
        mbar_arrive_expect_tx(&ctl->a_full[rp.slot], SLAB_BYTES);
        tma_load_2d(sA + rp.slot * SLAB_BYTES, &jb.mapA, s * 64, row0, &ctl->a_full[rp.slot]);
        rp.next(NA);
        ++na;
      }
    }
    if (!ok) fail_timeout(ctl, fm);
    if (nb > 0) mbar_wait(&ctl->b_full, (nb - 1) & 1, abort, WAIT_NS / 4);
    for (int k = 1; k <= NA && na - k >= 0; ++k)
      mbar_wait(&ctl->a_full[(na - k) % NA], ((na - k) / NA) & 1, abort, WAIT_NS / 4);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: the keys of tile t, then the query contraction of tile t - 1
    // (whose rotated keys the epilogue writes back while the tensor core forms tile t's keys).
    int nb = 0, nc = 0, cur = -1;
    int64_t *fm = nullptr;
    bool ok = true;
    int pbuf = -1, puse = 0;
    RingPos rp;
    const uint64_t da0 = sw128_desc(smem_u32(sA)), db0 = sw128_desc(smem_u32(sB));
    const uint64_t dq0 = sw128_desc(smem_u32(sQ));
    auto contract = [&](int buf, int use) -> bool {
      if (!mbar_wait(&ctl->kst_full[buf], use & 1, abort, WAIT_NS)) return false;
      fence_after_sync();
      for (int h = 0; h < HP; ++h) {
        const uint32_t a = tmem + buf * NN + h * HN;  // rotated keys: 64 columns, K = 128
        const uint64_t dq = desc_add(dq0, h * SCO_Q_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(a + 64, a + kk * 8,
                      desc_add(dq, (kk >> 2) * (SCO_QN * 128) + (kk & 3) * 32), idesc_q, kk != 0);
      }
      mma_commit(&ctl->s_full[buf]);
      return true;
    };
    for (Cur c = c_first; c.t >= 0 && ok && !*abort; c = advance(c)) {
      const int j = c.j;
      fm = jobs[j].meta;
      if (j != cur) {
        if (nb > 0) mma_commit(&ctl->b_empty);
        if (!mbar_wait(&ctl->b_full, nb & 1, abort, WAIT_NS)) { ok = false; break; }
        cur = j;
        ++nb;
      }
      const int buf = nc & 1, use = nc >> 1;
      if (use > 0 && !mbar_wait(&ctl->acc_empty[buf], (use - 1) & 1, abort, WAIT_NS)) { ok = false; break; }
      fence_after_sync();
      const uint32_t d0 = tmem + buf * NN;
      for (int s = 0; s < KS; ++s) {
        if (!mbar_wait(&ctl->a_full[rp.slot], rp.phase, abort, WAIT_NS)) { ok = false; break; }
        fence_after_sync();
        const uint64_t da = desc_add(da0, rp.slot * SLAB_BYTES);
        const uint64_t db = desc_add(db0, s * HP * SLAB_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(d0, desc_add(da, kk * 32), desc_add(db, kk * 32), idesc, (s | kk) != 0);
        mma_commit(&ctl->a_empty[rp.slot]);
        rp.next(NA);
      }
      if (!ok) break;
      mma_commit(&ctl->acc_full[buf]);
      if (pbuf >= 0 && !contract(pbuf, puse)) { ok = false; break; }
      pbuf = buf;
      puse = use;
      ++nc;
    }
    if (ok && pbuf >= 0 && !*abort && !contract(pbuf, puse)) ok = false;
    if (!ok) fail_timeout(ctl, fm);
    mma_commit(&ctl->done);
    mbar_wait(&ctl->done, 0, abort, WAIT_NS / 4);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM keys -> RoPE -> bf16 keys back to TMEM; scores -> S
    const int q = warp & 3, half = (warp - 2) >> 2;
    const int j0 = half * 32;  // this warp's pairs j0 .. j0 + 31 of every head (cols j, j + 64)
    const int srow = q * 32 + lane;
    const int et = threadIdx.x - 64;
    // RoPE by angle addition where a warp's 32 rows sit at consecutive positions p0 + lane: the
    // rotation by lane omega_j is fixed per thread (computed once), the one by p0 omega_j is
    // shared by the warp (one angle per lane, exchanged through shared memory). Both angles are
    // reduced exactly in fixed point; the product adds float32 rounding only.
    float oc[32], os[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) rope_angle(rope_tab, j0 + i, (uint32_t)lane, oc[i], os[i]);
    float2 *wbase = sBase + (warp - 2) * 32;
    int hj = -1;
    const int32_t *h_pos = nullptr;
    float *h_S = nullptr;
    float h_scale = 0.f;
    int64_t h_rows = 0, h_total = 0;
    bool h_rope = false;
    auto hist = [&](int j) {
      if (j != hj) {
        hj = j;
        const TcJob &jb = jobs[j];
        h_pos = jb.pos;
        h_S = jb.S;
        h_scale = jb.scale;
        h_rows = rows_of(j);
        h_total = jb.n_total;
        h_rope = jb.rope != 0;
      }
    };
    auto row_pos = [&](const Cur &c) -> int32_t {
      if (c.t < 0) return 0;
      hist(c.j);
      const int64_t row = (int64_t)c.k * TC_M + srow;
      return row < h_rows ? __ldg(h_pos + row) : 0;
    };
    int q_job = -1;
    int nc = 0;
    Cur c = c_first;
    int32_t ps_next = row_pos(c);
    // The tile about to be staged, prepared one step ahead (while the previous tile's query
    // contraction runs): its history, row validity and position, rotation mode, where its scores
    // go, and (mode 1) the warp's base angles in wbase. The history fields are copied here: the
    // position prefetch of the tile after it may move the cached fields to the next history.
    int jj = 0, mode = 0;
    bool valid = false;
    int64_t ps = 0, t_total = 0;
    float *t_S = nullptr;
    float t_scale = 0.f;
    Cur cn = c;
    auto prepare = [&]() {
      jj = c.j;
      const int32_t ps_raw = ps_next;
      hist(jj);
      valid = c.k * TC_M + srow < h_rows;
      t_S = h_S;
      t_total = h_total;
      t_scale = h_scale;
      const bool rope = h_rope;
      ps = valid ? (int64_t)ps_raw : 0;
      if (valid && (ps < 0 || ps >= t_total)) {
        record_status(jobs[jj].meta, ISKV_ERR_SHAPE);
        valid = false;
      }
      cn = advance(c);
      ps_next = row_pos(cn);
      // 0: no rotation, 1: consecutive positions (angle addition), 2: each row on its own.
      const int64_t p0 = __shfl_sync(~0u, ps, 0);
      mode = !rope ? 0 : __all_sync(~0u, valid && ps == p0 + lane) ? 1 : 2;
      if (mode == 1) {  // the last reads of wbase are behind this warp's last __syncwarp
        float c0, s0;
        rope_angle(rope_tab, j0 + lane, (uint32_t)p0, c0, s0);
        wbase[lane] = make_float2(c0, s0);
        __syncwarp();
      }
    };
    if (c.t >= 0) prepare();
    for (;;) {
      if (c.t < 0 || *abort) break;
      if (jj != q_job) {
        // The history's query operand. Row n < QPK: the bf16 head of query n of the CTA's head;
        // row QPK + n: its bf16 remainder; other rows zero. K index 2j + e holds component
        // j + 64 e (the column order of the rotated keys). Every contraction that read the
        // previous operand has completed: this thread waited for its scores.
        const float *qg = jobs[jj].q;
        for (int e = et; e < HP * SCO_QN * 64; e += 32 * SCO_EPW) {
          const int hh = e / (SCO_QN * 64), n = (e >> 6) % SCO_QN, j = e & 63;
          uint32_t w = 0;
          if (n < 2 * QPK) {
            const float *qr = qg + (size_t)((member * HP + hh) * QPK + n % QPK) * HN;
            float x0 = qr[j], x1 = qr[j + 64];
            if (n >= QPK) {
              x0 -= __bfloat162float(__float2bfloat16_rn(x0));
              x1 -= __bfloat162float(__float2bfloat16_rn(x1));
            }
            w = pack_bf16(x0, x1);
          }
          // K index 2j: K slab j / 32, byte 4 (j % 32) of the 128-byte row, whose 16-byte chunks
          // are swizzled by the row (the layout a 128-byte-swizzled TMA box has).
          const int chunk = (j & 31) >> 2;
          *reinterpret_cast<uint32_t *>(sQ + hh * SCO_Q_BYTES + (j >> 5) * (SCO_QN * 128) +
                                        n * 128 + ((chunk ^ (n & 7)) << 4) + 4 * (j & 3)) = w;
        }
        fence_proxy_async_smem();
        q_job = jj;
      }
      const int buf = nc & 1, use = nc >> 1;
      if (!mbar_wait(&ctl->acc_full[buf], use & 1, abort, WAIT_NS)) {
        fail_timeout(ctl, jobs[jj].meta);
        break;
      }
      fence_after_sync();
      const uint32_t base = tmem + buf * NN + ((uint32_t)(q * 32) << 16);
#pragma unroll
      for (int jb16 = 0; jb16 < 32; jb16 += 16) {
        float cs[16], sn[16];
        if (mode == 1) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 a = wbase[jb16 + i];
            cs[i] = a.x * oc[jb16 + i] - a.y * os[jb16 + i];
            sn[i] = a.y * oc[jb16 + i] + a.x * os[jb16 + i];
          }
        } else if (mode == 2 && valid) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            rope_angle(rope_tab, j0 + jb16 + i, (uint32_t)ps, cs[i], sn[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            cs[i] = 1.f;
            sn[i] = 0.f;
          }
        }
        for (int h = 0; h < HP; ++h) {
          float lo[16], hi[16];
          tmem_ld16(base + h * HN + j0 + jb16, lo);
          tmem_ld16(base + h * HN + 64 + j0 + jb16, hi);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16(lo[i] * cs[i] - hi[i] * sn[i], hi[i] * cs[i] + lo[i] * sn[i]);
          // Over this warp's own low-component columns, already read.
          tmem_st16(base + h * HN + j0 + jb16, w);
        }
      }
      tmem_st_wait();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->kst_full[buf]);
      // This tile's scores go where it was prepared to send them; the next tile is prepared
      // while its contraction runs.
      const int j_done = jj;
      float *const s_out = t_S;
      const int64_t s_total = t_total, s_ps = ps;
      const float s_scale = t_scale;
      const bool s_valid = valid;
      c = cn;
      if (c.t >= 0) prepare();
      if (!mbar_wait(&ctl->s_full[buf], use & 1, abort, WAIT_NS)) {
        fail_timeout(ctl, jobs[j_done].meta);
        break;
      }
      fence_after_sync();
      if (half < HP) {  // warp half h reads head h's scores: columns 64 .. 64 + 2 QPK
        float sc[16];
        tmem_ld16(base + half * HN + 64, sc);
        tmem_ld_wait();
        if (s_valid) {
#pragma unroll
          for (int g = 0; g < QPK; ++g)
            s_out[(size_t)((member * HP + half) * QPK + g) * s_total + s_ps] =
                s_scale * (sc[g] + sc[QPK + g]);
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->acc_empty[buf]);
      ++nc;
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

// ================================================================================================
// Gram matrices for the re-orthogonalisation: G = X^T X over the rows of X = U (n rows) or B (d
// rows). The contraction runs over rows, so both operands are read MN-major: a TMA box of 64 rows
// x 64 columns is one MN-major stack of 128-byte rows, slabs of 64 columns sit 8 KB apart. Each
// CTA reduces one split of up to GRAM_SPLIT rows into an r x r float32 partial (two M = 128,
// N = r accumulators in tensor memory); a second kernel sums the partials.
constexpr int GRAM_THREADS = 192;  // producer warp, MMA warp, 4 epilogue warps
constexpr int GRAM_STAGES = 4;
constexpr int GRAM_RING = 6;       // stages of the Gram kernel's ring
constexpr int GRAM_KT = 64;        // rows per pipeline stage

// Shared memory before the barriers: the stage ring, or the staged 128-row half of a partial
// (rows padded to r + 4 floats), whichever is larger.
__host__ __device__ inline int gram_area_bytes(int r) {
  const int ring = GRAM_RING * (r / 64) * GRAM_KT * 128, stg = 128 * (r + 4) * 4;
  return ring > stg ? ring : stg;
}

__global__ void __launch_bounds__(GRAM_THREADS, 1) k_gram_tc(const TcJob *jobs, GramParams p) {
  // The U chunks of every job come first (they are the long ones), then the B chunks.
  const int nU = p.count * p.nsu;
  int job, which, split;
  if ((int)blockIdx.x < nU) {
    job = blockIdx.x / p.nsu;
    which = 0;
    split = blockIdx.x % p.nsu;
  } else {
    const int b = blockIdx.x - nU;
    job = b / p.nsb;
    which = 1;
    split = b % p.nsb;
  }
  const TcJob &jb = jobs[job];
  const int32_t *sc = jb.sc;
  const int R = p.r, SL = R / 64, MH = R / 128, N = R;
  const int rows_total = which ? p.d : sc[FS_N_OLD];
  const int chunk = which ? p.split : gram_chunk(rows_total, p.nsu);
  const int r0 = split * chunk;
  const int nrows = min(chunk, rows_total - r0);
  if (sc[FS_SKIP] || nrows <= 0 || sc[FS_K_OLD] == 0) return;  // uniform over the CTA
  const int nk = (nrows + GRAM_KT - 1) / GRAM_KT;
  const CUtensorMap *map = which ? &jb.mapB : &jb.mapA;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int STAGE_BYTES = SL * GRAM_KT * 128;
  TcCtl *ctl = reinterpret_cast<TcCtl *>(smem + gram_area_bytes(R));
  uint64_t *full = reinterpret_cast<uint64_t *>(ctl + 1);   // [GRAM_RING]
  uint64_t *empty = full + GRAM_RING;                      // [GRAM_RING]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = MH * N <= 128 ? 128 : (MH * N <= 256 ? 256 : 512);
  const uint32_t idesc = idesc_bf16_f32_mn(128, N);
  if (threadIdx.x == 0) {
    for (int i = 0; i < GRAM_RING; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(&ctl->acc_full[0], 1);
    mbar_init(&ctl->done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&ctl->tmem, ncols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int *abort = &ctl->abort;

  if (warp == 0 && lane == 0) {
    tensormap_acquire(map);
    for (int kt = 0; kt < nk && !*abort; ++kt) {
      const int st = kt % GRAM_RING, use = kt / GRAM_RING;
      if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, abort, WAIT_NS)) {
        fail_timeout(ctl, jb.meta);
        break;
      }
      mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
      for (int sl = 0; sl < SL; ++sl)
        tma_load_2d(smem + st * STAGE_BYTES + sl * GRAM_KT * 128, map, sl * 64, r0 + kt * GRAM_KT,
                    &full[st]);
    }
    for (int k = 1; k <= GRAM_RING && nk - k >= 0; ++k)
      mbar_wait(&full[(nk - k) % GRAM_RING], ((nk - k) / GRAM_RING) & 1, abort, WAIT_NS / 4);
  } else if (warp == 1 && lane == 0) {
    bool ok = true;
    for (int kt = 0; kt < nk && ok && !*abort; ++kt) {
      const int st = kt % GRAM_RING, use = kt / GRAM_RING;
      if (!mbar_wait(&full[st], use & 1, abort, WAIT_NS)) { ok = false; break; }
      fence_after_sync();
      const uint32_t base = smem_u32(smem + st * STAGE_BYTES);
#pragma unroll
      for (int kk = 0; kk < GRAM_KT / 16; ++kk) {
        const uint64_t bdesc = sw128_mn_desc(base + kk * 2048, GRAM_KT * 128);
        for (int h = 0; h < MH; ++h) {
          const uint64_t adesc = sw128_mn_desc(base + h * 2 * GRAM_KT * 128 + kk * 2048, GRAM_KT * 128);
          mma_bf16(tmem + h * N, adesc, bdesc, idesc, (kt | kk) != 0);
        }
      }
      mma_commit(&empty[st]);
    }
    if (!ok) fail_timeout(ctl, jb.meta);
    mma_commit(&ctl->acc_full[0]);
    mma_commit(&ctl->done);
    mbar_wait(&ctl->done, 0, abort, WAIT_NS / 4);
  } else if (warp >= 2) {
    const int q = warp & 3;
    // A job's single B chunk writes its Gram matrix itself; U chunks write partials.
    float *out = reinterpret_cast<float *>(jb.out) +
                 (which ? (p.nsb == 1 ? p.off_g1 : p.off_gb) : p.off_gu) / sizeof(float) +
                 (size_t)split * R * R;
    // Once the accumulators are complete, the stage buffers are idle: each 128-row half of the
    // partial is staged there (rows of R + 4 floats, so that the 32 rows a warp writes at once
    // fall in distinct banks) and leaves in whole coalesced rows.
    float *stg = reinterpret_cast<float *>(smem);
    const int LDS = R + 4;
    // One decision per warp: tcgen05.ld is a warp-wide instruction; the four epilogue warps meet
    // at named barrier 1 whatever they decided.
    const bool ok = __all_sync(~0u, mbar_wait(&ctl->acc_full[0], 0, abort, WAIT_NS) && !*abort);
    if (!ok) fail_timeout(ctl, jb.meta);
    fence_after_sync();
    for (int h = 0; h < MH; ++h) {
      if (ok) {
        float *srow = stg + (size_t)(q * 32 + lane) * LDS;
        for (int c0 = 0; c0 < N; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + h * N + ((uint32_t)(q * 32) << 16) + c0, v);
          tmem_ld_wait();
          float4 *dst = reinterpret_cast<float4 *>(srow + c0);
          dst[0] = make_float4(v[0], v[1], v[2], v[3]);
          dst[1] = make_float4(v[4], v[5], v[6], v[7]);
          dst[2] = make_float4(v[8], v[9], v[10], v[11]);
          dst[3] = make_float4(v[12], v[13], v[14], v[15]);
        }
      }
      named_sync(1, 128);
      if (ok)
        for (int i = 0; i < 32; ++i) {
          const int row = q * 32 + i;
          const float4 *src = reinterpret_cast<const float4 *>(stg + (size_t)row * LDS);
          float4 *dst = reinterpret_cast<float4 *>(out + (size_t)(h * 128 + row) * R);
          for (int c = lane; c < N / 4; c += 32) dst[c] = src[c];
        }
      named_sync(1, 128);
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

// Sigma-scaled basis for the reconstruction: bsig[c][l] = bf16(sigma_l * B[c][l]) for l < k, else 0.
__global__ void k_bsig(const ReconJob *jobs, int d, int r) {
  const ReconJob &jb = jobs[blockIdx.y];
  const int k = (int)jb.meta[ISKV_META_K];
  const __nv_bfloat16 *B = static_cast<const __nv_bfloat16 *>(jb.B);
  __nv_bfloat16 *bs = static_cast<__nv_bfloat16 *>(jb.bsig);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < d * r; e += gridDim.x * blockDim.x) {
    const int l = e % r;
    bs[e] = __float2bfloat16_rn(l < k ? jb.sigma[l] * __bfloat162float(B[e]) : 0.f);
  }
}

// ================================================================================================
// Failure-path self-test: a bounded wait on a barrier that nothing arrives at.
__global__ void k_wait_timeout(int64_t *meta, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort, limit_ns)) record_status(meta, ISKV_ERR_TIMEOUT);
}

cudaError_t launch_wait_timeout(int64_t *meta, uint64_t limit_ns, cudaStream_t s) {
  k_wait_timeout<<<1, 32, 0, s>>>(meta, limit_ns);
  count_launches(1);
  return cudaGetLastError();
}

// ================================================================================================
// Host side: tensor-map encoding through the driver entry point, job tables, launches.

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D two-byte row-major matrix [rows][cols], box {box_cols, box_rows} (box_cols x 2 bytes no
// wider than the swizzle span), 128-byte swizzle unless given.
bool encode_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows,
               uint32_t box_cols = 64, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

int tc_sm_count() { return num_sms(); }

bool tc_rotation_supported(int r, int storage) {
  return storage == ISKV_BF16 && r % 64 == 0 && r >= 64 && r <= 256 && encode_fn() != nullptr;
}

bool tc_recon_supported(int r, int storage, int out_dtype, int head_dim) {
  return storage == ISKV_BF16 && out_dtype == ISKV_BF16 && head_dim == 128 && r % 64 == 0 &&
         r >= 64 && r <= 256 && encode_fn() != nullptr;
}

constexpr size_t kRotSmemCap = 227 * 1024;

// Shared memory of a rotation with `stages` A slabs: the resident transpose (kslabs slabs of
// r rows x 128 B), the ring, the epilogue's staged rows (stg), the barriers and the 1 KB
// alignment slack.
size_t tc_rotate_smem(int r, int kslabs, int stages, int stg) {
  return 1024 + (size_t)kslabs * r * 128 + (size_t)stages * SLAB_BYTES +
         (stg ? 8 * ROT_STG_BYTES : 0) + sizeof(RotCtl);
}

// Ring depth and epilogue form: tile stores (r a multiple of 128, so that a warp's columns are
// whole 64-column boxes) with at least two ring stages when they fit, else per-row stores; the
// deepest ring (up to ROT_MAX_STAGES, after the staging) that fits. stages = 0: does not fit.
void tc_rotate_shape(int r, int kslabs, int &stages, int &stg) {
  for (stg = (r % 128 == 0) ? 1 : 0; stg >= 0; --stg)
    for (stages = ROT_MAX_STAGES; stages >= 2; --stages)
      if (tc_rotate_smem(r, kslabs, stages, stg) <= kRotSmemCap) return;
  stages = 0;
  stg = 0;
}

static cudaError_t launch_rotate(const TcJob *djobs, int count, int r, int d, int kslabs,
                                 int mode, int tiles_per_job, cudaStream_t s) {
  TcParams tp;
  tp.r = r;
  tp.d = d;
  tp.n_heads = 0;
  tp.hp = 0;
  tp.kslabs = kslabs;
  tp.mode = mode;
  tc_rotate_shape(r, kslabs, tp.stages, tp.stg);
  tp.count = count;
  tp.tiles_per_job = tiles_per_job;
  tp.theta = 0.0;
  if (tp.stages == 0) return cudaErrorInvalidConfiguration;
  const size_t smem = tc_rotate_smem(r, kslabs, tp.stages, tp.stg);
  cudaError_t e = cudaFuncSetAttribute(k_rotate_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int total = tp.count * tp.tiles_per_job;
  const int grid = total < num_sms() ? total : num_sms();
  k_rotate_tc<<<grid, ROT_THREADS, smem, s>>>(djobs, tp);
  count_launches(1);
  return cudaGetLastError();
}

// Resident basis rows for hp heads, the U slab ring, the output staging rows, the barriers and the
// RoPE frequencies.
size_t tc_rec_smem(int r, int hp, int stages) {
  return 1024 + (size_t)hp * (r / 64) * SLAB_BYTES + (size_t)stages * SLAB_BYTES +
         (size_t)REC_STG_BYTES + sizeof(RecCtl) + sizeof(RopeTab);
}

constexpr size_t kRecSmemCap = 227 * 1024;

// Heads per CTA and U ring depth for the reconstruction: two heads when the head count is even,
// and as many 16 KB slabs (up to REC_MAX_STAGES) as the shared memory left over holds.
void tc_rec_shape(int r, int n_heads, int &hp, int &stages) {
  hp = (n_heads % 2 == 0 && tc_rec_smem(r, 2, 3) <= kRecSmemCap) ? 2 : 1;
  stages = REC_MAX_STAGES;
  while (stages > 2 && tc_rec_smem(r, hp, stages) > kRecSmemCap) --stages;
}

cudaError_t launch_tc_rotation(const TcJob *djobs, int count, int r, int64_t n_cap_max,
                               cudaStream_t s) {
  return launch_rotate(djobs, count, r, 0, r / 64, 0, (int)((n_cap_max + TC_M - 1) / TC_M), s);
}

bool encode_rotation_job(TcJob &tj, void *U, int64_t n_cap, int r, const void *gtb,
                         const int32_t *sc, int64_t *meta) {
  std::memset(&tj, 0, sizeof(tj));
  if (!encode_2d(&tj.mapA, U, (uint64_t)n_cap, (uint64_t)r, 128)) return false;
  if (!encode_2d(&tj.mapB, gtb, (uint64_t)r, (uint64_t)r, (uint32_t)r)) return false;
  if (!encode_2d(&tj.mapS, U, (uint64_t)n_cap, (uint64_t)r, 32)) return false;
  tj.U = U;
  tj.sc = sc;
  tj.meta = meta;
  return true;
}

static bool basis_fits(int r, int bpad) {
  int stages, stg;
  tc_rotate_shape(r, (r + bpad) / 64, stages, stg);
  return stages > 0;
}

bool tc_basis_supported(int r, int bpad, int storage) {
  return storage == ISKV_BF16 && r % 64 == 0 && r >= 64 && r <= 256 && bpad % 64 == 0 &&
         basis_fits(r, bpad) && encode_fn() != nullptr;
}

bool encode_basis_job(TcJob &tj, void *B, int d, int r, const void *Pb, int bpad,
                      const void *Htb, const int32_t *sc, int64_t *meta) {
  std::memset(&tj, 0, sizeof(tj));
  if (!encode_2d(&tj.mapA, B, (uint64_t)d, (uint64_t)r, 128)) return false;
  if (bpad > 0 && !encode_2d(&tj.mapO, Pb, (uint64_t)d, (uint64_t)bpad, 128)) return false;
  if (!encode_2d(&tj.mapB, Htb, (uint64_t)r, (uint64_t)(r + bpad), (uint32_t)r)) return false;
  if (!encode_2d(&tj.mapS, B, (uint64_t)d, (uint64_t)r, 32)) return false;
  tj.U = B;
  tj.sc = sc;
  tj.meta = meta;
  return true;
}

cudaError_t launch_tc_basis(const TcJob *djobs, int count, int d, int r, int kpad, cudaStream_t s) {
  return launch_rotate(djobs, count, r, d, kpad / 64, 1, (d + TC_M - 1) / TC_M, s);
}

bool encode_recon_job(TcJob &tj, const void *U, int64_t n_cap, int r, const void *bsig, int d,
                      void *out, const int32_t *pos, int64_t *meta, int64_t n_total, int rope) {
  std::memset(&tj, 0, sizeof(tj));
  if (!encode_2d(&tj.mapA, U, (uint64_t)n_cap, (uint64_t)r, 128)) return false;
  if (!encode_2d(&tj.mapB, bsig, (uint64_t)d, (uint64_t)r, 128)) return false;
  tj.tiles_ok = n_total >= 32;
  if (tj.tiles_ok && !encode_2d(&tj.mapO, out, (uint64_t)n_total, (uint64_t)d, 32, 32,
                                CU_TENSOR_MAP_SWIZZLE_64B))
    return false;
  tj.out = out;
  tj.pos = pos;
  tj.meta = meta;
  tj.n_total = n_total;
  tj.rope = rope;
  return true;
}

cudaError_t launch_recon_bsig(const ReconJob *djobs_recon, const ReconParams &p, cudaStream_t s) {
  k_bsig<<<dim3(64, p.count), 256, 0, s>>>(djobs_recon, p.d, p.r);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tc_recon(const TcJob *djobs, const ReconParams &p, cudaStream_t s) {
  TcParams tp;
  tp.r = p.r;
  tp.d = p.d;
  tp.n_heads = p.n_heads;
  tp.count = p.count;
  tp.tiles_per_job = (int)((p.n_cap_max + TC_M - 1) / TC_M);
  tp.theta = p.theta;
  tc_rec_shape(p.r, p.n_heads, tp.hp, tp.stages);
  const size_t smem = tc_rec_smem(p.r, tp.hp, tp.stages);
  cudaError_t e = cudaFuncSetAttribute(k_rec_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // Whole groups of n_heads / hp CTAs, as many as fit one per SM (at least one group), and no
  // more groups than row tiles.
  const int G = p.n_heads / tp.hp;
  const int total = tp.count * tp.tiles_per_job;
  int groups = num_sms() / G;
  if (groups < 1) groups = 1;
  if (groups > total) groups = total;
  k_rec_tc<<<groups * G, REC_THREADS, smem, s>>>(djobs, tp, make_rope_tab(p.theta));
  count_launches(1);
  return cudaGetLastError();
}

bool tc_attn_supported(int r, int storage, int head_dim, int n_q, int n_kv) {
  if (n_kv < 1 || n_q % n_kv) return false;
  const int qpk = n_q / n_kv;
  return storage == ISKV_BF16 && head_dim == 128 && r % 64 == 0 && r >= 64 && r <= 256 &&
         (qpk == 1 || qpk == 2 || qpk == 4 || qpk == 8) && encode_fn() != nullptr;
}

bool encode_attn_job(TcJob &tj, const void *U, int64_t n_cap, int r, const void *bsig, int d,
                     float *S, const float *q, const int32_t *pos, int64_t *meta, int64_t n_total,
                     float scale) {
  std::memset(&tj, 0, sizeof(tj));
  if (!encode_2d(&tj.mapA, U, (uint64_t)n_cap, (uint64_t)r, 128)) return false;
  if (!encode_2d(&tj.mapB, bsig, (uint64_t)d, (uint64_t)r, 128)) return false;
  tj.pos = pos;
  tj.meta = meta;
  tj.n_total = n_total;
  tj.rope = 1;
  tj.tiles_ok = 0;
  tj.S = S;
  tj.q = q;
  tj.scale = scale;
  return true;
}

template <int QPK>
static cudaError_t attn_scores_qpk(const TcJob *djobs, const TcParams &tp, int G, cudaStream_t s) {
  const size_t smem = tc_sco_smem(tp.r, tp.hp, tp.stages);
  cudaError_t e = cudaFuncSetAttribute(k_scores_tc<QPK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int total = tp.count * tp.tiles_per_job;
  int groups = num_sms() / G;
  if (groups < 1) groups = 1;
  if (groups > total) groups = total;
  k_scores_tc<QPK><<<groups * G, SCO_THREADS, smem, s>>>(djobs, tp, make_rope_tab(tp.theta));
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tc_attn_scores(const TcJob *djobs, const AttnParams &p, cudaStream_t s) {
  TcParams tp;
  tp.r = p.rk;
  tp.d = p.d;
  tp.n_heads = p.n_kv;
  tp.count = p.count;
  tp.tiles_per_job = (int)((p.n_cap_max + TC_M - 1) / TC_M);
  tp.theta = p.theta;
  const int qpk = p.n_q / p.n_kv;
  // Two heads per CTA when the head count is even; as deep a U slab ring as the rest leaves room for.
  tp.hp = (p.n_kv % 2 == 0 && tc_sco_smem(p.rk, 2, 3) <= kRecSmemCap) ? 2 : 1;
  tp.stages = REC_MAX_STAGES;
  while (tp.stages > 2 && tc_sco_smem(p.rk, tp.hp, tp.stages) > kRecSmemCap) --tp.stages;
  const int G = p.n_kv / tp.hp;
  switch (qpk) {
    case 1: return attn_scores_qpk<1>(djobs, tp, G, s);
    case 2: return attn_scores_qpk<2>(djobs, tp, G, s);
    case 4: return attn_scores_qpk<4>(djobs, tp, G, s);
    case 8: return attn_scores_qpk<8>(djobs, tp, G, s);
    default: return cudaErrorInvalidValue;
  }
}

bool tc_gram_supported(int r, int storage) {
  return storage == ISKV_BF16 && (r == 128 || r == 256) && encode_fn() != nullptr;
}

// ================================================================================================
// Decode-attention value mixing on the tensor cores: for each split of ATTN_CHUNK value rows,
// D = U_split^T P_split (r x 64), the coordinates of the history rows weighted by the query
// heads' probabilities (P: [n_cap][64] bf16, queries padded to 64 columns). The structure is the
// Gram kernel's: both operands MN-major, 64-row stages of r/64 U slabs plus one P slab, two
// M = 128 halves, N = 64; the epilogue writes the float32 partial [split][r][64].
__global__ void __launch_bounds__(GRAM_THREADS, 1) k_pv_tc(const TcJob *jobs, PvParams p) {
  const int job = blockIdx.x / p.nsplit, split = blockIdx.x % p.nsplit;
  const TcJob &jb = jobs[job];
  const int R = p.r, SL = R / 64, MH = R / 128, N = 64;
  const int64_t n = jb.meta[ISKV_META_N];
  const int r0 = split * ATTN_CHUNK;
  const int nrows = (int)(n - r0 < ATTN_CHUNK ? n - r0 : ATTN_CHUNK);
  float *out = reinterpret_cast<float *>(jb.out) + (size_t)split * R * N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (nrows <= 0) {  // an empty split contributes zeros (uniform over the CTA)
    for (int e = threadIdx.x; e < R * N; e += blockDim.x) out[e] = 0.f;
    return;
  }
  const int nk = (nrows + GRAM_KT - 1) / GRAM_KT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int SLAB = GRAM_KT * 128;  // 64 rows x 64 columns bf16
  const int STAGE_BYTES = (SL + 1) * SLAB;
  TcCtl *ctl = reinterpret_cast<TcCtl *>(smem + GRAM_STAGES * STAGE_BYTES);
  uint64_t *full = reinterpret_cast<uint64_t *>(ctl + 1);   // [GRAM_STAGES]
  uint64_t *empty = full + GRAM_STAGES;                      // [GRAM_STAGES]
  const uint32_t ncols = MH * N <= 128 ? 128 : 256;
  const uint32_t idesc = idesc_bf16_f32_mn(128, N);
  if (threadIdx.x == 0) {
    for (int i = 0; i < GRAM_STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(&ctl->acc_full[0], 1);
    mbar_init(&ctl->done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&ctl->tmem, ncols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int *abort = &ctl->abort;

  if (warp == 0 && lane == 0) {
    tensormap_acquire(&jb.mapA);
    tensormap_acquire(&jb.mapB);
    for (int kt = 0; kt < nk && !*abort; ++kt) {
      const int st = kt % GRAM_STAGES, use = kt / GRAM_STAGES;
      if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, abort, WAIT_NS)) {
        fail_timeout(ctl, jb.meta);
        break;
      }
      mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
      uint8_t *stage = smem + st * STAGE_BYTES;
      for (int sl = 0; sl < SL; ++sl)
        tma_load_2d(stage + sl * SLAB, &jb.mapA, sl * 64, r0 + kt * GRAM_KT, &full[st]);
      tma_load_2d(stage + SL * SLAB, &jb.mapB, 0, r0 + kt * GRAM_KT, &full[st]);
    }
    for (int k = 1; k <= GRAM_STAGES && nk - k >= 0; ++k)
      mbar_wait(&full[(nk - k) % GRAM_STAGES], ((nk - k) / GRAM_STAGES) & 1, abort, WAIT_NS / 4);
  } else if (warp == 1 && lane == 0) {
    bool ok = true;
    for (int kt = 0; kt < nk && ok && !*abort; ++kt) {
      const int st = kt % GRAM_STAGES, use = kt / GRAM_STAGES;
      if (!mbar_wait(&full[st], use & 1, abort, WAIT_NS)) { ok = false; break; }
      fence_after_sync();
      const uint32_t base = smem_u32(smem + st * STAGE_BYTES);
#pragma unroll
      for (int kk = 0; kk < GRAM_KT / 16; ++kk) {
        const uint64_t bdesc = sw128_mn_desc(base + SL * SLAB + kk * 2048, SLAB);
        for (int h = 0; h < MH; ++h) {
          const uint64_t adesc = sw128_mn_desc(base + h * 2 * SLAB + kk * 2048, SLAB);
          mma_bf16(tmem + h * N, adesc, bdesc, idesc, (kt | kk) != 0);
        }
      }
      mma_commit(&empty[st]);
    }
    if (!ok) fail_timeout(ctl, jb.meta);
    mma_commit(&ctl->acc_full[0]);
    mma_commit(&ctl->done);
    mbar_wait(&ctl->done, 0, abort, WAIT_NS / 4);
  } else if (warp >= 2) {
    const int q = warp & 3;
    if (__all_sync(~0u, mbar_wait(&ctl->acc_full[0], 0, abort, WAIT_NS) && !*abort)) {
      fence_after_sync();
      for (int h = 0; h < MH; ++h) {
        const int row = h * 128 + q * 32 + lane;
        for (int c0 = 0; c0 < N; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + h * N + ((uint32_t)(q * 32) << 16) + c0, v);
          tmem_ld_wait();
          float4 *dst = reinterpret_cast<float4 *>(out + (size_t)row * N + c0);
          dst[0] = make_float4(v[0], v[1], v[2], v[3]);
          dst[1] = make_float4(v[4], v[5], v[6], v[7]);
          dst[2] = make_float4(v[8], v[9], v[10], v[11]);
          dst[3] = make_float4(v[12], v[13], v[14], v[15]);
        }
      }
    } else {
      fail_timeout(ctl, jb.meta);
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

bool tc_pv_supported(int r, int storage, int n_q) {
  return storage == ISKV_BF16 && r % 128 == 0 && r >= 128 && r <= 256 && n_q <= 64 &&
         encode_fn() != nullptr;
}

bool encode_pv_job(TcJob &tj, const void *U, int64_t n_cap, int r, const void *Pb, float *wpart,
                   int64_t *meta) {
  std::memset(&tj, 0, sizeof(tj));
  if (!encode_2d(&tj.mapA, U, (uint64_t)n_cap, (uint64_t)r, GRAM_KT)) return false;
  if (!encode_2d(&tj.mapB, Pb, (uint64_t)n_cap, 64, GRAM_KT)) return false;
  tj.meta = meta;
  tj.out = wpart;
  return true;
}

cudaError_t launch_tc_pv(const TcJob *djobs, const PvParams &p, cudaStream_t s) {
  const size_t smem = 1024 + (size_t)GRAM_STAGES * (p.r / 64 + 1) * GRAM_KT * 128 + sizeof(TcCtl) +
                      2 * GRAM_STAGES * sizeof(uint64_t);
  cudaError_t e = cudaFuncSetAttribute(k_pv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_pv_tc<<<p.count * p.nsplit, GRAM_THREADS, smem, s>>>(djobs, p);
  count_launches(1);
  return cudaGetLastError();
}

bool encode_gram_job(TcJob &tj, const void *U, int64_t n_cap, const void *B, int d, int r,
                     const int32_t *sc, int64_t *meta, void *ws) {
  std::memset(&tj, 0, sizeof(tj));
  if (!encode_2d(&tj.mapA, U, (uint64_t)n_cap, (uint64_t)r, GRAM_KT)) return false;
  if (!encode_2d(&tj.mapB, B, (uint64_t)d, (uint64_t)r, GRAM_KT)) return false;
  tj.sc = sc;
  tj.meta = meta;
  tj.out = ws;
  return true;
}

cudaError_t launch_tc_gram(const TcJob *djobs, const GramParams &p, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  const size_t smem = 1024 + gram_area_bytes(p.r) + sizeof(TcCtl) + 2 * GRAM_RING * sizeof(uint64_t);
  e = cudaFuncSetAttribute(k_gram_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_gram_tc<<<p.count * (p.nsu + p.nsb), GRAM_THREADS, smem, s>>>(djobs, p);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Projection of the fold on the tensor cores.
static_assert(sizeof(ProjJob) <= sizeof(TcJob), "projection jobs use a TcJob-sized table");

bool tc_project_supported(int d, int r, int b, int storage, int f_dtype) {
  return storage == ISKV_BF16 && f_dtype == ISKV_BF16 && b == PROJ_B && (r == 128 || r == 256) &&
         d % 128 == 0 && d >= 128 && d <= 1024 && encode_fn() != nullptr;
}

bool encode_project_job(ProjJob &pj, void *B, int d, int r, const void *F, int b, float *C,
                        float *E, void *E1, const int32_t *sc, int64_t *meta) {
  std::memset(&pj, 0, sizeof(pj));
  if (!encode_2d(&pj.mapBm, B, (uint64_t)d, (uint64_t)r, 64)) return false;
  if (!encode_2d(&pj.mapBk, B, (uint64_t)d, (uint64_t)r, 128)) return false;
  if (!encode_2d(&pj.mapF, F, (uint64_t)b, (uint64_t)d, 64)) return false;
  if (!encode_2d(&pj.mapE1, E1, (uint64_t)(2 * b), (uint64_t)d, 64)) return false;
  pj.B = static_cast<__nv_bfloat16 *>(B);
  pj.F = static_cast<const __nv_bfloat16 *>(F);
  pj.C = C;
  pj.E = E;
  pj.E1 = static_cast<__nv_bfloat16 *>(E1);
  pj.sc = sc;
  pj.meta = meta;
  return true;
}

cudaError_t launch_tc_project(const ProjJob *djobs, int count, int d, int r, cudaStream_t s) {
  ProjParams pp;
  pp.r = r;
  pp.d = d;
  pp.count = count;
  const size_t smem = 1024 + (size_t)PROJ_STAGES * PROJ_STAGE_BYTES + (size_t)(r / 64) * PROJ_B * 128 +
                      sizeof(ProjCtl);
  cudaError_t e = cudaFuncSetAttribute(k_project_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_project_tc<<<count, TC_THREADS, smem, s>>>(djobs, pp);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace iskv
