// Opt-in stage timing and launch counting for libiskv (host side).
//
// When enabled, every entry point records a CUDA event on the caller's stream before its first
// kernel and after each internal stage; iskv_stage_* read back the accumulated device time per
// stage. The launch counter counts every kernel the library launches, enabled or not.
#pragma once

#include <cuda_runtime.h>

namespace iskv {

enum Stage {
  ST_FOLD_PROJECT = 0,
  ST_FOLD_RESIDUAL,
  ST_FOLD_CORE,
  ST_FOLD_BASIS,
  ST_FOLD_COORDS,
  ST_FOLD_FINALIZE,
  ST_REORTH_GRAM,
  ST_REORTH_NS,
  ST_REORTH_CORE,
  ST_REORTH_COORDS,
  ST_REORTH_BASIS,
  ST_RECON_PREPARE,
  ST_RECON_COMPRESSED,
  ST_RECON_EXACT,
  ST_SELECT,
  ST_UPLOAD,
  ST_ATTN_PREPARE,
  ST_ATTN_SCORES,
  ST_ATTN_SOFTMAX,
  ST_ATTN_VALUES,
  ST_CACHE_APPEND,
  ST_CACHE_EVICT,
  ST_COUNT
};

const char *stage_name(int s);

// Begin a timed section on stream s (records the start event when timing is on).
void stage_begin(cudaStream_t s);
// Close stage `id`: the time since the previous mark on this section is charged to it.
void stage_mark(cudaStream_t s, int id);

// Count `n` kernel launches.
void count_launches(int n);

}  // namespace iskv
