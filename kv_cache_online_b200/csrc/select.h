// Prompt-block selection: workspace layout and launcher.
#pragma once

#include "common.cuh"

namespace iskv {

constexpr int64_t SCAN_CHUNK = 8192;

struct SelectWsLayout {
  size_t scores, blkflag, prot, near, cntK, cntV, chunk, total;
};

SelectWsLayout select_ws_layout(int64_t L, int H, int block);

struct SelectArgs {
  const void *keys;
  int k_dtype;
  int64_t L;
  int H, hd, block, per_head, suffix_blocks, v_radius;
  int32_t *pk_out, *pv_out, *head_blocks;
  int64_t *counts;
  void *ws;
};

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s);

}  // namespace iskv
