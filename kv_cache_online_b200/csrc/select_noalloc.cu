// Prompt-block selection that needs no caller workspace and allocates nothing.
//
// Who needs this: code that runs inside a host framework which owns all device memory and hands
// a plugin only its inputs and outputs (an inference-engine plugin, for instance, has no
// allocator of its own to ask for scratch), and code on a latency-critical path that must not
// call cudaMalloc, which can synchronise the whole device. Such callers cannot provide the
// workspace that iskv_select_prompt_blocks() takes.
//
// Instead the scratch lives in one file-scope device array of fixed size, ISKV_NOALLOC_SCRATCH
// bytes, which the CUDA runtime places on every GPU that loads this library and keeps until the
// process exits. The selection kernels are the same ones the workspace form launches.
//
// In host code the array's name is only a host-side stand-in: a kernel given it would fault or,
// where the GPU can reach host memory, silently use the wrong memory. Its device address is
// therefore looked up with cudaGetSymbolAddress, once per device, with that device current, the
// first time this entry point runs on that device.
#include <mutex>

#include "iskv.h"
#include "profiling.h"
#include "select.h"

namespace iskv {

static __device__ __align__(256) unsigned char g_select_scratch[ISKV_NOALLOC_SCRATCH];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up on first use).
cudaError_t scratch_address(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace iskv

using namespace iskv;

extern "C" iskv_status iskv_select_prompt_blocks_noalloc(
    const void *keys, int32_t k_dtype, int64_t L, int32_t n_heads, int32_t head_dim, int32_t block,
    int32_t per_head, int32_t suffix_blocks, int32_t v_radius, int32_t *pk_out, int32_t *pv_out,
    int32_t *head_blocks_out, int64_t *counts_out, void *stream) {
  if (!keys || !pk_out || !pv_out || !head_blocks_out || !counts_out) return ISKV_ERR_ARG;
  if (k_dtype != ISKV_F32 && k_dtype != ISKV_BF16) return ISKV_ERR_ARG;
  if (L < 1 || L > ((int64_t)1 << 24) || n_heads < 1 || n_heads > 64 || head_dim < 2 ||
      head_dim > 256 || head_dim % 2 || block < 1 || block > 64 || per_head < 0 ||
      per_head > 4096 || suffix_blocks < 0 || v_radius < 0)
    return ISKV_ERR_SHAPE;
  // The scratch has a fixed size: larger problems are refused, never truncated.
  if (select_ws_layout(L, n_heads, block).total > (size_t)ISKV_NOALLOC_SCRATCH)
    return ISKV_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return ISKV_ERR_CUDA;
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
  a.ws = scratch;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  stage_begin(s);
  if (launch_select(a, s) != cudaSuccess) return ISKV_ERR_CUDA;
  stage_mark(s, ST_SELECT);
  return ISKV_OK;
}
