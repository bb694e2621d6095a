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
// therefore looked up with cudaGetSymbolAddress, with the caller's device current, on every call:
// the lookup is a host-side query, and an address is never carried over from an earlier call, so
// a context that the host framework tore down and re-created (cudaDeviceReset) gets the array's
// new address. The first call on a device may load the library's device code there; make it
// before any stream capture on that device.
#include "api_error.h"
#include "iskv.h"
#include "profiling.h"
#include "select.h"

namespace iskv {

static __device__ __align__(256) unsigned char g_select_scratch[ISKV_NOALLOC_SCRATCH];

}  // namespace iskv

using namespace iskv;

extern "C" iskv_status iskv_select_prompt_blocks_noalloc(
    const void *keys, int32_t k_dtype, int64_t L, int32_t n_heads, int32_t head_dim, int32_t block,
    int32_t per_head, int32_t suffix_blocks, int32_t v_radius, int32_t *pk_out, int32_t *pv_out,
    int32_t *head_blocks_out, int64_t *counts_out, void *stream) {
  const char *who = "iskv_select_prompt_blocks_noalloc";
  clear_last_error();
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
  // The scratch has a fixed size: larger problems are refused, never truncated.
  const size_t need = select_ws_layout(L, n_heads, block).total;
  if (need > (size_t)ISKV_NOALLOC_SCRATCH)
    return fail(ISKV_ERR_WORKSPACE,
                "%s: this prompt needs %zu bytes of scratch, more than the %u-byte fixed array", who,
                need, (unsigned)ISKV_NOALLOC_SCRATCH);
  void *scratch = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&scratch, g_select_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "iskv_select_prompt_blocks_noalloc: scratch address");
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
  e = launch_select(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "iskv_select_prompt_blocks_noalloc: launch");
  stage_mark(s, ST_SELECT);
  return ISKV_OK;
}
