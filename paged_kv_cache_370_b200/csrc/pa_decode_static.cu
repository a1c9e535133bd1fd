// pa_decode_static.cu -- pa_decode for callers that cannot allocate device memory.
//
// The split-context scratch that pa_decode takes from its caller lives here in
// a fixed file-scope device array instead. Every GPU that loads the library
// holds the array (PA_STATIC_WORKSPACE_BYTES) until the process exits. In host
// code the array's name only stands for the symbol -- it is not a device
// address -- so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and passes the result on.

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "pa.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

void *g_static_workspace_addr[kMaxDevices];
cudaError_t g_static_workspace_err[kMaxDevices];
std::once_flag g_static_workspace_once[kMaxDevices];

}  // namespace

extern "C" pa_status pa_decode_static_workspace(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
    int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int num_blocks, float scale, pa_dtype dtype, int partition_tokens,
    void *stream) {
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               max_context_len, partition_tokens);
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_UNSUPPORTED;  // beyond the fixed array
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  // once per device, with that device current: the array's device address
  std::call_once(g_static_workspace_once[dev], [dev] {
    g_static_workspace_err[dev] =
        cudaGetSymbolAddress(&g_static_workspace_addr[dev], g_static_workspace);
  });
  if (g_static_workspace_err[dev] != cudaSuccess || !g_static_workspace_addr[dev])
    return PA_ERR_CUDA;
  return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                   max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                   num_blocks, scale, dtype, g_static_workspace_addr[dev],
                   PA_STATIC_WORKSPACE_BYTES, partition_tokens, stream);
}
