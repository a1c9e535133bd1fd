// pa_decode_static.cu -- pa_decode for callers that cannot allocate device memory.
//
// The split-context scratch that pa_decode takes from its caller lives here in
// a fixed file-scope device array instead. Every GPU that loads the library
// holds the array (PA_STATIC_WORKSPACE_BYTES) until the process exits. In host
// code the array's name only stands for the symbol -- it is not a device
// address -- so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and passes the result on.
// Only a successful lookup is kept; a failed one is retried by the next call.
//
// pa_decode requires the first bytes of its workspace (the even-split kernel's
// per-CTA counters) to be zero when a call starts. A completed call leaves them
// zero, but a call that gave up a wait (PA_DEVERR_TIMEOUT) may not, and the
// caller of this entry point has no pointer to the array to clear them. So
// every call first clears that region on its own stream (cudaMemsetAsync:
// stream-ordered, no allocation) and then runs pa_decode.

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

std::mutex g_static_workspace_mu;
void *g_static_workspace_addr[kMaxDevices];  // nullptr until a lookup succeeded

static_assert(kPaCounterRegionBytes <= PA_STATIC_WORKSPACE_BYTES, "counters fit the array");

// The array's device address on the current device, looked up once per device.
void *static_workspace_address(int dev) {
  std::lock_guard<std::mutex> lock(g_static_workspace_mu);
  if (!g_static_workspace_addr[dev]) {
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_static_workspace) != cudaSuccess || !addr) {
      cudaGetLastError();  // do not leave the failure for the next CUDA call to report
      return nullptr;
    }
    g_static_workspace_addr[dev] = addr;
  }
  return g_static_workspace_addr[dev];
}

}  // namespace

extern "C" pa_status pa_decode_static_workspace(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
    int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int num_blocks, float scale, pa_dtype dtype, int partition_tokens,
    void *stream) {
  // the scratch of the kernel this call runs (pa_decode itself rejects bad arguments)
  const size_t need = pa_internal_decode_need(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              block_size, num_blocks, max_context_len,
                                              partition_tokens);
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_UNSUPPORTED;  // beyond the fixed array
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  void *ws = static_workspace_address(dev);
  if (!ws) return PA_ERR_CUDA;
  if (need > 0 && cudaMemsetAsync(ws, 0, kPaCounterRegionBytes,
                                  static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                   max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                   num_blocks, scale, dtype, ws, PA_STATIC_WORKSPACE_BYTES, partition_tokens,
                   stream);
}
