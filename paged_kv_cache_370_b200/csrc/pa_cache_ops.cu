// pa_cache_ops.cu -- the two bit-exact copy kernels of the paged KV cache.
//
//  * pa_reshape_and_cache: store each new token's K and V rows at its slot
//    (page "08. PagedAttention：把 KV Cache 分页管理", section
//    "为什么叫 PagedAttention": slot = block_table[logical block] * block_size
//    + offset; a small GPU kernel writes every token's K/V to its slot).
//  * pa_copy_blocks: whole-block copies for copy-on-write (page
//    "PagedAttention 核心思想解析", section 2.3: allocate a new block, copy
//    the original block's contents, update the table).
//  * pa_swap_out / pa_swap_in: whole-block copies between the device pools and
//    a host swap space (page "08. PagedAttention：把 KV Cache 分页管理",
//    section "分页还顺带解决了什么": a preempted request's blocks go to CPU
//    memory and come back later; same-size blocks make this easy). The swap
//    space is pinned host memory mapped into the device's address space, so
//    one kernel moves every block of a swap over PCIe / C2C, instead of one
//    copy call per block.
//
// Both move 16-byte vectors (every row is head_dim * 2 bytes, a multiple of
// 16), index in 64 bits, and check the ids they are given: a slot or block
// outside the pool skips the access and sets a bit of this file's device
// error word instead of faulting.

#include <cuda_runtime.h>

#include <cstdint>
#include <new>

#include "pa.h"
#include "pa_internal.h"

namespace {

__device__ int g_cache_ops_error;

// One thread per 16-byte chunk of a (token, kv head) row; the thread moves the
// chunk of K and the chunk of V.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
    const int64_t *__restrict__ slot_mapping, uint4 *__restrict__ k_cache,
    uint4 *__restrict__ v_cache, int64_t total_chunks, int chunks_per_row, int num_kv_heads,
    int block_size, int64_t num_slots) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total_chunks) return;
  const int64_t row = i / chunks_per_row;          // (token, head) row
  const int c = (int)(i - row * chunks_per_row);   // chunk in the row
  const int64_t t = row / num_kv_heads;
  const int h = (int)(row - t * num_kv_heads);
  const int64_t slot = __ldg(slot_mapping + t);
  if (slot < 0) return;                            // padding token
  if (slot >= num_slots) {
    atomicOr(&g_cache_ops_error, PA_DEVERR_SLOT);
    return;
  }
  const int64_t blk = slot / block_size;
  const int64_t off = slot - blk * block_size;
  const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * chunks_per_row + c;
  k_cache[dst] = __ldg(k_new + i);
  v_cache[dst] = __ldg(v_new + i);
}

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// grid = (chunks of a block / (threads * unroll), num_pairs, 2: K then V)
__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(
    uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
    const int64_t *__restrict__ block_pairs, int64_t chunks_per_block, int num_blocks) {
  const int pair = blockIdx.y;
  const int64_t src = __ldg(block_pairs + 2 * pair);
  const int64_t dst = __ldg(block_pairs + 2 * pair + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0)
      atomicOr(&g_cache_ops_error, PA_DEVERR_COPY_PAIR);
    return;
  }
  if (src == dst) return;
  uint4 *pool = blockIdx.z == 0 ? k_cache : v_cache;
  const uint4 *s = pool + src * chunks_per_block;
  uint4 *d = pool + dst * chunks_per_block;
  const int64_t base = (int64_t)blockIdx.x * kCopyThreads * kCopyUnroll + threadIdx.x;
  uint4 buf[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t j = base + (int64_t)u * kCopyThreads;
    if (j < chunks_per_block) buf[u] = s[j];
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t j = base + (int64_t)u * kCopyThreads;
    if (j < chunks_per_block) d[j] = buf[u];
  }
}

constexpr int kSwapUnroll = 8;  // 16-byte loads in flight per thread (host memory is far)

// grid = (chunks of a block / (threads * unroll), pairs, 2: K then V). Pair i
// copies source block pairs[i][0] to destination block pairs[i][1].
__global__ void __launch_bounds__(kCopyThreads) swap_blocks_kernel(
    uint4 *__restrict__ dst_k, uint4 *__restrict__ dst_v, int64_t dst_blocks,
    const uint4 *__restrict__ src_k, const uint4 *__restrict__ src_v, int64_t src_blocks,
    const int64_t *__restrict__ block_pairs, int64_t chunks_per_block) {
  const int pair = blockIdx.y;
  const int64_t src = block_pairs[2 * pair];
  const int64_t dst = block_pairs[2 * pair + 1];
  if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0)
      atomicOr(&g_cache_ops_error, PA_DEVERR_COPY_PAIR);
    return;
  }
  const uint4 *s = (blockIdx.z == 0 ? src_k : src_v) + src * chunks_per_block;
  uint4 *d = (blockIdx.z == 0 ? dst_k : dst_v) + dst * chunks_per_block;
  const int64_t base = (int64_t)blockIdx.x * kCopyThreads * kSwapUnroll + threadIdx.x;
  uint4 buf[kSwapUnroll];
#pragma unroll
  for (int u = 0; u < kSwapUnroll; ++u) {
    const int64_t j = base + (int64_t)u * kCopyThreads;
    if (j < chunks_per_block) buf[u] = s[j];
  }
#pragma unroll
  for (int u = 0; u < kSwapUnroll; ++u) {
    const int64_t j = base + (int64_t)u * kCopyThreads;
    if (j < chunks_per_block) d[j] = buf[u];
  }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_pool_args(int num_blocks, int num_kv_heads, int block_size, int head_dim,
                     pa_dtype dtype) {
  return num_blocks > 0 && num_kv_heads > 0 && block_size > 0 && head_dim > 0 &&
         (head_dim * 2) % 16 == 0 && (dtype == PA_F16 || dtype == PA_BF16);
}

}  // namespace

extern "C" pa_status pa_reshape_and_cache(const void *k_new, const void *v_new,
                                          const int64_t *slot_mapping, int num_tokens,
                                          void *k_cache, void *v_cache, int num_blocks,
                                          int num_kv_heads, int block_size, int head_dim,
                                          pa_dtype dtype, void *stream) {
  if (num_tokens < 0 || !valid_pool_args(num_blocks, num_kv_heads, block_size, head_dim, dtype))
    return PA_ERR_INVALID;
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_INVALID;
  const int chunks_per_row = head_dim * 2 / 16;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * chunks_per_row;
  const int64_t blocks = (total + 255) / 256;
  if (blocks > INT32_MAX) return PA_ERR_INVALID;
  reshape_and_cache_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slot_mapping,
      static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), total, chunks_per_row,
      num_kv_heads, block_size, (int64_t)num_blocks * block_size);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_pairs,
                                    int num_pairs, int num_blocks, int num_kv_heads,
                                    int block_size, int head_dim, pa_dtype dtype, void *stream) {
  if (num_pairs < 0 || !valid_pool_args(num_blocks, num_kv_heads, block_size, head_dim, dtype))
    return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (num_pairs > 65535 || !k_cache || !v_cache || !block_pairs) return PA_ERR_INVALID;
  if (!aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(block_pairs) & 7u))
    return PA_ERR_INVALID;
  const int64_t chunks = (int64_t)num_kv_heads * block_size * head_dim * 2 / 16;
  const int64_t per_cta = (int64_t)kCopyThreads * kCopyUnroll;
  dim3 grid((unsigned)((chunks + per_cta - 1) / per_cta), (unsigned)num_pairs, 2);
  copy_blocks_kernel<<<grid, kCopyThreads, 0, (cudaStream_t)stream>>>(
      static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), block_pairs, chunks,
      num_blocks);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

struct pa_swap_space {
  void *k_host = nullptr;  // pinned, mapped: [num_blocks][num_kv_heads][block_size][head_dim]
  void *v_host = nullptr;
  uint4 *k_dev = nullptr;  // the same memory as the device sees it
  uint4 *v_dev = nullptr;
  int num_blocks = 0, num_kv_heads = 0, block_size = 0, head_dim = 0;
  pa_dtype dtype = PA_F16;
};

extern "C" {

pa_status pa_swap_space_create(int num_host_blocks, int num_kv_heads, int block_size, int head_dim,
                               pa_dtype dtype, pa_swap_space **out) {
  if (!out || !valid_pool_args(num_host_blocks, num_kv_heads, block_size, head_dim, dtype))
    return PA_ERR_INVALID;
  const size_t bytes = (size_t)num_host_blocks * num_kv_heads * block_size * head_dim * 2;
  pa_swap_space *sp = new (std::nothrow) pa_swap_space();
  if (!sp) return PA_ERR_INVALID;
  const unsigned flags = cudaHostAllocMapped | cudaHostAllocPortable;
  void *dk = nullptr, *dv = nullptr;
  if (cudaHostAlloc(&sp->k_host, bytes, flags) != cudaSuccess ||
      cudaHostAlloc(&sp->v_host, bytes, flags) != cudaSuccess ||
      cudaHostGetDevicePointer(&dk, sp->k_host, 0) != cudaSuccess ||
      cudaHostGetDevicePointer(&dv, sp->v_host, 0) != cudaSuccess) {
    if (sp->k_host) cudaFreeHost(sp->k_host);
    if (sp->v_host) cudaFreeHost(sp->v_host);
    delete sp;
    return PA_ERR_CUDA;
  }
  sp->k_dev = static_cast<uint4 *>(dk);
  sp->v_dev = static_cast<uint4 *>(dv);
  sp->num_blocks = num_host_blocks;
  sp->num_kv_heads = num_kv_heads;
  sp->block_size = block_size;
  sp->head_dim = head_dim;
  sp->dtype = dtype;
  *out = sp;
  return PA_OK;
}

void pa_swap_space_destroy(pa_swap_space *sp) {
  if (!sp) return;
  cudaFreeHost(sp->k_host);
  cudaFreeHost(sp->v_host);
  delete sp;
}

pa_status pa_swap_space_pools(const pa_swap_space *sp, void **k_host, void **v_host) {
  if (!sp || !k_host || !v_host) return PA_ERR_INVALID;
  *k_host = sp->k_host;
  *v_host = sp->v_host;
  return PA_OK;
}

}  // extern "C"

namespace {

pa_status launch_swap(uint4 *dst_k, uint4 *dst_v, int64_t dst_blocks, const uint4 *src_k,
                      const uint4 *src_v, int64_t src_blocks, const int64_t *block_pairs,
                      int num_pairs, int64_t chunks, cudaStream_t stream) {
  const int64_t per_cta = (int64_t)kCopyThreads * kSwapUnroll;
  for (int first = 0; first < num_pairs; first += 65535) {
    const int n = num_pairs - first < 65535 ? num_pairs - first : 65535;
    dim3 grid((unsigned)((chunks + per_cta - 1) / per_cta), (unsigned)n, 2);
    swap_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(dst_k, dst_v, dst_blocks, src_k, src_v,
                                                          src_blocks, block_pairs + 2 * (size_t)first,
                                                          chunks);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

bool swap_args_ok(const pa_swap_space *sp, const void *k_cache, const void *v_cache,
                  int num_blocks, const int64_t *block_pairs, int num_pairs) {
  return sp && num_pairs >= 0 && num_blocks > 0 &&
         (num_pairs == 0 || (k_cache && v_cache && block_pairs && aligned16(k_cache) &&
                             aligned16(v_cache) &&
                             (reinterpret_cast<uintptr_t>(block_pairs) & 7u) == 0));
}

}  // namespace

extern "C" {

pa_status pa_swap_out(const pa_swap_space *sp, const void *k_cache, const void *v_cache,
                      int num_blocks, const int64_t *block_pairs, int num_pairs, void *stream) {
  if (!swap_args_ok(sp, k_cache, v_cache, num_blocks, block_pairs, num_pairs)) return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  const int64_t chunks = (int64_t)sp->num_kv_heads * sp->block_size * sp->head_dim * 2 / 16;
  return launch_swap(sp->k_dev, sp->v_dev, sp->num_blocks, static_cast<const uint4 *>(k_cache),
                     static_cast<const uint4 *>(v_cache), num_blocks, block_pairs, num_pairs, chunks,
                     (cudaStream_t)stream);
}

pa_status pa_swap_in(const pa_swap_space *sp, void *k_cache, void *v_cache, int num_blocks,
                     const int64_t *block_pairs, int num_pairs, void *stream) {
  if (!swap_args_ok(sp, k_cache, v_cache, num_blocks, block_pairs, num_pairs)) return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  const int64_t chunks = (int64_t)sp->num_kv_heads * sp->block_size * sp->head_dim * 2 / 16;
  return launch_swap(static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), num_blocks,
                     sp->k_dev, sp->v_dev, sp->num_blocks, block_pairs, num_pairs, chunks,
                     (cudaStream_t)stream);
}

}  // extern "C"

// Read and clear this file's error word (stream-ordered; synchronises the stream).
pa_status pa_internal_cache_ops_status(cudaStream_t stream, int32_t *code) {
  int value = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&value, g_cache_ops_error, sizeof(int), 0,
                                cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_cache_ops_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                              stream) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return PA_ERR_CUDA;
  *code = value;
  return PA_OK;
}
