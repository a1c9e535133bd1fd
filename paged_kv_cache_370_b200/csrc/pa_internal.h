// pa_internal.h -- declarations shared between the library's own source files
// (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pa.h"

// Read and clear the device error word of each kernel file (synchronises `stream`).
pa_status pa_internal_cache_ops_status(cudaStream_t stream, int32_t *code);
pa_status pa_internal_decode_status(cudaStream_t stream, int32_t *code);
pa_status pa_internal_prefill_status(cudaStream_t stream, int32_t *code);

// Bytes at the start of a decode workspace that hold the even-split kernel's
// per-CTA counters (zero before a call; a completed call leaves them zero).
constexpr size_t kPaCounterRegionBytes = 64 * 1024;

// Workspace bytes a pa_decode call with these arguments needs for the kernel
// it runs (0: none, or invalid arguments -- pa_decode itself reports those).
size_t pa_internal_decode_need(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int num_blocks, int max_context_len,
                               int partition_tokens);

// TMA tensor map over a K or V pool viewed as [num_blocks * num_kv_heads *
// block_size rows][head_dim], boxes of 64 columns x box_rows rows, 128-byte
// swizzle (encoded once per pool and cached).
bool pa_internal_pool_tensor_map(CUtensorMap *map, const void *base, long long rows, int head_dim,
                                 int box_rows, pa_dtype dtype);
