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

// TMA tensor map over a K or V pool viewed as [num_blocks * num_kv_heads *
// block_size rows][head_dim], boxes of 64 columns x box_rows rows, 128-byte
// swizzle (encoded once per pool and cached).
bool pa_internal_pool_tensor_map(CUtensorMap *map, const void *base, long long rows, int head_dim,
                                 int box_rows, pa_dtype dtype);
