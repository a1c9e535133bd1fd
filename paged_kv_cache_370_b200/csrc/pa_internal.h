// pa_internal.h -- declarations shared between the library's own source files
// (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "pa.h"

// Read and clear the device error word of each kernel file (synchronises `stream`).
pa_status pa_internal_cache_ops_status(cudaStream_t stream, int32_t *code);
pa_status pa_internal_decode_status(cudaStream_t stream, int32_t *code);
