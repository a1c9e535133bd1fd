// pa_measure.cu -- a read-only HBM stream, to measure the rate this GPU reads memory at.
//
// Not part of the method: decode is bound by reading K/V from HBM, and its roofline
// fraction is stated against a copy's rate. This kernel gives the read-only rate beside
// it: every thread streams 16-byte loads (four in flight, evict-first) over a buffer
// larger than L2, folds them into an XOR so the loads are not dropped, and each warp
// XORs its result into one word.

#include <cuda_runtime.h>

#include <cstdint>

#include "pa.h"

namespace {

constexpr int kReadThreads = 512;

__global__ void __launch_bounds__(kReadThreads) hbm_read_kernel(const uint4 *__restrict__ buf,
                                                                size_t n16, uint32_t *sink) {
  const size_t stride = (size_t)gridDim.x * kReadThreads;
  size_t i = (size_t)blockIdx.x * kReadThreads + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = __ldcs(buf + i), b = __ldcs(buf + i + stride);
    const uint4 c = __ldcs(buf + i + 2 * stride), d = __ldcs(buf + i + 3 * stride);
    acc ^= (a.x ^ a.y ^ a.z ^ a.w) ^ (b.x ^ b.y ^ b.z ^ b.w) ^ (c.x ^ c.y ^ c.z ^ c.w) ^
           (d.x ^ d.y ^ d.z ^ d.w);
  }
  for (; i < n16; i += stride) {
    const uint4 a = __ldcs(buf + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
  for (int off = 16; off >= 1; off >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

}  // namespace

extern "C" pa_status pa_hbm_read(const void *buf, size_t bytes, uint32_t *sink, int ctas_per_sm,
                                 void *stream) {
  if (!buf || !sink || bytes == 0 || bytes % 16 || ctas_per_sm <= 0 || ctas_per_sm > 4 ||
      (reinterpret_cast<uintptr_t>(buf) & 15) || (reinterpret_cast<uintptr_t>(sink) & 3))
    return PA_ERR_INVALID;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(sink, 0, sizeof(uint32_t), st) != cudaSuccess) return PA_ERR_CUDA;
  hbm_read_kernel<<<sms * ctas_per_sm, kReadThreads, 0, st>>>(static_cast<const uint4 *>(buf),
                                                             bytes / 16, sink);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
