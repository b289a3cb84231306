// Copies between page-locked host buffers and the workspace for the host-buffer entry points.
//
// A decode step moves a few KB each way; as copy-engine transfers those cost several microseconds
// of latency apiece on the stream and break the overlap of consecutive launches. Page-locked host
// memory is addressable from the device (unified addressing), so small transfers run as a kernel
// instead, launched like the layer kernels (programmatic stream serialization): the copy in
// requests its host data before waiting for the previous kernel, the copy out starts right behind
// the layer. The caller uses this only for buffers the runtime reports as device-mapped host
// memory; anything else goes through cudaMemcpyAsync.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kIoThreads = 256;
constexpr int kIoPer = 4;  // 16-byte words per thread

// dst[i] = src[i] for n 16-byte words. `early`: the source (host data) is read before the wait for
// the previous kernel, the destination written after it.
__global__ void __launch_bounds__(kIoThreads) io_copy_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                            size_t n, int early) {
  const size_t i0 = (size_t)blockIdx.x * kIoThreads * kIoPer + threadIdx.x;
  uint4 v[kIoPer];
  if (early) {
#pragma unroll
    for (int j = 0; j < kIoPer; ++j) {
      const size_t i = i0 + (size_t)j * kIoThreads;
      if (i < n) v[j] = src[i];
    }
  }
  pdl_launch_dependents();
  pdl_wait();
  if (!early) {
#pragma unroll
    for (int j = 0; j < kIoPer; ++j) {
      const size_t i = i0 + (size_t)j * kIoThreads;
      if (i < n) v[j] = src[i];
    }
  }
#pragma unroll
  for (int j = 0; j < kIoPer; ++j) {
    const size_t i = i0 + (size_t)j * kIoThreads;
    if (i < n) dst[i] = v[j];
  }
}

}  // namespace

cudaError_t launch_io_copy(const void *src, void *dst, size_t bytes, bool early, cudaStream_t s) {
  const size_t n = bytes / 16;
  if (n == 0) return cudaSuccess;
  const size_t per_block = (size_t)kIoThreads * kIoPer;
  const unsigned blocks = (unsigned)((n + per_block - 1) / per_block);
  return launch_pdl(io_copy_kernel, dim3(blocks), dim3(kIoThreads), 0, s, static_cast<const uint4 *>(src),
                    static_cast<uint4 *>(dst), n, early ? 1 : 0);
}

}  // namespace moe
