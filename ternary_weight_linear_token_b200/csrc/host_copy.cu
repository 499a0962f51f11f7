// host_copy.cu -- small copies between page-locked host memory and the device
// for the host-to-host entry points.
//
// A copy-engine transfer of a few KB costs several microseconds of setup and
// completion, more than the decode product it feeds.  A single CTA that
// moves the bytes in 16-byte pieces through the unified address space
// (page-locked memory is device-addressable at its host address) starts
// like any kernel and, launched with programmatic dependent launch, lets the
// product that follows start its weight prefetch while the activations are
// still on their way.
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kCopyThreads = 512;

// dst[i] = src[i] for i < n (16-byte pieces).  Waits for the previous grid
// in the stream first: it may still read dst (the previous product reads
// X_dev) or write src (the product writes Y_dev).
__global__ void __launch_bounds__(kCopyThreads) copy16_kernel(const uint4 *src, uint4 *dst,
                                                              int64_t n) {
  pdl_wait();
  pdl_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * kCopyThreads)
    dst[i] = src[i];
}

}  // namespace

bool small_copy_ok(const void *host, const void *dev, size_t bytes) {
  if (bytes == 0 || bytes > kSmallCopyMax || bytes % 16 != 0) return false;
  if ((reinterpret_cast<uintptr_t>(host) | reinterpret_cast<uintptr_t>(dev)) % 16 != 0) return false;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost && a.devicePointer == host;
}

cudaError_t launch_small_copy(const void *src, void *dst, size_t bytes, const LaunchCtx &ctx) {
  const int64_t n = static_cast<int64_t>(bytes / 16);
  const int64_t blocks = (n + kCopyThreads - 1) / kCopyThreads;
  return launch_k(copy16_kernel, dim3(static_cast<unsigned>(blocks < 8 ? blocks : 8)),
                  dim3(kCopyThreads), 0, ctx, static_cast<const uint4 *>(src),
                  static_cast<uint4 *>(dst), n);
}

}  // namespace bitnet
