// noalloc.cu -- bitnet_w158a8_matmul for callers that cannot allocate
// device memory.
//
// Some callers cannot give the library a workspace: a plugin inside a host
// framework that owns all device memory and hands out none, or a serving
// loop that must never call cudaMalloc because cudaMalloc can block until
// the whole device is idle.  For them this file keeps one scratch array in
// the library itself, a file-scope __device__ array of a fixed size, and
// runs the regular product with it as the workspace.  Nothing is allocated
// at any point.
//
// The array exists once per GPU that loads the library and stays until the
// process exits.  Every call on a device shares it and leaves its contents
// behind; no part of it has to start at zero, because each call overwrites
// the part it reads (the quantised activations and their scales) before
// reading it.  Calls whose kernels overlap on the GPU race on the array.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/bitnet158.h"
#include "internal.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[BITNET_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device.  Host code
// cannot use the array's name as a device pointer (on the host it names a
// stand-in, not device memory), so the address is looked up once per device,
// with that device current, and cached.
bitnet_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BITNET_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
      return BITNET_ERR_CUDA;
    g_scratch_addr[dev] = addr;
  }
  *out = g_scratch_addr[dev];
  return BITNET_OK;
}

}  // namespace

extern "C" bitnet_status bitnet_w158a8_matmul_noalloc(const void *X, bitnet_dtype x_dtype,
                                                      const float *s, const uint8_t *packed,
                                                      const float *gamma, int64_t M, int64_t N,
                                                      int64_t K, bitnet_epilogue epi, void *Y,
                                                      bitnet_dtype y_dtype, uint32_t flags,
                                                      bitnet_stream_t stream) {
  // The regular argument checks first (a bad dtype, flag or size is an
  // invalid argument, whatever scratch it would need), then the size limit;
  // both before anything touches the device.
  if (const int st = bitnet::matmul_args_status(X, x_dtype, s, packed, gamma, M, N, K, epi, Y,
                                                y_dtype, flags))
    return static_cast<bitnet_status>(st);
  if (M > 0 && N > 0 &&
      bitnet_w158a8_matmul_workspace_size(M, N, K, x_dtype) > BITNET_STATIC_SCRATCH_BYTES)
    return BITNET_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (M > 0 && N > 0) {
    if (bitnet_status st = scratch_address(&scratch)) return st;
  }
  return bitnet_w158a8_matmul(X, x_dtype, s, packed, gamma, M, N, K, epi, Y, y_dtype, scratch,
                              BITNET_STATIC_SCRATCH_BYTES, flags, stream);
}
