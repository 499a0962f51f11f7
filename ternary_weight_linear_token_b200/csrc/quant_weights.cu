// quant_weights.cu -- absmean ternary weight quantisation and 4-per-byte
// packing ("Microsoft BitNet 深度研究报告", 技术原理 item 2: Q(w) =
// round(clamp(w / gamma, -1, 1)), gamma = (1/n) sum |w_i|, stored value
// {0 -> 0, +1 -> 1, -1 -> 2}; BitNet b1.58 2B4T report write-up, GPU kernel
// section: four ternary weights per int8).
//
// Three kernels, all stream-ordered, no host synchronisation:
//   row_abs_sums  one thread per row sums |w| sequentially in k, in fp64
//                 (tiles staged through shared memory so loads coalesce);
//   gamma_finish  one thread sums the row sums sequentially in n (fp64) and
//                 writes gamma = (float)(sum / (N*K));
//   pack_codes    one thread per 16-element group: codes, one 32-bit word.
// The fixed summation order makes gamma bit-identical to the CPU oracle's,
// which matters because the rounding threshold |w| = gamma/2 depends on
// gamma's last bit.  This is an offline step (once per weight matrix).
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kRowsPerCta = 128;
constexpr int kTileK = 32;

template <int KIND>
__device__ __forceinline__ float load_w(const void *W, int64_t idx) {
  if (KIND == kF32) return static_cast<const float *>(W)[idx];
  const uint16_t b = static_cast<const uint16_t *>(W)[idx];
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

template <int KIND>
__global__ void __launch_bounds__(kRowsPerCta) row_abs_sums_kernel(const void *W, int64_t N,
                                                                   int64_t K, double *row_sums) {
  __shared__ float tile[kRowsPerCta][kTileK + 1];
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;
  const int tid = threadIdx.x;
  double acc = 0.0;
  for (int64_t k0 = 0; k0 < K; k0 += kTileK) {
    const int width = static_cast<int>(K - k0 < kTileK ? K - k0 : kTileK);
    // cooperative coalesced load: 32 consecutive k of one row per warp pass
    for (int e = tid; e < kRowsPerCta * kTileK; e += kRowsPerCta) {
      const int r = e / kTileK, c = e % kTileK;
      const int64_t n = row0 + r;
      tile[r][c] = (n < N && c < width) ? load_w<KIND>(W, n * K + k0 + c) : 0.0f;
    }
    __syncthreads();
    for (int c = 0; c < width; ++c) acc = __dadd_rn(acc, fabs(static_cast<double>(tile[tid][c])));
    __syncthreads();
  }
  const int64_t n = row0 + tid;
  if (n < N) row_sums[n] = acc;
}

__global__ void gamma_finish_kernel(const double *row_sums, int64_t N, int64_t K, float *gamma) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double total = 0.0;
  for (int64_t n = 0; n < N; ++n) total = __dadd_rn(total, row_sums[n]);
  const double mean = __ddiv_rn(total, static_cast<double>(N * K));
  *gamma = __double2float_rn(mean);
}

template <int KIND>
__global__ void __launch_bounds__(256) pack_codes_kernel(const void *W, int64_t N, int64_t K,
                                                          const float *gamma_ptr,
                                                          uint8_t *packed) {
  const int64_t groups_per_row = K / 16;
  const int64_t total = N * groups_per_row;
  const float gamma = *gamma_ptr;
  for (int64_t gidx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; gidx < total;
       gidx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = gidx / groups_per_row, g = gidx % groups_per_row;
    const int64_t base = n * K + 16 * g;
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      uint32_t code = 0;
      if (gamma != 0.0f) {
        float t = __fdiv_rn(load_w<KIND>(W, base + e), gamma);
        t = fminf(fmaxf(t, -1.0f), 1.0f);
        const float q = roundf(t);
        code = q > 0.0f ? 1u : (q < 0.0f ? 2u : 0u);
      }
      const int i = e & 3, j = e >> 2;
      word |= code << (8 * i + 2 * j);
    }
    reinterpret_cast<uint32_t *>(packed + n * (K / 4))[g] = word;
  }
}

}  // namespace

cudaError_t launch_quantize_weights(const void *W, int w_kind, int64_t N, int64_t K,
                                    uint8_t *packed, float *gamma, double *row_sums,
                                    const LaunchCtx &ctx) {
  const dim3 g1(static_cast<unsigned>(ceil_div(N, kRowsPerCta)));
  if (w_kind == kF32)
    row_abs_sums_kernel<kF32><<<g1, kRowsPerCta, 0, ctx.stream>>>(W, N, K, row_sums);
  else
    row_abs_sums_kernel<kBF16><<<g1, kRowsPerCta, 0, ctx.stream>>>(W, N, K, row_sums);
  gamma_finish_kernel<<<1, 32, 0, ctx.stream>>>(row_sums, N, K, gamma);
  const int64_t groups = N * (K / 16);
  const unsigned blocks =
      static_cast<unsigned>(ceil_div(groups, 256) < 8 * ctx.num_sms ? ceil_div(groups, 256)
                                                                     : 8 * ctx.num_sms);
  if (w_kind == kF32)
    pack_codes_kernel<kF32><<<blocks, 256, 0, ctx.stream>>>(W, N, K, gamma, packed);
  else
    pack_codes_kernel<kBF16><<<blocks, 256, 0, ctx.stream>>>(W, N, K, gamma, packed);
  return cudaGetLastError();
}

}  // namespace bitnet
