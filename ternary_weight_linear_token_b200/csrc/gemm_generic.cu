// gemm_generic.cu -- shape-general BitLinear contraction for what the fast
// kernels do not take: K % 64 != 0 (rows of packed bytes not 16-byte
// aligned), or very large K at decode sizes.  Activations arrive already
// quantised (int8 xq and per-token s).
//
// One warp per output feature n and per block of up to 16 tokens: lanes
// stride over the 32-bit packed words of row n, unpack each into four int8x4
// vectors in natural k order and accumulate xq . q with dp4a (the
// add/subtract identity of "Microsoft BitNet 深度研究报告", 技术原理 item 3,
// done as signed int8 products with q in {-1, 0, +1}); a shuffle reduction
// gives the exact int32 dot product, and lane 0 applies the epilogue.
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kWarps = 8;
constexpr int kTokens = 16;

template <int YK, bool RELU2>
__global__ void __launch_bounds__(32 * kWarps) generic_kernel(const int8_t *xq, const float *s,
                                                               const uint8_t *packed,
                                                               const float *gamma_ptr, int64_t M,
                                                               int64_t N, int64_t K, void *Y) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  // token blocks of kTokens, strided over gridDim.y (at most 65535 of them)
  for (int64_t m0 = static_cast<int64_t>(blockIdx.y) * kTokens; n < N && m0 < M;
       m0 += static_cast<int64_t>(gridDim.y) * kTokens) {
    const float gamma = *gamma_ptr;
    const uint32_t *row = reinterpret_cast<const uint32_t *>(packed + n * (K / 4));
    const int64_t words = K / 16;
    const int64_t m1 = (m0 + kTokens < M) ? m0 + kTokens : M;
    for (int64_t m = m0; m < m1; ++m) {
      const int *x = reinterpret_cast<const int *>(xq + m * K);
      int acc = 0;
      for (int64_t g = lane; g < words; g += 32) {
        const uint32_t w = row[g];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          acc = __dp4a(static_cast<int>(unpack_natural(w, j)), x[4 * g + j], acc);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        const size_t idx = static_cast<size_t>(m) * N + n;
        if (YK == kI32) {
          static_cast<int *>(Y)[idx] = acc;
        } else {
          const float y = epilogue_value(acc, __fdiv_rn(gamma, s[m]), RELU2);
          if (YK == kF32)
            static_cast<float *>(Y)[idx] = y;
          else
            static_cast<__nv_bfloat16 *>(Y)[idx] = __float2bfloat16_rn(y);
        }
      }
    }
  }
  pdl_launch_dependents();
}

template <int YK, bool RELU2>
cudaError_t go(const int8_t *xq, const float *s, const uint8_t *packed, const float *gamma,
               int64_t M, int64_t N, int64_t K, void *Y, const LaunchCtx &ctx) {
  const int64_t mblocks = ceil_div(M, kTokens);
  const dim3 grid(static_cast<unsigned>(ceil_div(N, kWarps)),
                  static_cast<unsigned>(mblocks < 65535 ? mblocks : 65535));
  return launch_k(generic_kernel<YK, RELU2>, grid, dim3(32 * kWarps), 0, ctx, xq, s, packed,
                  gamma, M, N, K, Y);
}

}  // namespace

cudaError_t launch_generic(const int8_t *xq, const float *s, const uint8_t *packed,
                           const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2,
                           void *Y, int y_kind, const LaunchCtx &ctx) {
  if (y_kind == kI32) return go<kI32, false>(xq, s, packed, gamma, M, N, K, Y, ctx);
  if (y_kind == kF32)
    return relu2 ? go<kF32, true>(xq, s, packed, gamma, M, N, K, Y, ctx)
                 : go<kF32, false>(xq, s, packed, gamma, M, N, K, Y, ctx);
  return relu2 ? go<kBF16, true>(xq, s, packed, gamma, M, N, K, Y, ctx)
               : go<kBF16, false>(xq, s, packed, gamma, M, N, K, Y, ctx);
}

}  // namespace bitnet
