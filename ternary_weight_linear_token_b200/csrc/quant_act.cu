// quant_act.cu -- per-token absmax int8 activation quantisation (BitNet
// b1.58 2B4T model card, 模型详情 -> 量化: activations to 8-bit integers with
// per-token absmax), and the weightless RMS normalisation used as glue
// between chained BitLinears (the card's "subln", formula not given).
//
// One warp per token row, 8 rows per CTA: the row's max |x| is reduced with
// warp shuffles (max is order-independent, so it is exact), then
// s = 127 / amax and xq = clamp(round_half_away(x * s), -127, 127).  The
// second pass re-reads the row, which is still in L1.  16 elements (one
// 16-byte int8 output chunk) per lane-step, four steps per lane in flight at
// a time (a K = 2560 row is two dependent rounds of loads, not five);
// K % 16 == 0.
//
// On the tensor-core path the same launch also expands the packed weights
// into int8 scratch: blocks past the quantiser's take 1024 packed words each.
// The quantiser is bound by its FMA/ALU issue, so the expansion's memory
// traffic (4.4 MB in, 17.7 MB out for 6912 x 2560) runs beside it instead of
// as a launch of its own.
#include "common.cuh"
#include "internal.h"
#include "quant_row.cuh"

namespace bitnet {
namespace {

constexpr int kRowsPerCta = 8;

constexpr int kExpandWords = 4;  // packed words per thread
constexpr int64_t kExpandBlockWords = 32 * kRowsPerCta * kExpandWords;

// Packed word w (16 weights) -> bytes 16w..16w+15 of the int8 weights: the
// packed matrix [N][K/16 words] and the int8 one [N][K] share their row
// order, so the flat word index maps straight through.  A warp handles 128
// consecutive words: 4-byte loads and 16-byte stores, contiguous across it.
template <bool PERM>
__device__ __forceinline__ void expand_block(const ExpandJob &job, int64_t block) {
  const uint32_t *packed = reinterpret_cast<const uint32_t *>(job.packed);
  uint4 *w8 = reinterpret_cast<uint4 *>(job.w8);
  const int64_t base = block * kExpandBlockWords + (threadIdx.x >> 5) * (32 * kExpandWords) +
                       (threadIdx.x & 31);
  uint32_t w[kExpandWords];
#pragma unroll
  for (int j = 0; j < kExpandWords; ++j) {
    const int64_t i = base + 32 * j;
    w[j] = i < job.words ? packed[i] : 0u;
  }
#pragma unroll
  for (int j = 0; j < kExpandWords; ++j) {
    const int64_t i = base + 32 * j;
    if (i < job.words) w8[i] = expand_word<PERM>(w[j]);
  }
}

template <bool PERM>
__global__ void __launch_bounds__(32 * kRowsPerCta) expand_weights_kernel(const ExpandJob job) {
  pdl_launch_dependents();
  pdl_wait();  // the previous product may still be reading the scratch
  expand_block<PERM>(job, blockIdx.x);
}

// Blocks [0, qblocks) quantise 8 token rows each; later blocks expand the
// weights of `job` (none when job.words == 0).
template <int KIND, bool PERM>
__global__ void __launch_bounds__(32 * kRowsPerCta) quantize_act_kernel(const void *X, int64_t M,
                                                                         int64_t K, int8_t *xq,
                                                                         float *s,
                                                                         const ExpandJob job,
                                                                         int qblocks) {
  // Let the next kernel (the product that reads xq) launch now: its CTAs can
  // set up and prefetch their weights while this grid runs; its own
  // grid-dependency wait still lasts until this grid has completed.
  pdl_launch_dependents();
  pdl_wait();
  if (static_cast<int>(blockIdx.x) >= qblocks) {
    expand_block<PERM>(job, static_cast<int64_t>(blockIdx.x) - qblocks);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t m = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + (threadIdx.x >> 5);
  if (m < M) quantize_row_warp<KIND, PERM>(X, m, K, lane, xq, s);
}

// Few tokens: one CTA per row, 8 warps splitting it, so that a long row is
// not one warp's chain of dependent loads.  Each thread keeps at most
// kRowChunks 16-element chunks in registers (K <= 8 * 32 * 16 * kRowChunks);
// max |x| is reduced over the warps in shared memory.
constexpr int kRowChunks = 2;
constexpr int kRowThreads = 256;
constexpr int64_t kRowMaxK = int64_t(kRowThreads) * 16 * kRowChunks;

template <int KIND, bool PERM>
__global__ void __launch_bounds__(kRowThreads) quantize_row_kernel(const void *X, int64_t K,
                                                                   int8_t *xq, float *s) {
  __shared__ float wmax[kRowThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t m = blockIdx.x;
  constexpr int kWords = KIND == kF32 ? 4 : 2;  // uint4 per 16 elements
  const int64_t chunks = K / 16;
  const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(X) +
                                                    m * K * (KIND == kF32 ? 4 : 2));
  uint4 raw[kRowChunks][kWords];
  uint32_t amax_bits = 0;  // |x| of a float (or of a bf16) orders as an unsigned integer
#pragma unroll
  for (int i = 0; i < kRowChunks; ++i) {
    const int64_t c = tid + int64_t(i) * kRowThreads;
    if (c < chunks) {
#pragma unroll
      for (int j = 0; j < kWords; ++j) raw[i][j] = row[c * kWords + j];
    }
  }
#pragma unroll
  for (int i = 0; i < kRowChunks; ++i) {
    if (tid + int64_t(i) * kRowThreads < chunks) {
#pragma unroll
      for (int j = 0; j < kWords; ++j) {
        const uint32_t w[4] = {raw[i][j].x, raw[i][j].y, raw[i][j].z, raw[i][j].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          if (KIND == kF32) {
            amax_bits = max(amax_bits, w[h] & 0x7FFFFFFFu);
          } else {
            amax_bits = max(amax_bits, (w[h] & 0x7FFFu) << 16);
            amax_bits = max(amax_bits, w[h] & 0x7FFF0000u);
          }
        }
      }
    }
  }
  amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
  if (lane == 0) wmax[warp] = __uint_as_float(amax_bits);
  __syncthreads();
  float amax = wmax[0];
#pragma unroll
  for (int i = 1; i < kRowThreads / 32; ++i) amax = fmaxf(amax, wmax[i]);
  const float sm = act_scale(amax);
#pragma unroll
  for (int i = 0; i < kRowChunks; ++i) {
    const int64_t c = tid + int64_t(i) * kRowThreads;
    if (c < chunks) {
      float v[16];
#pragma unroll
      for (int j = 0; j < kWords; ++j) {
        const uint32_t w[4] = {raw[i][j].x, raw[i][j].y, raw[i][j].z, raw[i][j].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          if (KIND == kF32) {
            v[4 * j + h] = __uint_as_float(w[h]);
          } else {
            v[8 * j + 2 * h] = __uint_as_float(w[h] << 16);
            v[8 * j + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
          }
        }
      }
      int q[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) q[e] = quant_i8(v[e], sm);
      *reinterpret_cast<uint4 *>(xq + m * K + 16 * c) =
          PERM ? pack_permuted(q)
               : make_uint4(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]),
                            pack4(q[8], q[9], q[10], q[11]), pack4(q[12], q[13], q[14], q[15]));
    }
  }
  if (tid == 0) s[m] = sm;
}

template <int XK, int YK>
__global__ void __launch_bounds__(32 * kRowsPerCta) rms_norm_kernel(const void *X, int64_t M,
                                                                     int64_t K, void *Y) {
  pdl_launch_dependents();  // the next kernel may set up while this one runs
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t m = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + (threadIdx.x >> 5);
  if (m < M) {
    const int64_t chunks = K / 16;
    double ss = 0.0;
    for (int64_t c = lane; c < chunks; c += 32) {
      float v[16];
      load16<XK>(X, m * K + 16 * c, v);
#pragma unroll
      for (int e = 0; e < 16; ++e) ss = add_sq(ss, v[e]);
    }
    const float inv = rms_factor(warp_sum_f64(ss), K);
    for (int64_t c = lane; c < chunks; c += 32) {
      float v[16];
      load16<XK>(X, m * K + 16 * c, v);
      if (YK == kF32) {
        float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(Y) + m * K + 16 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          p[q] = make_float4(v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv,
                             v[4 * q + 3] * inv);
      } else {
        uint32_t o[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * h] * inv, v[2 * h + 1] * inv);
          o[h] = *reinterpret_cast<const uint32_t *>(&b);
        }
        uint4 *p = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(Y) + m * K + 16 * c);
        p[0] = make_uint4(o[0], o[1], o[2], o[3]);
        p[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_expand_weights(const ExpandJob &job, bool permuted, const LaunchCtx &ctx) {
  if (job.words <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(ceil_div(job.words, kExpandBlockWords)));
  const dim3 block(32 * kRowsPerCta);
  return permuted ? launch_k(expand_weights_kernel<true>, grid, block, 0, ctx, job)
                  : launch_k(expand_weights_kernel<false>, grid, block, 0, ctx, job);
}

cudaError_t launch_quantize_act(const void *X, int x_kind, int64_t M, int64_t K, int8_t *xq,
                                float *s, bool permuted, const LaunchCtx &ctx,
                                const ExpandJob &expand) {
  if (M <= ctx.num_sms && K <= kRowMaxK) {  // few tokens: one CTA per row
    const dim3 grid(static_cast<unsigned>(M)), block(kRowThreads);
    cudaError_t e;
    if (x_kind == kF32)
      e = permuted ? launch_k(quantize_row_kernel<kF32, true>, grid, block, 0, ctx, X, K, xq, s)
                   : launch_k(quantize_row_kernel<kF32, false>, grid, block, 0, ctx, X, K, xq, s);
    else
      e = permuted ? launch_k(quantize_row_kernel<kBF16, true>, grid, block, 0, ctx, X, K, xq, s)
                   : launch_k(quantize_row_kernel<kBF16, false>, grid, block, 0, ctx, X, K, xq, s);
    if (e != cudaSuccess) return e;
    return launch_expand_weights(expand, permuted, ctx);
  }
  const int64_t qblocks = ceil_div(M, kRowsPerCta);
  const int64_t eblocks = expand.words > 0 ? ceil_div(expand.words, kExpandBlockWords) : 0;
  const dim3 grid(static_cast<unsigned>(qblocks + eblocks));
  const dim3 block(32 * kRowsPerCta);
  const int qb = static_cast<int>(qblocks);
  if (x_kind == kF32)
    return permuted ? launch_k(quantize_act_kernel<kF32, true>, grid, block, 0, ctx, X, M, K, xq, s, expand, qb)
                    : launch_k(quantize_act_kernel<kF32, false>, grid, block, 0, ctx, X, M, K, xq, s, expand, qb);
  return permuted ? launch_k(quantize_act_kernel<kBF16, true>, grid, block, 0, ctx, X, M, K, xq, s, expand, qb)
                  : launch_k(quantize_act_kernel<kBF16, false>, grid, block, 0, ctx, X, M, K, xq, s, expand, qb);
}

cudaError_t launch_rms_norm(const void *X, int x_kind, int64_t M, int64_t K, void *Y, int y_kind,
                            const LaunchCtx &ctx) {
  const dim3 grid(static_cast<unsigned>(ceil_div(M, kRowsPerCta)));
  const dim3 block(32 * kRowsPerCta);
  if (x_kind == kF32 && y_kind == kF32)
    return launch_k(rms_norm_kernel<kF32, kF32>, grid, block, 0, ctx, X, M, K, Y);
  if (x_kind == kF32)
    return launch_k(rms_norm_kernel<kF32, kBF16>, grid, block, 0, ctx, X, M, K, Y);
  if (y_kind == kF32)
    return launch_k(rms_norm_kernel<kBF16, kF32>, grid, block, 0, ctx, X, M, K, Y);
  return launch_k(rms_norm_kernel<kBF16, kBF16>, grid, block, 0, ctx, X, M, K, Y);
}

}  // namespace bitnet
