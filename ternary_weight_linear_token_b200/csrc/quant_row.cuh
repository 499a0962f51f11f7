// quant_row.cuh -- one warp quantises one token row to int8 (per-token
// absmax, the BitNet b1.58 2B4T model card's 模型详情 -> 量化), and one warp
// expands packed ternary weights to int8; shared by the stand-alone
// quantiser kernels and the tensor-core kernel that quantises its own
// activations.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

// Load 16 consecutive activations (16-byte aligned) as fp32.
template <int KIND>
__device__ __forceinline__ void load16(const void *X, int64_t idx, float (&v)[16]) {
  if (KIND == kF32) {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(X) + idx);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = p[q];
      v[4 * q + 0] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  } else {
    const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(X) + idx);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 u = p[q];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        v[8 * q + 2 * h + 0] = __uint_as_float(w[h] << 16);
        v[8 * q + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
      }
    }
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// A bf16 row of up to 32 * kRegChunks 16-element chunks, one warp: the whole
// row is loaded into registers with every load issued up front, so it costs
// one round trip to memory, where the two-pass loop below costs one per pass
// and load round.
constexpr int kRegChunks = 6;
template <bool PERM>
__device__ __forceinline__ void quantize_row_resident(const uint4 *row, int chunks, int lane,
                                                      int8_t *out, float *s_out) {
  uint4 raw[kRegChunks][2];
#pragma unroll
  for (int i = 0; i < kRegChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < chunks) {
      raw[i][0] = row[2 * c];
      raw[i][1] = row[2 * c + 1];
    } else {
      raw[i][0] = raw[i][1] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  uint32_t amax_pair = 0;  // 16-bit SIMD max of |x| bit patterns (zeros past the row)
#pragma unroll
  for (int i = 0; i < kRegChunks; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      amax_pair = __vmaxu2(amax_pair, raw[i][j].x & 0x7FFF7FFFu);
      amax_pair = __vmaxu2(amax_pair, raw[i][j].y & 0x7FFF7FFFu);
      amax_pair = __vmaxu2(amax_pair, raw[i][j].z & 0x7FFF7FFFu);
      amax_pair = __vmaxu2(amax_pair, raw[i][j].w & 0x7FFF7FFFu);
    }
  const uint32_t amax_bits = max(amax_pair & 0xFFFFu, amax_pair >> 16) << 16;
  const float sm = act_scale(warp_max(__uint_as_float(amax_bits)));
#pragma unroll
  for (int i = 0; i < kRegChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < chunks) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t w[4] = {raw[i][j].x, raw[i][j].y, raw[i][j].z, raw[i][j].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          v[8 * j + 2 * h] = __uint_as_float(w[h] << 16);
          v[8 * j + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
        }
      }
      int q[16];
      quant16(v, sm, q);
      *reinterpret_cast<uint4 *>(out + 16 * c) =
          PERM ? pack_permuted(q)
               : make_uint4(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]),
                            pack4(q[8], q[9], q[10], q[11]), pack4(q[12], q[13], q[14], q[15]));
    }
  }
  if (lane == 0) *s_out = sm;
}

// Any row (fp32 or bf16, any K % 16 == 0): two passes, 16-element steps
// per lane with several steps' raw words in registers at a time.
template <int KIND, bool PERM>
__device__ __forceinline__ void quantize_row_general(const void *X, int64_t m, int64_t K, int lane,
                                                     int8_t *xq, float *s) {
  // 16-element steps per lane per round: the raw words stay in registers
  constexpr int kInFlight = KIND == kF32 ? 2 : 4;
  constexpr int kWords = KIND == kF32 ? 4 : 2;  // uint4 per 16 elements
  const int64_t chunks = K / 16;
  const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(X) +
                                                    m * K * (KIND == kF32 ? 4 : 2));
  // max |x| on the bit patterns: |x| of a float (or of a bf16) orders as
  // an unsigned integer; bf16 pairs go through the 16-bit SIMD max
  uint32_t amax_bits = 0, amax_pair = 0;
  for (int64_t c0 = lane; c0 < chunks; c0 += 32 * kInFlight) {
    uint4 raw[kInFlight][kWords];
#pragma unroll
    for (int i = 0; i < kInFlight; ++i)
      if (c0 + 32 * i < chunks) {
#pragma unroll
        for (int j = 0; j < kWords; ++j) raw[i][j] = row[(c0 + 32 * i) * kWords + j];
      }
#pragma unroll
    for (int i = 0; i < kInFlight; ++i)
      if (c0 + 32 * i < chunks) {
#pragma unroll
        for (int j = 0; j < kWords; ++j) {
          const uint32_t w[4] = {raw[i][j].x, raw[i][j].y, raw[i][j].z, raw[i][j].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (KIND == kF32)
              amax_bits = max(amax_bits, w[h] & 0x7FFFFFFFu);
            else
              amax_pair = __vmaxu2(amax_pair, w[h] & 0x7FFF7FFFu);
          }
        }
      }
  }
  if (KIND != kF32) amax_bits = max(amax_pair & 0xFFFFu, amax_pair >> 16) << 16;
  const float amax = warp_max(__uint_as_float(amax_bits));
  const float sm = act_scale(amax);
  for (int64_t c0 = lane; c0 < chunks; c0 += 32 * kInFlight) {
    uint4 raw[kInFlight][kWords];
#pragma unroll
    for (int i = 0; i < kInFlight; ++i)
      if (c0 + 32 * i < chunks) {
#pragma unroll
        for (int j = 0; j < kWords; ++j) raw[i][j] = row[(c0 + 32 * i) * kWords + j];
      }
#pragma unroll
    for (int i = 0; i < kInFlight; ++i) {
      const int64_t c = c0 + 32 * i;
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
        quant16(v, sm, q);
        *reinterpret_cast<uint4 *>(xq + m * K + 16 * c) =
            PERM ? pack_permuted(q)
                 : make_uint4(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]),
                              pack4(q[8], q[9], q[10], q[11]), pack4(q[12], q[13], q[14], q[15]));
      }
    }
  }
  if (lane == 0) s[m] = sm;
}

// Row m of X [M][K] -> xq row m and s[m], by one warp.
template <int KIND, bool PERM>
__device__ __forceinline__ void quantize_row_warp(const void *X, int64_t m, int64_t K, int lane,
                                                  int8_t *xq, float *s) {
  if (KIND == kBF16 && K <= 32 * 16 * kRegChunks)
    quantize_row_resident<PERM>(
        reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(X) + m * K),
        static_cast<int>(K / 16), lane, xq + m * K, s + m);
  else
    quantize_row_general<KIND, PERM>(X, m, K, lane, xq, s);
}

// Packed weight row n ([K/16] words) -> int8 row n ([K] bytes), by one warp:
// 4-byte loads and 16-byte stores, contiguous across the warp.
template <bool PERM>
__device__ __forceinline__ void expand_row_warp(const uint8_t *packed, int8_t *w8, int64_t n,
                                                int64_t K, int lane) {
  const uint32_t *src = reinterpret_cast<const uint32_t *>(packed + n * (K / 4));
  uint4 *dst = reinterpret_cast<uint4 *>(w8 + n * K);
  const int words = static_cast<int>(K / 16);
  for (int w0 = lane; w0 < words; w0 += 32 * 4) {
    uint32_t v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = w0 + 32 * j < words ? src[w0 + 32 * j] : 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (w0 + 32 * j < words) dst[w0 + 32 * j] = expand_word<PERM>(v[j]);
  }
}

}  // namespace
}  // namespace bitnet
