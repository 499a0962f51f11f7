// gemv_decode.cu -- fused BitLinear forward for decode-sized batches
// (M <= 32 tokens).  This regime is bound by HBM bandwidth on the packed
// weights: 2 bits per weight, four per byte (BitNet b1.58 2B4T report
// write-up, GPU kernel section: "pack, store, load, unpack, compute").
//
// One CTA owns 16 output features (rows of the packed matrix) over the full
// K.  Its 16 x K/4 packed bytes are contiguous in HBM and arrive by 16 bulk
// copies (one per row, into padded shared-memory rows), issued before the
// grid-dependency wait when the caller promises the weights are static, so
// they stream while the previous kernel in the stream finishes.  After the
// wait the CTA quantises the activations per token (s = 127 / max|x|,
// round half away, clamp +-127 -- identical to bitnet_quantize_act) into
// shared memory: one token is spread over all 8 warps (each element loaded
// once, amax reduced across the block), several tokens go one per warp.
// Then the 8 warps split K into 64-element steps (balanced to within one
// step) and run int8 mma.sync m16n8k32: A = 16 weight rows x 32 k (unpacked
// from 2-bit codes in registers), B = 32 k x 8 tokens, two independent
// accumulator chains per warp.  Accumulation is exact int32; the warps are
// reduced in shared memory and the epilogue applies gamma / s and the
// optional ReLU^2.
//
// Unpack: a 32-bit packed word holds element 16g + 4j + i at bits 8i + 2j.
// Shifting the word by 0, 2, 16 or 18 and masking with 0x3333 puts four
// 2-bit codes in the low bits of the four selector nibbles of a byte
// permute, which looks them up in the constant {0, +1, -1, -1}: four int8
// weights for 3 instructions.  The four elements a shift selects are
// {0,8,1,9}, {4,12,5,13}, {2,10,3,11}, {6,14,7,15}; the dot product does not
// depend on the order of k, so the activations are stored in shared memory
// in that same order (one 16-byte chunk per packed word, words in order).
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kRows = 16;
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kSmemLimit = 227 * 1024;

struct DecodeParams {
  const void *X;
  const float *s_in;
  const uint8_t *packed;
  const float *gamma;
  void *Y;
  int *status;
  int M, N, K;
  int ws;  // shared-memory stride of a weight row (bytes)
  int xs;  // shared-memory stride of a token row (bytes)
  int tg;  // tokens per group held in shared memory
  int weights_static;
};

// Smallest b >= bytes with b % 16 == 0 and b % 128 == r.
__host__ __device__ constexpr int pad_to(int bytes, int r) {
  const int b = (bytes + 15) & ~15;
  return b + (((r - b % 128) % 128) + 128) % 128;
}
// Weight rows 16 mod 128 bytes apart: the 8 rows x 4 consecutive words a warp
// reads per step land on 32 distinct banks.  Token rows 64 mod 128 apart:
// the two tokens x 4 chunks of a quarter-warp's 16-byte reads do too.
int weight_row_bytes(int K) { return pad_to(K / 4, 16); }
int token_row_bytes(int K) { return pad_to(K, 64); }

__host__ __device__ constexpr int red_bytes(int mt) { return kWarps * mt * 32 * 16; }
constexpr int kHeader = 256;  // mbarrier, per-token scales, amax partials

size_t smem_bytes(int mt, int K) {
  return kHeader + red_bytes(mt) + static_cast<size_t>(kRows) * weight_row_bytes(K) +
         static_cast<size_t>(8 * mt) * token_row_bytes(K);
}

__device__ __forceinline__ uint32_t unpack_sel(uint32_t w, int shift) {
  return __byte_perm(kTernaryLut, 0u, (w >> shift) & 0x3333u);
}

__device__ __forceinline__ void mma_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int KIND>
__device__ __forceinline__ void load16(const void *X, size_t idx, float (&v)[16]) {
  if (KIND == kF32) {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(X) + idx);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = p[q];
      v[4 * q] = f.x;
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
        v[8 * q + 2 * h] = __uint_as_float(w[h] << 16);
        v[8 * q + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
      }
    }
  }
}

template <int YK, bool RELU2>
__device__ __forceinline__ void emit(const DecodeParams &p, int n, int m, int acc, float r) {
  const size_t o = static_cast<size_t>(m) * p.N + n;
  if (YK == kI32) {
    static_cast<int *>(p.Y)[o] = acc;
  } else {
    const float y = epilogue_value(acc, r, RELU2);
    if (YK == kF32)
      static_cast<float *>(p.Y)[o] = y;
    else
      static_cast<__nv_bfloat16 *>(p.Y)[o] = __float2bfloat16_rn(y);
  }
}

// One token quantised by the whole block: each 16-element chunk is loaded
// once (up to kCache chunks per thread stay in registers for the second
// use), the row's max |x| is reduced across the 8 warps.
template <int XK>
__device__ __forceinline__ float quantize_token_block(const DecodeParams &p, int m, uint8_t *xrow,
                                                      float *amax_sh) {
  constexpr int kCache = 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int words = p.K / 16;
  const size_t base = static_cast<size_t>(m) * p.K;
  float v[kCache][16];
  float amax = 0.0f;
#pragma unroll
  for (int c = 0; c < kCache; ++c) {
    const int w = tid + c * kThreads;
    if (w < words) {
      load16<XK>(p.X, base + 16 * w, v[c]);
#pragma unroll
      for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[c][e]));
    }
  }
  for (int w = tid + kCache * kThreads; w < words; w += kThreads) {
    float t[16];
    load16<XK>(p.X, base + 16 * w, t);
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(t[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) amax_sh[warp] = amax;
  __syncthreads();
  amax = amax_sh[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) amax = fmaxf(amax, amax_sh[i]);
  const float sm = act_scale(amax);
#pragma unroll
  for (int c = 0; c < kCache; ++c) {
    const int w = tid + c * kThreads;
    if (w < words) {
      int q[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) q[e] = quant_i8(v[c][e], sm);
      *reinterpret_cast<uint4 *>(xrow + 16 * w) = pack_permuted(q);
    }
  }
  for (int w = tid + kCache * kThreads; w < words; w += kThreads) {
    float t[16];
    load16<XK>(p.X, base + 16 * w, t);
    int q[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) q[e] = quant_i8(t[e], sm);
    *reinterpret_cast<uint4 *>(xrow + 16 * w) = pack_permuted(q);
  }
  return sm;
}

// One token quantised by one warp (used when the group has several tokens).
template <int XK>
__device__ __forceinline__ float quantize_token_warp(const DecodeParams &p, int m, uint8_t *xrow) {
  const int lane = threadIdx.x & 31;
  const int words = p.K / 16;
  const size_t base = static_cast<size_t>(m) * p.K;
  float amax = 0.0f;
  for (int w = lane; w < words; w += 32) {
    float t[16];
    load16<XK>(p.X, base + 16 * w, t);
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(t[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float sm = act_scale(amax);
  for (int w = lane; w < words; w += 32) {
    float t[16];
    load16<XK>(p.X, base + 16 * w, t);
    int q[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) q[e] = quant_i8(t[e], sm);
    *reinterpret_cast<uint4 *>(xrow + 16 * w) = pack_permuted(q);
  }
  return sm;
}

template <int MT, int XK, int YK, bool RELU2>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
  float *s_sh = reinterpret_cast<float *>(smem + 16);      // 32 per-token scales
  float *amax_sh = reinterpret_cast<float *>(smem + 160);  // kWarps partial maxima
  int4 *red = reinterpret_cast<int4 *>(smem + kHeader);
  uint8_t *wsh = smem + kHeader + red_bytes(MT);
  uint8_t *xsh = wsh + kRows * p.ws;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kRows;
  const int rows = min(kRows, p.N - n0);
  const uint32_t row_bytes = static_cast<uint32_t>(p.K) / 4;
  const int words = p.K / 16;
  const int steps = words / 4;  // 64-element steps (K % 64 == 0)
  const int st0 = warp * steps / kWarps, st1 = (warp + 1) * steps / kWarps;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (p.weights_static && warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar, rows * row_bytes);
    __syncwarp();
    if (lane < rows)
      bulk_g2s(wsh + lane * p.ws, p.packed + static_cast<size_t>(n0 + lane) * row_bytes,
               row_bytes, bar);
  }
  pdl_launch_dependents();
  pdl_wait();
  if (!p.weights_static && warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar, rows * row_bytes);
    __syncwarp();
    if (lane < rows)
      bulk_g2s(wsh + lane * p.ws, p.packed + static_cast<size_t>(n0 + lane) * row_bytes,
               row_bytes, bar);
  }
  const float gamma = *p.gamma;
  bool weights_ok = true, waited = false;
  const int g = lane >> 2, tq = lane & 3;

  for (int m0 = 0; m0 < p.M; m0 += p.tg) {
    const int mg = min(p.tg, p.M - m0);
    // ---- activations of this token group -> shared memory (permuted int8)
    if (XK == kI8) {
      for (int i = tid; i < mg * words; i += kThreads) {
        const int t = i / words, w = i - t * words;
        const uint4 v = *reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(p.X) +
                                                         static_cast<size_t>(m0 + t) * p.K + 16 * w);
        uint4 o;
        o.x = __byte_perm(v.x, v.z, 0x5140);
        o.y = __byte_perm(v.y, v.w, 0x5140);
        o.z = __byte_perm(v.x, v.z, 0x7362);
        o.w = __byte_perm(v.y, v.w, 0x7362);
        *reinterpret_cast<uint4 *>(xsh + t * p.xs + 16 * w) = o;
      }
      if (tid < mg) s_sh[tid] = p.s_in[m0 + tid];
    } else if (mg == 1) {
      const float sm = quantize_token_block<XK>(p, m0, xsh, amax_sh);
      if (tid == 0) s_sh[0] = sm;
    } else {
      for (int t = warp; t < mg; t += kWarps) {
        const float sm = quantize_token_warp<XK>(p, m0 + t, xsh + t * p.xs);
        if (lane == 0) s_sh[t] = sm;
      }
    }
    __syncthreads();
    if (!waited) {
      weights_ok = mbar_wait(bar, 0, p.status);
      waited = true;
    }

    // ---- contraction: warp w takes 64-element steps [st0, st1)
    int c[MT][2][4];
#pragma unroll
    for (int tt = 0; tt < MT; ++tt)
#pragma unroll
      for (int h = 0; h < 2; ++h) c[tt][h][0] = c[tt][h][1] = c[tt][h][2] = c[tt][h][3] = 0;
    const int mt_active = (mg + 7) >> 3;
    if (weights_ok) {
      const uint32_t *wa_row = reinterpret_cast<const uint32_t *>(wsh + g * p.ws);
      const uint32_t *wb_row = reinterpret_cast<const uint32_t *>(wsh + (g + 8) * p.ws);
#pragma unroll 2
      for (int st = st0; st < st1; ++st) {
        const int word = 4 * st + tq;
        const uint32_t wa = wa_row[word], wb = wb_row[word];
        const uint32_t a0 = unpack_sel(wa, 0), a2 = unpack_sel(wa, 2);
        const uint32_t a1 = unpack_sel(wb, 0), a3 = unpack_sel(wb, 2);
        const uint32_t e0 = unpack_sel(wa, 16), e2 = unpack_sel(wa, 18);
        const uint32_t e1 = unpack_sel(wb, 16), e3 = unpack_sel(wb, 18);
        const int h = st & 1;
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
          if (tt < mt_active) {
            uint4 b = make_uint4(0, 0, 0, 0);
            if (tt * 8 + g < mg)
              b = *reinterpret_cast<const uint4 *>(xsh + (tt * 8 + g) * p.xs + 16 * word);
            if (h == 0) {
              mma_16832(c[tt][0], a0, a1, a2, a3, b.x, b.y);
              mma_16832(c[tt][0], e0, e1, e2, e3, b.z, b.w);
            } else {
              mma_16832(c[tt][1], a0, a1, a2, a3, b.x, b.y);
              mma_16832(c[tt][1], e0, e1, e2, e3, b.z, b.w);
            }
          }
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < MT; ++tt)
      red[(warp * MT + tt) * 32 + lane] =
          make_int4(c[tt][0][0] + c[tt][1][0], c[tt][0][1] + c[tt][1][1],
                    c[tt][0][2] + c[tt][1][2], c[tt][0][3] + c[tt][1][3]);
    __syncthreads();

    // ---- reduce the 8 warps and apply the epilogue
    if (tid < 32 * mt_active) {
      const int tt = tid >> 5, l = tid & 31, gr = l >> 2, tc = l & 3;
      int4 sum = red[tt * 32 + l];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) {
        const int4 v = red[(w * MT + tt) * 32 + l];
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      const int tok0 = tt * 8 + 2 * tc, tok1 = tok0 + 1;
      const float r0 = tok0 < mg ? __fdiv_rn(gamma, s_sh[tok0]) : 0.0f;
      const float r1 = tok1 < mg ? __fdiv_rn(gamma, s_sh[tok1]) : 0.0f;
      if (weights_ok) {
        if (gr < rows && tok0 < mg) emit<YK, RELU2>(p, n0 + gr, m0 + tok0, sum.x, r0);
        if (gr < rows && tok1 < mg) emit<YK, RELU2>(p, n0 + gr, m0 + tok1, sum.y, r1);
        if (gr + 8 < rows && tok0 < mg) emit<YK, RELU2>(p, n0 + gr + 8, m0 + tok0, sum.z, r0);
        if (gr + 8 < rows && tok1 < mg) emit<YK, RELU2>(p, n0 + gr + 8, m0 + tok1, sum.w, r1);
      }
    }
    __syncthreads();
  }
}

template <int MT, int XK, int YK, bool RELU2>
cudaError_t launch_t(const DecodeParams &p, size_t smem, const LaunchCtx &ctx) {
  auto kern = decode_kernel<MT, XK, YK, RELU2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(ceil_div(p.N, kRows)));
  return launch_k(kern, grid, dim3(kThreads), smem, ctx, p);
}

template <int MT, int XK>
cudaError_t dispatch_y(const DecodeParams &p, size_t smem, int y_kind, bool relu2,
                       const LaunchCtx &ctx) {
  if (y_kind == kI32) return launch_t<MT, XK, kI32, false>(p, smem, ctx);
  if (y_kind == kF32)
    return relu2 ? launch_t<MT, XK, kF32, true>(p, smem, ctx)
                 : launch_t<MT, XK, kF32, false>(p, smem, ctx);
  return relu2 ? launch_t<MT, XK, kBF16, true>(p, smem, ctx)
               : launch_t<MT, XK, kBF16, false>(p, smem, ctx);
}

// The library quantises the activations of this path once, in their own
// kernel, so the kernel is instantiated for int8 input only.
template <int MT>
cudaError_t dispatch_x(const DecodeParams &p, size_t smem, int x_kind, int y_kind, bool relu2,
                       const LaunchCtx &ctx) {
  if (x_kind != kI8) return cudaErrorInvalidValue;
  return dispatch_y<MT, kI8>(p, smem, y_kind, relu2, ctx);
}

}  // namespace

bool decode_supported(int64_t M, int64_t N, int64_t K) {
  return M > 8 && M <= 32 && N >= 1 && K % 64 == 0 && N < (1LL << 31) &&
         smem_bytes(1, static_cast<int>(K)) <= static_cast<size_t>(kSmemLimit);
}

cudaError_t launch_decode(const void *X, int x_kind, const float *s, const uint8_t *packed,
                          const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2,
                          void *Y, int y_kind, bool weights_static, const LaunchCtx &ctx) {
  int mt = static_cast<int>((M + 7) / 8);
  while (mt > 1 && smem_bytes(mt, static_cast<int>(K)) > static_cast<size_t>(kSmemLimit)) --mt;
  DecodeParams p;
  p.X = X;
  p.s_in = s;
  p.packed = packed;
  p.gamma = gamma;
  p.Y = Y;
  p.status = ctx.status;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ws = weight_row_bytes(static_cast<int>(K));
  p.xs = token_row_bytes(static_cast<int>(K));
  p.tg = 8 * mt;
  p.weights_static = weights_static ? 1 : 0;
  const size_t smem = smem_bytes(mt, static_cast<int>(K));
  switch (mt) {
    case 1: return dispatch_x<1>(p, smem, x_kind, y_kind, relu2, ctx);
    case 2: return dispatch_x<2>(p, smem, x_kind, y_kind, relu2, ctx);
    case 3: return dispatch_x<3>(p, smem, x_kind, y_kind, relu2, ctx);
    default: return dispatch_x<4>(p, smem, x_kind, y_kind, relu2, ctx);
  }
}

}  // namespace bitnet
