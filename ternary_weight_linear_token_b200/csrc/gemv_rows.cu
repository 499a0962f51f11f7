// gemv_rows.cu -- lowest-latency BitLinear forward for 1 to 4 tokens.
//
// At this size the packed weights of a projection (1.6 to 4.4 MB for the
// decode shapes) stream from HBM in well under a microsecond, so the time a
// call takes is set by its serial latency.  This kernel keeps that chain
// short: one warp per output feature n, 16 features per CTA.
//   1. Before waiting for the previous kernel in the stream (programmatic
//      dependent launch), the CTA starts asynchronous copies (cp.async) of
//      its 16 rows of packed weights into shared memory, when the caller
//      flags the weights as static; otherwise right after the wait.
//   2. After the wait, the CTA quantises the activations: every 16-element
//      group is loaded once, the per-token max |x| is reduced with one
//      redux.sync per warp and one shared-memory atomicMax (|x| >= 0, so its
//      bit pattern orders like an unsigned integer), and the int8 values
//      (s = 127 / amax, round half away, clamp +-127 -- identical to
//      bitnet_quantize_act) go to shared memory in the K order of the
//      unpack below.
//   3. Each lane takes words l, l+32, ... of its row (a 32-bit word holds
//      element 16g + 4j + i at bits 8i + 2j; shifting by 0, 2, 16, 18 and
//      masking with 0x3333 makes four byte-permute selectors that look the
//      2-bit codes up in {0, +1, -1, -1}) and accumulates xq . q with dp4a
//      on two independent chains, exactly, in int32 -- the add/subtract
//      identity of "Microsoft BitNet 深度研究报告" (技术原理 item 3) done as
//      signed byte products.
//   4. redux.sync.add gives the dot product; lane t applies
//      y = (float)acc * (gamma / s_t) and the optional ReLU^2 and stores y.
// No tensor cores: with one token the contraction is 2 ops per weight byte
// per token, far below what the SM's integer pipes sustain.
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxTok = 4;
constexpr int kSmemLimit = 227 * 1024;
constexpr uint32_t kTernaryLut = 0xFFFF0100u;  // code 0 -> 0, 1 -> +1, 2 -> -1, 3 -> -1

struct RowsParams {
  const void *X;
  const float *s_in;
  const uint8_t *packed;
  const float *gamma;
  void *Y;
  int M, N, K;
  int xs;  // shared-memory bytes per token row
  int ws;  // shared-memory bytes per weight row
  int weights_static;
};

constexpr int kHeader = 128;  // kMaxTok scales, kMaxTok amax words
int x_row_bytes(int K) { return (K + 127) / 128 * 128; }
int w_row_bytes(int K) { return (K / 4 + 15) / 16 * 16; }
size_t rows_smem(int M, int K) {
  return kHeader + static_cast<size_t>(M) * x_row_bytes(K) +
         static_cast<size_t>(kWarps) * w_row_bytes(K);
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// The CTA's rows of packed weights -> shared memory (asynchronous).
__device__ __forceinline__ void start_weight_copy(const RowsParams &p, int n0, int rows,
                                                  uint8_t *wsh) {
  const int row_bytes = p.K / 4;
  if ((row_bytes & 15) == 0) {
    const int per_row = row_bytes / 16;
    for (int i = threadIdx.x; i < rows * per_row; i += kThreads) {
      const int r = i / per_row, c = i - r * per_row;
      cp_async16(wsh + r * p.ws + 16 * c, p.packed + static_cast<size_t>(n0 + r) * row_bytes + 16 * c);
    }
  } else {
    const int per_row = row_bytes / 4;
    for (int i = threadIdx.x; i < rows * per_row; i += kThreads) {
      const int r = i / per_row, c = i - r * per_row;
      cp_async4(wsh + r * p.ws + 4 * c, p.packed + static_cast<size_t>(n0 + r) * row_bytes + 4 * c);
    }
  }
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

__device__ __forceinline__ int dot_word(uint32_t w, uint4 x, int acc) {
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, w & 0x3333u)), static_cast<int>(x.x), acc);
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, (w >> 2) & 0x3333u)), static_cast<int>(x.y), acc);
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, (w >> 16) & 0x3333u)), static_cast<int>(x.z), acc);
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, (w >> 18) & 0x3333u)), static_cast<int>(x.w), acc);
  return acc;
}

template <int MT, int XK, int YK, bool RELU2>
__global__ void __launch_bounds__(kThreads) rows_kernel(const RowsParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  float *s_sh = reinterpret_cast<float *>(smem);                   // kMaxTok scales
  unsigned *amax_sh = reinterpret_cast<unsigned *>(smem + 16);     // kMaxTok |x| maxima (bits)
  uint8_t *xsh = smem + kHeader;
  uint8_t *wsh = xsh + MT * p.xs;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kWarps;
  const int rows = min(kWarps, p.N - n0);
  const int words = p.K / 16;

  if (tid < kMaxTok) amax_sh[tid] = 0u;
  if (p.weights_static) start_weight_copy(p, n0, rows, wsh);
  __syncthreads();  // amax_sh zeroed before any atomicMax
  pdl_launch_dependents();
  pdl_wait();
  if (!p.weights_static) start_weight_copy(p, n0, rows, wsh);

  // ---- activations -> shared memory (int8, unpack order), per-token scales
  if (XK == kI8) {
    for (int i = tid; i < MT * words; i += kThreads) {
      const int t = i / words, w = i - t * words;
      const uint4 v = *reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(p.X) +
                                                       static_cast<size_t>(t) * p.K + 16 * w);
      uint4 o;
      o.x = __byte_perm(v.x, v.z, 0x5140);
      o.y = __byte_perm(v.y, v.w, 0x5140);
      o.z = __byte_perm(v.x, v.z, 0x7362);
      o.w = __byte_perm(v.y, v.w, 0x7362);
      *reinterpret_cast<uint4 *>(xsh + t * p.xs + 16 * w) = o;
    }
    if (tid < MT) s_sh[tid] = p.s_in[tid];
  } else {
    float v0[MT][16];  // the thread's first group of each token, kept for the second use
    unsigned amax[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      float a = 0.0f;
      if (tid < words) {
        load16<XK>(p.X, static_cast<size_t>(t) * p.K + 16 * tid, v0[t]);
#pragma unroll
        for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(v0[t][e]));
      }
      for (int w = tid + kThreads; w < words; w += kThreads) {
        float v[16];
        load16<XK>(p.X, static_cast<size_t>(t) * p.K + 16 * w, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(v[e]));
      }
      amax[t] = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
    }
    if (lane == 0) {
#pragma unroll
      for (int t = 0; t < MT; ++t) atomicMax(&amax_sh[t], amax[t]);
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const float sm = act_scale(__uint_as_float(amax_sh[t]));
      if (tid == 0) s_sh[t] = sm;
      if (tid < words) {
        int q[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) q[e] = quant_i8(v0[t][e], sm);
        *reinterpret_cast<uint4 *>(xsh + t * p.xs + 16 * tid) = pack_permuted(q);
      }
      for (int w = tid + kThreads; w < words; w += kThreads) {
        float v[16];
        load16<XK>(p.X, static_cast<size_t>(t) * p.K + 16 * w, v);
        int q[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) q[e] = quant_i8(v[e], sm);
        *reinterpret_cast<uint4 *>(xsh + t * p.xs + 16 * w) = pack_permuted(q);
      }
    }
  }
  cp_async_commit_wait();
  __syncthreads();
  if (warp >= rows) return;

  // ---- dot products of row n0 + warp with each token
  const uint32_t *wrow = reinterpret_cast<const uint32_t *>(wsh + warp * p.ws);
  int acc[MT][2];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = 0;
  int w = lane;
  for (; w + 32 < words; w += 64) {
    const uint32_t wa = wrow[w], wb = wrow[w + 32];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      acc[t][0] = dot_word(wa, *reinterpret_cast<const uint4 *>(xsh + t * p.xs + 16 * w), acc[t][0]);
      acc[t][1] = dot_word(wb, *reinterpret_cast<const uint4 *>(xsh + t * p.xs + 16 * (w + 32)), acc[t][1]);
    }
  }
  if (w < words) {
    const uint32_t wa = wrow[w];
#pragma unroll
    for (int t = 0; t < MT; ++t)
      acc[t][0] = dot_word(wa, *reinterpret_cast<const uint4 *>(xsh + t * p.xs + 16 * w), acc[t][0]);
  }
  int res = 0;
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    const int a = __reduce_add_sync(0xffffffffu, acc[t][0] + acc[t][1]);
    if (lane == t) res = a;
  }
  if (lane < MT) {
    const int n = n0 + warp;
    const size_t o = static_cast<size_t>(lane) * p.N + n;
    if (YK == kI32) {
      static_cast<int *>(p.Y)[o] = res;
    } else {
      const float y = epilogue_value(res, __fdiv_rn(*p.gamma, s_sh[lane]), RELU2);
      if (YK == kF32)
        static_cast<float *>(p.Y)[o] = y;
      else
        static_cast<__nv_bfloat16 *>(p.Y)[o] = __float2bfloat16_rn(y);
    }
  }
}

template <int MT, int XK, int YK, bool RELU2>
cudaError_t launch_t(const RowsParams &p, size_t smem, const LaunchCtx &ctx) {
  auto kern = rows_kernel<MT, XK, YK, RELU2>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(static_cast<unsigned>(ceil_div(p.N, kWarps)));
  return launch_k(kern, grid, dim3(kThreads), smem, ctx, p);
}

template <int MT, int XK>
cudaError_t dispatch_y(const RowsParams &p, size_t smem, int y_kind, bool relu2,
                       const LaunchCtx &ctx) {
  if (y_kind == kI32) return launch_t<MT, XK, kI32, false>(p, smem, ctx);
  if (y_kind == kF32)
    return relu2 ? launch_t<MT, XK, kF32, true>(p, smem, ctx) : launch_t<MT, XK, kF32, false>(p, smem, ctx);
  return relu2 ? launch_t<MT, XK, kBF16, true>(p, smem, ctx) : launch_t<MT, XK, kBF16, false>(p, smem, ctx);
}

template <int MT>
cudaError_t dispatch_x(const RowsParams &p, size_t smem, int x_kind, int y_kind, bool relu2,
                       const LaunchCtx &ctx) {
  if (x_kind == kI8) return dispatch_y<MT, kI8>(p, smem, y_kind, relu2, ctx);
  if (x_kind == kF32) return dispatch_y<MT, kF32>(p, smem, y_kind, relu2, ctx);
  return dispatch_y<MT, kBF16>(p, smem, y_kind, relu2, ctx);
}

}  // namespace

bool rows_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 1 && M <= kMaxTok && N >= 1 && N < (1LL << 31) && K % 16 == 0 &&
         rows_smem(static_cast<int>(M), static_cast<int>(K)) <= static_cast<size_t>(kSmemLimit);
}

cudaError_t launch_rows(const void *X, int x_kind, const float *s, const uint8_t *packed,
                        const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2, void *Y,
                        int y_kind, bool weights_static, const LaunchCtx &ctx) {
  RowsParams p;
  p.X = X;
  p.s_in = s;
  p.packed = packed;
  p.gamma = gamma;
  p.Y = Y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.xs = x_row_bytes(static_cast<int>(K));
  p.ws = w_row_bytes(static_cast<int>(K));
  p.weights_static = weights_static ? 1 : 0;
  const size_t smem = rows_smem(static_cast<int>(M), static_cast<int>(K));
  switch (M) {
    case 1: return dispatch_x<1>(p, smem, x_kind, y_kind, relu2, ctx);
    case 2: return dispatch_x<2>(p, smem, x_kind, y_kind, relu2, ctx);
    case 3: return dispatch_x<3>(p, smem, x_kind, y_kind, relu2, ctx);
    default: return dispatch_x<4>(p, smem, x_kind, y_kind, relu2, ctx);
  }
}

}  // namespace bitnet
