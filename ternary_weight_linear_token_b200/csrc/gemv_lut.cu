// gemv_lut.cu -- table-lookup BitLinear forward for 1 to 8 tokens, kept as a
// measured comparison with the byte-permute + dp4a kernel (gemv_rows.cu).
//
// "Microsoft BitNet 深度研究报告" (技术原理 item 3, 查找表优化, and its
// bitnet.cpp kernel table: TL1/TL2, "int2 + LUT") describes the CPU kernels
// that avoid multiplications by precomputing, for each small group of
// activations, every sum a group of ternary weights can select, and then
// reading one table entry per group of weights.  This is that idea on the
// GPU, with groups of two weights, which is what one 4-bit nibble of the
// packed layout holds: byte i of the packed word of group g carries elements
// 16g + i and 16g + i + 4 in its low nibble, 16g + i + 8 and 16g + i + 12 in
// its high nibble.  Per token and per nibble position the table holds the
// 16 sums v(c0) * xq[e0] + v(c1) * xq[e1] (c = c0 + 4 * c1, v = {0, +1, -1,
// -1}), as int16; a packed byte then costs two table reads and two adds
// instead of one byte-permute and a quarter of a dp4a.  The sums are exact, so
// the int32 accumulators, the epilogue and the outputs are identical to the
// other kernels'.
//
// Layout of one token's table: [8 nibble positions j][16 values c][words w]
// int16, so that the 32 lanes of a warp, which read the same (j, c) of 32
// consecutive words at most, hit 16 different banks.  Every CTA builds the
// tables of all tokens for the whole K (16 * K bytes per token), which is
// exactly the cost that the per-SM split of a GEMV cannot amortise: at M = 1 a
// CTA owns some 18 rows, and builds 8 * K table entries for them.  Tokens are
// processed in batches whose tables fit in shared memory.
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxTok = 8;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kHeader = 512;  // scales [8], gamma / s [8], per-warp maxima [kWarps][8]
constexpr int kMaxRowsPerCta = 32;

struct LutParams {
  const void *X;
  const float *s_in;
  const uint8_t *packed;
  const float *gamma;
  void *Y;
  int M, N, K;
  int ctas;
  int ws;             // shared-memory bytes per weight row
  int tb;             // tokens per table batch
  int weights_static;
};

int lut_ctas(int64_t N, int num_sms) {
  const int64_t per_sm_rows = (N + num_sms - 1) / num_sms;
  const int64_t ctas = num_sms * ((per_sm_rows + kMaxRowsPerCta - 1) / kMaxRowsPerCta);
  return static_cast<int>(ctas < N ? ctas : N);
}
int lut_w_row_bytes(int K) { return (K / 4 + 15) / 16 * 16; }
__host__ __device__ inline size_t lut_table_bytes(int K) { return static_cast<size_t>(K) * 16; }  // 8 * 16 * (K/16) * 2
size_t lut_fixed_bytes(int M, int K, int rows) {
  return kHeader + static_cast<size_t>(M) * K + static_cast<size_t>(rows) * lut_w_row_bytes(K);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Ternary value of a 2-bit code: 0 -> 0, 1 -> +1, 2 and 3 -> -1.
__device__ __forceinline__ int code_value(int c) { return c == 0 ? 0 : (c == 1 ? 1 : -1); }

template <int XK, int YK, bool RELU2>
__global__ void __launch_bounds__(kThreads, 1) lut_kernel(const LutParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  float *s_sh = reinterpret_cast<float *>(smem);
  float *r_sh = reinterpret_cast<float *>(smem + 32);
  float *wmax = reinterpret_cast<float *>(smem + 64);  // [kWarps][kMaxTok]
  int8_t *xq = reinterpret_cast<int8_t *>(smem + kHeader);                 // [M][K], natural order
  uint8_t *wsh = smem + kHeader + static_cast<size_t>(p.M) * p.K;          // [rows][ws]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.N / p.ctas);
  const int n1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.N / p.ctas);
  const int rows = n1 - n0;
  const int words = p.K / 16;
  int16_t *tables = reinterpret_cast<int16_t *>(wsh + static_cast<size_t>(rows) * p.ws);

  // the CTA's rows of packed weights -> shared memory
  auto copy_weights = [&]() {
    const int row_bytes = p.K / 4;
    if ((row_bytes & 15) == 0) {
      const int per_row = row_bytes / 16;
      for (int i = tid; i < rows * per_row; i += kThreads) {
        const int r = i / per_row, c = i - r * per_row;
        cp_async16(wsh + r * p.ws + 16 * c, p.packed + static_cast<size_t>(n0 + r) * row_bytes + 16 * c);
      }
    } else {
      const int per_row = row_bytes / 4;
      for (int i = tid; i < rows * per_row; i += kThreads) {
        const int r = i / per_row, c = i - r * per_row;
        cp_async4(wsh + r * p.ws + 4 * c, p.packed + static_cast<size_t>(n0 + r) * row_bytes + 4 * c);
      }
    }
  };
  float gamma = 0.0f;
  if (p.weights_static) {
    copy_weights();
    gamma = *p.gamma;
  }
  pdl_launch_dependents();
  pdl_wait();
  if (!p.weights_static) {
    copy_weights();
    gamma = *p.gamma;
  }

  // ---- activations -> int8 in shared memory (natural K order), scales
  const int chunks = p.K / 8;
  if (XK == kI8) {
    for (int i = tid; i < p.M * (p.K / 16); i += kThreads) {
      const int t = i / (p.K / 16), c = i - t * (p.K / 16);
      *reinterpret_cast<uint4 *>(xq + static_cast<size_t>(t) * p.K + 16 * c) =
          *reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(p.X) +
                                           static_cast<size_t>(t) * p.K + 16 * c);
    }
    if (tid < p.M) {
      s_sh[tid] = p.s_in[tid];
      r_sh[tid] = __fdiv_rn(gamma, p.s_in[tid]);
    }
  } else {
    for (int t = 0; t < p.M; ++t) {
      float a = 0.0f;
      for (int c = tid; c < chunks; c += kThreads) {
        float v[8];
        if (XK == kF32) {
          const float4 *q = reinterpret_cast<const float4 *>(static_cast<const float *>(p.X) +
                                                             static_cast<size_t>(t) * p.K + 8 * c);
          const float4 u = q[0], w = q[1];
          v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w; v[4] = w.x; v[5] = w.y; v[6] = w.z; v[7] = w.w;
        } else {
          const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.X) +
                                                           static_cast<size_t>(t) * p.K + 8 * c);
          const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[2 * h] = __uint_as_float(wd[h] << 16);
            v[2 * h + 1] = __uint_as_float(wd[h] & 0xFFFF0000u);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[e]));
      }
      a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
      if (lane == 0) wmax[warp * kMaxTok + t] = a;
    }
    __syncthreads();
    for (int t = 0; t < p.M; ++t) {
      const float a = __uint_as_float(__reduce_max_sync(
          0xffffffffu, __float_as_uint(lane < kWarps ? wmax[lane * kMaxTok + t] : 0.0f)));
      const float sm = act_scale(a);
      if (tid == 0) {
        s_sh[t] = sm;
        r_sh[t] = __fdiv_rn(gamma, sm);
      }
      for (int c = tid; c < chunks; c += kThreads) {
        float v[8];
        if (XK == kF32) {
          const float4 *q = reinterpret_cast<const float4 *>(static_cast<const float *>(p.X) +
                                                             static_cast<size_t>(t) * p.K + 8 * c);
          const float4 u = q[0], w = q[1];
          v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w; v[4] = w.x; v[5] = w.y; v[6] = w.z; v[7] = w.w;
        } else {
          const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.X) +
                                                           static_cast<size_t>(t) * p.K + 8 * c);
          const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[2 * h] = __uint_as_float(wd[h] << 16);
            v[2 * h + 1] = __uint_as_float(wd[h] & 0xFFFF0000u);
          }
        }
        int q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = quant_i8(v[e], sm);
        *reinterpret_cast<uint2 *>(xq + static_cast<size_t>(t) * p.K + 8 * c) =
            make_uint2(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]));
      }
    }
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  const size_t tstride = lut_table_bytes(p.K) / 2;  // int16 entries per token's table
  for (int tb0 = 0; tb0 < p.M; tb0 += p.tb) {
    const int nt = p.M - tb0 < p.tb ? p.M - tb0 : p.tb;
    // ---- tables of tokens tb0 .. tb0 + nt - 1: entry (j, c, w) at (j * 16 + c) * words + w
    for (int idx = tid; idx < nt * 8 * words; idx += kThreads) {
      const int t = idx / (8 * words);
      const int rem = idx - t * 8 * words;
      const int j = rem / words, w = rem - j * words;
      const int e0 = 16 * w + (j >> 1) + 8 * (j & 1);
      const int xa = xq[static_cast<size_t>(tb0 + t) * p.K + e0];
      const int xb = xq[static_cast<size_t>(tb0 + t) * p.K + e0 + 4];
      int16_t *T = tables + t * tstride + static_cast<size_t>(j) * 16 * words + w;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        T[c * words] = static_cast<int16_t>(code_value(c & 3) * xa + code_value(c >> 2) * xb);
    }
    __syncthreads();
    // ---- dot products by lookups: warp w takes rows w, w + kWarps, ...
    for (int rl = warp; rl < rows; rl += kWarps) {
      const uint32_t *wrow = reinterpret_cast<const uint32_t *>(wsh + rl * p.ws);
      int acc[kMaxTok];
#pragma unroll
      for (int t = 0; t < kMaxTok; ++t) acc[t] = 0;
      for (int w = lane; w < words; w += 32) {
        const uint32_t word = wrow[w];
#pragma unroll
        for (int t = 0; t < kMaxTok; ++t) {
          if (t < nt) {
            const int16_t *T = tables + t * tstride + w;
            int a = acc[t];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t lo = (word >> (8 * i)) & 15u, hi = (word >> (8 * i + 4)) & 15u;
              a += T[((2 * i) * 16 + lo) * words] + T[((2 * i + 1) * 16 + hi) * words];
            }
            acc[t] = a;
          }
        }
      }
      int res = 0;
#pragma unroll
      for (int t = 0; t < kMaxTok; ++t) {
        if (t < nt) {
          const int v = __reduce_add_sync(0xffffffffu, acc[t]);
          if (lane == t) res = v;
        }
      }
      if (lane < nt) {
        const int t = tb0 + lane;
        const size_t o = static_cast<size_t>(t) * p.N + n0 + rl;
        if (YK == kI32) {
          static_cast<int *>(p.Y)[o] = res;
        } else {
          const float y = epilogue_value(res, r_sh[t], RELU2);
          if (YK == kF32)
            static_cast<float *>(p.Y)[o] = y;
          else
            static_cast<__nv_bfloat16 *>(p.Y)[o] = __float2bfloat16_rn(y);
        }
      }
    }
    __syncthreads();  // before the next batch's tables overwrite these
  }
}

template <int XK, int YK, bool RELU2>
cudaError_t launch_t(const LutParams &p, size_t smem, const LaunchCtx &ctx) {
  auto kern = lut_kernel<XK, YK, RELU2>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_k(kern, dim3(static_cast<unsigned>(p.ctas)), dim3(kThreads), smem, ctx, p);
}

template <int XK>
cudaError_t dispatch_y(const LutParams &p, size_t smem, int y_kind, bool relu2,
                       const LaunchCtx &ctx) {
  if (y_kind == kI32) return launch_t<XK, kI32, false>(p, smem, ctx);
  if (y_kind == kF32)
    return relu2 ? launch_t<XK, kF32, true>(p, smem, ctx) : launch_t<XK, kF32, false>(p, smem, ctx);
  return relu2 ? launch_t<XK, kBF16, true>(p, smem, ctx) : launch_t<XK, kBF16, false>(p, smem, ctx);
}

// Tokens per table batch for these sizes on a device with `num_sms` SMs
// (0: the tables of even one token do not fit).
int lut_batch(int64_t M, int64_t N, int64_t K, int num_sms) {
  const int ctas = lut_ctas(N, num_sms);
  const int rows = static_cast<int>((N + ctas - 1) / ctas);
  const size_t fixed = lut_fixed_bytes(static_cast<int>(M), static_cast<int>(K), rows);
  if (fixed >= static_cast<size_t>(kSmemLimit)) return 0;
  const int64_t tb = static_cast<int64_t>((kSmemLimit - fixed) / lut_table_bytes(static_cast<int>(K)));
  return static_cast<int>(tb < M ? tb : M);
}

}  // namespace

bool lut_supported(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > kMaxTok || N < 1 || N >= (1LL << 31) || K % 16 != 0 || K > (1 << 16))
    return false;
  return lut_batch(M, N, K, 16) >= 1;  // worst case rows per CTA on a device with 16 SMs
}

cudaError_t launch_lut(const void *X, int x_kind, const float *s, const uint8_t *packed,
                       const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2, void *Y,
                       int y_kind, bool weights_static, const LaunchCtx &ctx) {
  LutParams p;
  p.X = X;
  p.s_in = s;
  p.packed = packed;
  p.gamma = gamma;
  p.Y = Y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ctas = lut_ctas(N, ctx.num_sms);
  p.ws = lut_w_row_bytes(p.K);
  p.tb = lut_batch(M, N, K, ctx.num_sms);
  p.weights_static = weights_static ? 1 : 0;
  if (p.tb < 1) return cudaErrorInvalidValue;
  const int rows = static_cast<int>((N + p.ctas - 1) / p.ctas);
  const size_t smem = lut_fixed_bytes(p.M, p.K, rows) + static_cast<size_t>(p.tb) * lut_table_bytes(p.K);
  if (x_kind == kI8) return dispatch_y<kI8>(p, smem, y_kind, relu2, ctx);
  if (x_kind == kF32) return dispatch_y<kF32>(p, smem, y_kind, relu2, ctx);
  return dispatch_y<kBF16>(p, smem, y_kind, relu2, ctx);
}

}  // namespace bitnet
