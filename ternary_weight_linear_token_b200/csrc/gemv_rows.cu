// gemv_rows.cu -- lowest-latency BitLinear forward for 1 to 8 tokens.
//
// At this size the packed weights of a projection (1.6 to 4.4 MB for the
// decode shapes) stream from HBM in well under a microsecond, so the time a
// call takes is set by its serial latency and by the busiest SM.  The grid
// has one CTA per SM (up to 32 warps each, more CTAs only for very wide
// projections), and each CTA owns a contiguous, balanced range of output
// features (17 or 18 of N = 2560 on 148 SMs); warp w takes features w,
// w + warps, ... of that range.
//   1. Before waiting for the previous kernel in the stream (programmatic
//      dependent launch), the CTA starts asynchronous copies (cp.async) of
//      its rows of packed weights into shared memory, when the caller flags
//      the weights as static; otherwise right after the wait.
//   2. After the wait, the CTA quantises the activations, 8 elements per
//      thread: each element is loaded once, the per-token max |x| is reduced
//      with one redux.sync per warp and one block barrier, and the int8
//      values (s = 127 / amax, round half away, clamp +-127 -- identical to
//      bitnet_quantize_act) go to shared memory in the K order of the unpack
//      below (neighbouring threads swap 4 bytes with one shuffle for that).
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
//
// Shared-memory K order of one 16-element group (16 bytes): the elements the
// unpack pairs with selector shifts 0, 16, 2, 18 -- {0,8,1,9}, {2,10,3,11},
// {4,12,5,13}, {6,14,7,15} -- so elements 0..7 of the group fill bytes 0..7
// with the help of 4 bytes from elements 8..11, and vice versa.
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kMaxWarps = 32;
constexpr int kMaxTok = 8;
constexpr int kSmemLimit = 227 * 1024;

struct RowsParams {
  const void *X;
  const float *s_in;
  const uint8_t *packed;
  const float *gamma;
  void *Y;
  int M, N, K;
  int ctas;      // grid size: CTA c owns rows [c*N/ctas, (c+1)*N/ctas)
  int xs;        // shared-memory bytes per token row
  int ws;        // shared-memory bytes per weight row
  int weights_static;
  void *Xn;      // NORM: the normalised input, written by CTA 0 (may be null)
  int rpw;       // rows per warp in the dot products (1, 2 or 4; > 1 only for M <= 2)
};

// scales [kMaxTok], gamma/s [kMaxTok], per-warp maxima [kMaxWarps][kMaxTok]
// (fp32), then per-warp sums of squares [kMaxWarps][kMaxTok] (fp64)
constexpr int kHeader = 32 + 32 + kMaxWarps * kMaxTok * 4 + kMaxWarps * kMaxTok * 8;
int x_row_bytes(int K) { return (K + 127) / 128 * 128; }
int w_row_bytes(int K) { return (K / 4 + 15) / 16 * 16; }
// One CTA per SM, so that a wide projection never runs a second wave (two
// such CTAs do not fit on one SM together), unless a CTA would own more than
// kMaxRowsPerCta features; never more CTAs than features.
constexpr int kMaxRowsPerCta = 64;
int rows_ctas(int64_t N, int num_sms) {
  const int64_t per_sm_rows = (N + num_sms - 1) / num_sms;
  const int64_t ctas = num_sms * ((per_sm_rows + kMaxRowsPerCta - 1) / kMaxRowsPerCta);
  return static_cast<int>(ctas < N ? ctas : N);
}
int rows_per_cta(int64_t N, int ctas) { return static_cast<int>((N + ctas - 1) / ctas); }
size_t rows_smem(int M, int K, int rows) {
  return kHeader + static_cast<size_t>(M) * x_row_bytes(K) + static_cast<size_t>(rows) * w_row_bytes(K);
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
    for (int i = threadIdx.x; i < rows * per_row; i += blockDim.x) {
      const int r = i / per_row, c = i - r * per_row;
      cp_async16(wsh + r * p.ws + 16 * c, p.packed + static_cast<size_t>(n0 + r) * row_bytes + 16 * c);
    }
  } else {
    const int per_row = row_bytes / 4;
    for (int i = threadIdx.x; i < rows * per_row; i += blockDim.x) {
      const int r = i / per_row, c = i - r * per_row;
      cp_async4(wsh + r * p.ws + 4 * c, p.packed + static_cast<size_t>(n0 + r) * row_bytes + 4 * c);
    }
  }
}

// 8 consecutive activations (16- or 32-byte aligned) as raw words, and
// their fp32 values.
template <int KIND>
struct Raw8 {
  uint4 u[KIND == kF32 ? 2 : 1];
};
template <int KIND>
__device__ __forceinline__ Raw8<KIND> load_raw8(const void *X, size_t idx) {
  Raw8<KIND> r;
  if (KIND == kF32) {
    const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const float *>(X) + idx);
    r.u[0] = p[0];
    r.u[KIND == kF32 ? 1 : 0] = p[1];
  } else {
    r.u[0] = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(X) + idx);
  }
  return r;
}
template <int KIND>
__device__ __forceinline__ void raw8_to_float(const Raw8<KIND> &r, float (&v)[8]) {
  if (KIND == kF32) {
    const uint32_t w[8] = {r.u[0].x, r.u[0].y, r.u[0].z, r.u[0].w, r.u[KIND == kF32 ? 1 : 0].x,
                           r.u[KIND == kF32 ? 1 : 0].y, r.u[KIND == kF32 ? 1 : 0].z,
                           r.u[KIND == kF32 ? 1 : 0].w};
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(w[e]);
  } else {
    const uint32_t w[4] = {r.u[0].x, r.u[0].y, r.u[0].z, r.u[0].w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[2 * h] = __uint_as_float(w[h] << 16);
      v[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
    }
  }
}

// 8 consecutive activations (16- or 32-byte aligned) as fp32.
template <int KIND>
__device__ __forceinline__ void load8(const void *X, size_t idx, float (&v)[8]) {
  if (KIND == kF32) {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(X) + idx);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(X) + idx);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[2 * h] = __uint_as_float(w[h] << 16);
      v[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
    }
  }
}

// x rounded to the input's precision (the normalised input is stored in it).
template <int XK>
__device__ __forceinline__ float round_to_input(float x) {
  return XK == kBF16 ? __bfloat162float(__float2bfloat16_rn(x)) : x;
}

// 8 values in the input's precision to memory (16- or 32-byte aligned).
template <int XK>
__device__ __forceinline__ void store8(void *X, size_t idx, const float (&v)[8]) {
  if (XK == kF32) {
    float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(X) + idx);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h)
      o[h] = (__float_as_uint(v[2 * h]) >> 16) | (__float_as_uint(v[2 * h + 1]) & 0xFFFF0000u);
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(X) + idx) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// NORM: the input is first normalised per token, x / sqrt(mean(x^2) + 1e-6)
// in fp32, and rounded to its own precision; that is what gets quantised.
// Warps per CTA at most: four or more tokens need more registers per thread.
template <int MT>
constexpr int warp_cap() { return MT >= 4 ? kMaxWarps / 2 : kMaxWarps; }

template <int MT, int XK, int YK, bool RELU2, bool NORM>
__global__ void __launch_bounds__(32 * warp_cap<MT>(), 1) rows_kernel(const RowsParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  float *s_sh = reinterpret_cast<float *>(smem);                 // kMaxTok scales
  float *r_sh = reinterpret_cast<float *>(smem + 32);            // kMaxTok gamma / s
  float *wmax = reinterpret_cast<float *>(smem + 64);            // [kMaxWarps][kMaxTok]
  double *wss = reinterpret_cast<double *>(wmax + kMaxWarps * kMaxTok);  // [kMaxWarps][kMaxTok]
  uint8_t *xsh = smem + kHeader;
  uint8_t *wsh = xsh + p.M * p.xs;  // the host sizes shared memory for p.M token rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = blockDim.x >> 5;
  const int n0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.N / p.ctas);
  const int n1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.N / p.ctas);
  const int rows = n1 - n0;
  const int words = p.K / 16;

  // gamma belongs to the weights: with static weights it is read before the
  // wait too, so its load is not on the path from the wait to the epilogue
  float gamma = 0.0f;
  if (p.weights_static) {
    start_weight_copy(p, n0, rows, wsh);
    gamma = *p.gamma;
  }
  pdl_launch_dependents();
  pdl_wait();
  if (!p.weights_static) {
    start_weight_copy(p, n0, rows, wsh);
    gamma = *p.gamma;
  }

  // ---- activations -> shared memory (int8, unpack order), per-token scales
  if (XK == kI8) {
    for (int i = tid; i < p.M * words; i += blockDim.x) {
      const int t = i / words, w = i - t * words;
      const uint4 v = *reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(p.X) +
                                                       static_cast<size_t>(t) * p.K + 16 * w);
      uint4 o;
      o.x = __byte_perm(v.x, v.z, 0x5140);
      o.y = __byte_perm(v.x, v.z, 0x7362);
      o.z = __byte_perm(v.y, v.w, 0x5140);
      o.w = __byte_perm(v.y, v.w, 0x7362);
      *reinterpret_cast<uint4 *>(xsh + t * p.xs + 16 * w) = o;
    }
    if (tid < p.M) {
      s_sh[tid] = p.s_in[tid];
      r_sh[tid] = __fdiv_rn(gamma, p.s_in[tid]);
    }
  } else {
    const int chunks = p.K / 8;
    // Tokens whose first 8 elements (per thread) are loaded up front, all at
    // once, and stay in registers for both passes: the loads of different
    // tokens are then in flight together instead of one token after another.
    constexpr int kCached = XK == kF32 ? (MT < 4 ? MT : 4) : MT;
    Raw8<XK> c0[kCached];
#pragma unroll
    for (int t = 0; t < kCached; ++t)
      if (t < p.M && tid < chunks) c0[t] = load_raw8<XK>(p.X, static_cast<size_t>(t) * p.K + 8 * tid);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t >= p.M) break;
      float a = 0.0f;
      double ss = 0.0;
      if (tid < chunks) {
        float v[8];
        if (t < kCached)
          raw8_to_float<XK>(c0[t < kCached ? t : 0], v);
        else
          load8<XK>(p.X, static_cast<size_t>(t) * p.K + 8 * tid, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          a = fmaxf(a, fabsf(v[e]));
          if (NORM) ss = add_sq(ss, v[e]);
        }
      }
      for (int c = tid + blockDim.x; c < chunks; c += blockDim.x) {
        float v[8];
        load8<XK>(p.X, static_cast<size_t>(t) * p.K + 8 * c, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          a = fmaxf(a, fabsf(v[e]));
          if (NORM) ss = add_sq(ss, v[e]);
        }
      }
      a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
      if (NORM) ss = warp_sum_f64(ss);
      if (lane == 0) {
        wmax[warp * kMaxTok + t] = a;
        if (NORM) wss[warp * kMaxTok + t] = ss;
      }
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t >= p.M) break;
      // the per-warp maxima, one per lane, reduced by each warp at once (max
      // is exact in any order; a loop over them cost every thread nwarps
      // dependent shared-memory reads)
      const float wm = lane < nwarps ? wmax[lane * kMaxTok + t] : 0.0f;
      float a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(wm)));
      float inv = 1.0f;
      if (NORM) {
        // the per-warp sums, one per lane, summed by each warp at once (fp64)
        inv = rms_factor(warp_sum_f64(lane < nwarps ? wss[lane * kMaxTok + t] : 0.0), p.K);
        // rounding x * inv to the input's precision is monotone in |x|: the
        // max of the normalised values is the normalised max
        a = round_to_input<XK>(__fmul_rn(a, inv));
      }
      const float sm = act_scale(a);
      const bool write_n = NORM && p.Xn != nullptr && blockIdx.x == 0;
      if (tid == blockDim.x - 1) {  // a lane with no activation work in the common case
        s_sh[t] = sm;
        r_sh[t] = __fdiv_rn(gamma, sm);
      }
      uint8_t *xrow = xsh + t * p.xs;
      {
        float v[8];
        if (t < kCached) {
          if (tid < chunks) raw8_to_float<XK>(c0[t < kCached ? t : 0], v);
        } else if (tid < chunks) {
          load8<XK>(p.X, static_cast<size_t>(t) * p.K + 8 * tid, v);
        }
        if (NORM && tid < chunks) {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = round_to_input<XK>(__fmul_rn(v[e], inv));
          if (write_n) store8<XK>(p.Xn, static_cast<size_t>(t) * p.K + 8 * tid, v);
        }
        store_half_group(xrow, tid, v, sm, tid < chunks);
      }
      for (int c0 = blockDim.x; c0 < chunks; c0 += blockDim.x) {  // whole warps iterate together
        const int c = c0 + tid;
        float v[8];
        if (c < chunks) {
          load8<XK>(p.X, static_cast<size_t>(t) * p.K + 8 * c, v);
          if (NORM) {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = round_to_input<XK>(__fmul_rn(v[e], inv));
            if (write_n) store8<XK>(p.Xn, static_cast<size_t>(t) * p.K + 8 * c, v);
          }
        }
        store_half_group(xrow, c, v, sm, c < chunks);
      }
    }
  }
  cp_async_commit_wait();
  __syncthreads();

  // ---- dot products, rpw > 1 (one or two tokens): rpw rows per warp, 32 / rpw
  // lanes per row.  Lanes at the same word position of different rows read
  // the same activation bytes (a shared-memory broadcast), so the activations
  // are read rpw times less often than with one row per warp.
  if (MT <= 2 && p.rpw > 1) {
    const int G = 32 / p.rpw, g = lane / G, j = lane % G;
    for (int rb = warp * p.rpw; rb < rows; rb += nwarps * p.rpw) {
      const int rl = rb + g;
      const bool live = rl < rows;
      const uint32_t *wrow = reinterpret_cast<const uint32_t *>(wsh + (live ? rl : 0) * p.ws);
      int acc[MT][2];
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = 0;
      int w = j;
      for (; w + 3 * G < words; w += 4 * G) {  // four words of the row in flight per lane
        const Unpacked q0 = unpack_word(wrow[w]), q1 = unpack_word(wrow[w + G]);
        const Unpacked q2 = unpack_word(wrow[w + 2 * G]), q3 = unpack_word(wrow[w + 3 * G]);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (t < p.M) {
            const uint4 *xr = reinterpret_cast<const uint4 *>(xsh + t * p.xs);
            const int b0 = dot_word(q0, xr[w], 0), b1 = dot_word(q1, xr[w + G], 0);
            const int b2 = dot_word(q2, xr[w + 2 * G], 0), b3 = dot_word(q3, xr[w + 3 * G], 0);
            acc[t][0] += b0 + b2;
            acc[t][1] += b1 + b3;
          }
        }
      }
      for (; w < words; w += G) {
        const Unpacked q = unpack_word(wrow[w]);
#pragma unroll
        for (int t = 0; t < MT; ++t)
          if (t < p.M)
            acc[t][0] = dot_word(q, *reinterpret_cast<const uint4 *>(xsh + t * p.xs + 16 * w), acc[t][0]);
      }
      int res = 0;
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        int v = acc[t][0] + acc[t][1];
        for (int o = G >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (j == t) res = v;
      }
      if (live && j < p.M) {
        const size_t o = static_cast<size_t>(j) * p.N + n0 + rl;
        if (YK == kI32) {
          static_cast<int *>(p.Y)[o] = res;
        } else {
          const float y = epilogue_value(res, r_sh[j], RELU2);
          if (YK == kF32)
            static_cast<float *>(p.Y)[o] = y;
          else
            static_cast<__nv_bfloat16 *>(p.Y)[o] = __float2bfloat16_rn(y);
        }
      }
    }
    return;
  }
  // ---- dot products: warp w takes rows w, w + nwarps, ... of the CTA's range
  for (int rl = warp; rl < rows; rl += nwarps) {
    const uint32_t *wrow = reinterpret_cast<const uint32_t *>(wsh + rl * p.ws);
    int acc[MT][2];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = 0;
    int w = lane;
    if (MT <= 2) {  // four words of the row in flight per lane
      for (; w + 96 < words; w += 128) {
        const Unpacked q0 = unpack_word(wrow[w]), q1 = unpack_word(wrow[w + 32]);
        const Unpacked q2 = unpack_word(wrow[w + 64]), q3 = unpack_word(wrow[w + 96]);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (t < p.M) {
            const uint4 *xr = reinterpret_cast<const uint4 *>(xsh + t * p.xs);
            const int b0 = dot_word(q0, xr[w], 0), b1 = dot_word(q1, xr[w + 32], 0);
            const int b2 = dot_word(q2, xr[w + 64], 0), b3 = dot_word(q3, xr[w + 96], 0);
            acc[t][0] += b0 + b2;
            acc[t][1] += b1 + b3;
          }
        }
      }
    }
    for (; w + 32 < words; w += 64) {
      const Unpacked qa = unpack_word(wrow[w]), qb = unpack_word(wrow[w + 32]);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < p.M) {
          acc[t][0] = dot_word(qa, *reinterpret_cast<const uint4 *>(xsh + t * p.xs + 16 * w), acc[t][0]);
          acc[t][1] = dot_word(qb, *reinterpret_cast<const uint4 *>(xsh + t * p.xs + 16 * (w + 32)), acc[t][1]);
        }
      }
    }
    if (w < words) {
      const Unpacked qa = unpack_word(wrow[w]);
#pragma unroll
      for (int t = 0; t < MT; ++t)
        if (t < p.M)
          acc[t][0] = dot_word(qa, *reinterpret_cast<const uint4 *>(xsh + t * p.xs + 16 * w), acc[t][0]);
    }
    int res = 0;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int a = __reduce_add_sync(0xffffffffu, acc[t][0] + acc[t][1]);
      if (lane == t) res = a;
    }
    if (lane < p.M) {
      const size_t o = static_cast<size_t>(lane) * p.N + n0 + rl;
      if (YK == kI32) {
        static_cast<int *>(p.Y)[o] = res;
      } else {
        const float y = epilogue_value(res, r_sh[lane], RELU2);
        if (YK == kF32)
          static_cast<float *>(p.Y)[o] = y;
        else
          static_cast<__nv_bfloat16 *>(p.Y)[o] = __float2bfloat16_rn(y);
      }
    }
  }
}

template <int MT, int XK, int YK, bool RELU2, bool NORM>
cudaError_t launch_t(const RowsParams &p, size_t smem, const LaunchCtx &ctx) {
  auto kern = rows_kernel<MT, XK, YK, RELU2, NORM>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // At most half the SM's registers per CTA, so that the next call's CTA can
  // be resident (and prefetch its weights) while this one still runs.
  static const int max_warps = [&] {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, kern) != cudaSuccess || a.numRegs <= 0) return 16;
    const int regs = (a.numRegs + 7) / 8 * 8;  // allocation granularity
    const int w = 32768 / (32 * regs);
    return w < 2 ? 2 : (w > warp_cap<MT>() ? warp_cap<MT>() : w);
  }();
  const int rpc = rows_per_cta(p.N, p.ctas);
  const int want = (rpc + p.rpw - 1) / p.rpw;
  const int warps = want < max_warps ? want : max_warps;
  return launch_k(kern, dim3(static_cast<unsigned>(p.ctas)), dim3(32 * (warps < 2 ? 2 : warps)),
                  smem, ctx, p);
}

template <int MT, int XK, bool NORM>
cudaError_t dispatch_y(const RowsParams &p, size_t smem, int y_kind, bool relu2,
                       const LaunchCtx &ctx) {
  if (y_kind == kI32) return launch_t<MT, XK, kI32, false, NORM>(p, smem, ctx);
  if (y_kind == kF32)
    return relu2 ? launch_t<MT, XK, kF32, true, NORM>(p, smem, ctx)
                 : launch_t<MT, XK, kF32, false, NORM>(p, smem, ctx);
  return relu2 ? launch_t<MT, XK, kBF16, true, NORM>(p, smem, ctx)
               : launch_t<MT, XK, kBF16, false, NORM>(p, smem, ctx);
}

template <int MT>
cudaError_t dispatch_x(const RowsParams &p, size_t smem, int x_kind, int y_kind, bool relu2,
                       bool norm, const LaunchCtx &ctx) {
  if (x_kind == kI8) return dispatch_y<MT, kI8, false>(p, smem, y_kind, relu2, ctx);
  if (x_kind == kF32)
    return norm ? dispatch_y<MT, kF32, true>(p, smem, y_kind, relu2, ctx)
                : dispatch_y<MT, kF32, false>(p, smem, y_kind, relu2, ctx);
  return norm ? dispatch_y<MT, kBF16, true>(p, smem, y_kind, relu2, ctx)
              : dispatch_y<MT, kBF16, false>(p, smem, y_kind, relu2, ctx);
}

}  // namespace

bool rows_supported(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > kMaxTok || N < 1 || N >= (1LL << 31) || K % 16 != 0 || K > (1 << 20)) return false;
  // worst case rows per CTA on a device with at least 16 SMs
  const int rpc = rows_per_cta(N, rows_ctas(N, 16));
  return rows_smem(static_cast<int>(M), static_cast<int>(K), rpc) <= static_cast<size_t>(kSmemLimit);
}

cudaError_t launch_rows(const void *X, int x_kind, const float *s, const uint8_t *packed,
                        const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2, void *Y,
                        int y_kind, bool weights_static, bool norm, void *Xn,
                        const LaunchCtx &ctx) {
  if (norm && x_kind == kI8) return cudaErrorInvalidValue;
  RowsParams p;
  p.X = X;
  p.s_in = s;
  p.packed = packed;
  p.gamma = gamma;
  p.Y = Y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ctas = rows_ctas(N, ctx.num_sms);
  p.xs = x_row_bytes(static_cast<int>(K));
  p.ws = w_row_bytes(static_cast<int>(K));
  p.weights_static = weights_static ? 1 : 0;
  p.Xn = Xn;
  // Two rows per warp for one or two tokens when a CTA owns many rows: half
  // the activation re-reads of the dot products, for twice the words per
  // lane and half the warps.  Measured per M = 1 call (dependent calls, bf16):
  // N = 3840 (26 rows per CTA) 3.71 -> 3.09 us and N = 6912 (47 rows) 4.53 ->
  // 4.16 us, but N = 2560 (18 rows) 2.51 -> 3.53 us, where too few warps are
  // left for the activation prologue.
  p.rpw = (M <= 2 && rows_per_cta(N, p.ctas) >= 24) ? 2 : 1;
  const size_t smem = rows_smem(static_cast<int>(M), static_cast<int>(K), rows_per_cta(N, p.ctas));
  if (smem > static_cast<size_t>(kSmemLimit)) return cudaErrorInvalidValue;
  if (M == 1) return dispatch_x<1>(p, smem, x_kind, y_kind, relu2, norm, ctx);
  if (M == 2) return dispatch_x<2>(p, smem, x_kind, y_kind, relu2, norm, ctx);
  if (M <= 4) return dispatch_x<4>(p, smem, x_kind, y_kind, relu2, norm, ctx);
  return dispatch_x<8>(p, smem, x_kind, y_kind, relu2, norm, ctx);
}

}  // namespace bitnet
