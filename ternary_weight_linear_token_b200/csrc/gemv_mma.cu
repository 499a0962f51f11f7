// gemv_mma.cu -- BitLinear forward for a few tokens (4 <= M <= 32) on the
// int8 mma.sync path, with the tokens as the MMA's A operand.
//
// The activations arrive quantised (bitnet_quantize_act, int8 in the K order
// of the byte-permute weight unpack, one 16-byte chunk per packed word) and
// are staged in shared memory by one bulk copy per token when they fit
// beside the weights (else read from L2 in the loop, one K step ahead).  The
// grid has one CTA per SM, each owning a contiguous range of 8-row blocks of
// the weights (2 to 8 blocks), so the grid balances to within 8 rows; the
// CTA's packed rows arrive by bulk copies into padded shared-memory rows,
// issued before the grid-dependency wait when the caller flags the weights
// static.  The 8 warps split K into 64-element steps.  Per step a lane takes
// packed word 4*step + (lane % 4) of weight row lane / 4 of each block, and
// the matching 16-byte activation chunk of tokens lane / 4 and lane / 4 + 8
// (and + 16, + 24): the four byte-permute selectors of the word (shifts 0, 2,
// 16, 18) are the B fragments of two mma.sync.m16n8k32 per 16-token tile,
// and the chunk's four 4-byte parts are the A fragments -- both operands in
// the same K order, so the product is exact int32; the blocks and token
// tiles are independent accumulator chains.  The 8 warps' partial
// sums are reduced in shared memory and the epilogue applies gamma / s and
// the optional ReLU^2.
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxBlocks = 8;   // 8-row weight blocks per CTA
constexpr int kHeader = 256;    // mbarrier, gamma / s for 32 tokens
constexpr int kSmemLimit = 227 * 1024;

struct MmvParams {
  const int8_t *xq;     // [M][K], unpack order
  const float *s;       // [M]
  const uint8_t *packed;
  const float *gamma;
  void *Y;
  int *status;
  int M, N, K;
  int ctas, nblk;       // grid size, 8-row blocks of N
  int ws;               // shared-memory stride of a weight row (bytes)
  int weights_static;
  int x_smem;           // the activations are staged in shared memory (M * K bytes fit)
};

// Weight rows 16 mod 128 bytes apart: the 8 rows x 4 consecutive words a
// warp reads per step fall on 32 distinct banks.
int weight_row_stride(int K) {
  const int b = K / 4;  // a multiple of 16 (K % 64 == 0)
  return b + (((16 - b % 128) % 128) + 128) % 128;
}
template <int MT16>
__host__ __device__ constexpr int red_bytes() { return kWarps * kMaxBlocks * MT16 * 32 * 16; }
// Shared memory: header, the weight rows, then one area that first holds the
// staged activations (when they fit) and afterwards the warps' partial sums.
template <int MT16>
size_t smem_bytes(int K, size_t x_bytes) {
  const size_t tail = x_bytes > static_cast<size_t>(red_bytes<MT16>()) ? x_bytes : red_bytes<MT16>();
  return kHeader + static_cast<size_t>(8 * kMaxBlocks) * weight_row_stride(K) + tail;
}

__device__ __forceinline__ uint32_t sel(uint32_t w, int shift) {
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

template <int YK, bool RELU2>
__device__ __forceinline__ void emit(const MmvParams &p, int tok, int row, int acc, float r) {
  const size_t o = static_cast<size_t>(tok) * p.N + row;
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

template <int MT16, int YK, bool RELU2>
__global__ void __launch_bounds__(kThreads, 1) mmv_kernel(const MmvParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem);       // weights
  uint64_t *xbar = reinterpret_cast<uint64_t *>(smem + 8);  // staged activations
  float *r_sh = reinterpret_cast<float *>(smem + 128);      // gamma / s per token
  uint8_t *wsh = smem + kHeader;
  uint8_t *tail = wsh + 8 * kMaxBlocks * p.ws;
  int8_t *xsh = reinterpret_cast<int8_t *>(tail);           // [M][K] activations, when staged
  int4 *red = reinterpret_cast<int4 *>(tail);               // [kWarps][kMaxBlocks][MT16][32], after

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int blk0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.nblk / p.ctas);
  const int blk1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.nblk / p.ctas);
  const int nb = blk1 - blk0;
  const int r0 = 8 * blk0;
  const int rows = min(8 * blk1, p.N) - r0;
  const uint32_t row_bytes = static_cast<uint32_t>(p.K) / 4;
  const int steps = p.K / 64;
  const int st0 = warp * steps / kWarps, st1 = (warp + 1) * steps / kWarps;

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(xbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // the CTA's weight rows -> padded shared-memory rows (one bulk copy per row)
  if (p.weights_static && warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar, rows * row_bytes);
    __syncwarp();
    for (int r = lane; r < rows; r += 32)
      bulk_g2s(wsh + r * p.ws, p.packed + static_cast<size_t>(r0 + r) * row_bytes, row_bytes, bar);
  }
  pdl_launch_dependents();
  pdl_wait();
  if (!p.weights_static && warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar, rows * row_bytes);
    __syncwarp();
    for (int r = lane; r < rows; r += 32)
      bulk_g2s(wsh + r * p.ws, p.packed + static_cast<size_t>(r0 + r) * row_bytes, row_bytes, bar);
  }
  // the quantised activations (the previous kernel's output) -> shared memory
  if (p.x_smem && warp == 1) {
    if (lane == 0) mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.M) * p.K);
    __syncwarp();
    for (int t = lane; t < p.M; t += 32)
      bulk_g2s(xsh + static_cast<size_t>(t) * p.K, p.xq + static_cast<size_t>(t) * p.K,
               static_cast<uint32_t>(p.K), xbar);
  }
  if (tid < p.M) r_sh[tid] = __fdiv_rn(*p.gamma, p.s[tid]);
  // every lane waits (bounded); the warp computes only if all of them saw the copies land
  bool landed = mbar_wait(bar, 0, p.status);
  if (p.x_smem) landed = mbar_wait(xbar, 0, p.status) && landed;
  const bool weights_ok = __all_sync(0xffffffffu, landed);
  const int8_t *xsrc = p.x_smem ? xsh : p.xq;  // generic loads serve both

  int c[kMaxBlocks][MT16][4];  // independent accumulators: blocks x token tiles
#pragma unroll
  for (int b = 0; b < kMaxBlocks; ++b)
#pragma unroll
    for (int a = 0; a < MT16; ++a) c[b][a][0] = c[b][a][1] = c[b][a][2] = c[b][a][3] = 0;

  if (weights_ok) {
    // A: 16-byte activation chunks of this lane's tokens (zero past M); the
    // next step's chunks are loaded before this step's MMAs, so one load
    // latency overlaps one step of math
    uint4 xa[MT16][2], xn[MT16][2];
    auto load_x = [&](int st, uint4 (&dst)[MT16][2]) {
      const int word = 4 * st + tq;
#pragma unroll
      for (int a = 0; a < MT16; ++a)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int tok = 16 * a + 8 * h + g;
          dst[a][h] = tok < p.M ? *reinterpret_cast<const uint4 *>(xsrc + static_cast<size_t>(tok) * p.K + 16 * word)
                                : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    if (st0 < st1) load_x(st0, xa);
    for (int st = st0; st < st1; ++st) {
      const int word = 4 * st + tq;
      if (st + 1 < st1) load_x(st + 1, xn);
#pragma unroll
      for (int b = 0; b < kMaxBlocks; ++b) {
        if (b < nb) {
          const int row = 8 * b + g;
          const uint32_t w = row < rows ? reinterpret_cast<const uint32_t *>(wsh + row * p.ws)[word] : 0u;
          const uint32_t b0 = sel(w, 0), b1 = sel(w, 2), b2 = sel(w, 16), b3 = sel(w, 18);
#pragma unroll
          for (int a = 0; a < MT16; ++a) {
            mma_16832(c[b][a], xa[a][0].x, xa[a][1].x, xa[a][0].y, xa[a][1].y, b0, b1);
            mma_16832(c[b][a], xa[a][0].z, xa[a][1].z, xa[a][0].w, xa[a][1].w, b2, b3);
          }
        }
      }
#pragma unroll
      for (int a = 0; a < MT16; ++a) {
        xa[a][0] = xn[a][0];
        xa[a][1] = xn[a][1];
      }
    }
  }
  if (p.x_smem) __syncthreads();  // the partial sums overwrite the staged activations
#pragma unroll
  for (int b = 0; b < kMaxBlocks; ++b)
#pragma unroll
    for (int a = 0; a < MT16; ++a)
      if (b < nb)
        red[((warp * kMaxBlocks + b) * MT16 + a) * 32 + lane] =
            make_int4(c[b][a][0], c[b][a][1], c[b][a][2], c[b][a][3]);
  __syncthreads();

  // ---- reduce the 8 warps and apply the epilogue: one thread per (block, tile, lane)
  if (weights_ok) {
    for (int i = tid; i < nb * MT16 * 32; i += kThreads) {
      const int l = i & 31, a = (i >> 5) % MT16, b = (i >> 5) / MT16;
      int4 sum = red[(b * MT16 + a) * 32 + l];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) {
        const int4 v = red[((w * kMaxBlocks + b) * MT16 + a) * 32 + l];
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      // C fragment: rows (tokens) l / 4 and l / 4 + 8, columns (weight rows) 2 (l % 4) and + 1
      const int tok0 = 16 * a + (l >> 2), tok1 = tok0 + 8;
      const int row0 = 8 * b + 2 * (l & 3), row1 = row0 + 1;
      if (tok0 < p.M) {
        if (row0 < rows) emit<YK, RELU2>(p, tok0, r0 + row0, sum.x, r_sh[tok0]);
        if (row1 < rows) emit<YK, RELU2>(p, tok0, r0 + row1, sum.y, r_sh[tok0]);
      }
      if (tok1 < p.M) {
        if (row0 < rows) emit<YK, RELU2>(p, tok1, r0 + row0, sum.z, r_sh[tok1]);
        if (row1 < rows) emit<YK, RELU2>(p, tok1, r0 + row1, sum.w, r_sh[tok1]);
      }
    }
  }
}

template <int MT16, int YK, bool RELU2>
cudaError_t launch_t(const MmvParams &p, const LaunchCtx &ctx) {
  auto kern = mmv_kernel<MT16, YK, RELU2>;
  const size_t smem = smem_bytes<MT16>(p.K, p.x_smem ? static_cast<size_t>(p.M) * p.K : 0);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(kern, dim3(static_cast<unsigned>(p.ctas)), dim3(kThreads), smem, ctx, p);
}

template <int MT16>
cudaError_t dispatch_y(const MmvParams &p, int y_kind, bool relu2, const LaunchCtx &ctx) {
  if (y_kind == kI32) return launch_t<MT16, kI32, false>(p, ctx);
  if (y_kind == kF32)
    return relu2 ? launch_t<MT16, kF32, true>(p, ctx) : launch_t<MT16, kF32, false>(p, ctx);
  return relu2 ? launch_t<MT16, kBF16, true>(p, ctx) : launch_t<MT16, kBF16, false>(p, ctx);
}

}  // namespace

bool mmv_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 1 && M <= 32 && N >= 1 && N < (1LL << 30) && K % 64 == 0 && K <= (1 << 20) &&
         smem_bytes<2>(static_cast<int>(K), 0) <= static_cast<size_t>(kSmemLimit);
}

cudaError_t launch_mmv(const int8_t *xq, const float *s, const uint8_t *packed, const float *gamma,
                       int64_t M, int64_t N, int64_t K, bool relu2, void *Y, int y_kind,
                       bool weights_static, const LaunchCtx &ctx) {
  MmvParams p;
  p.xq = xq;
  p.s = s;
  p.packed = packed;
  p.gamma = gamma;
  p.Y = Y;
  p.status = ctx.status;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.nblk = static_cast<int>((N + 7) / 8);
  // one CTA per SM unless a CTA would own more than kMaxBlocks blocks
  const int per = (p.nblk + ctx.num_sms - 1) / ctx.num_sms;
  p.ctas = per <= kMaxBlocks ? (p.nblk < ctx.num_sms ? p.nblk : ctx.num_sms)
                             : (p.nblk + kMaxBlocks - 1) / kMaxBlocks;
  p.ws = weight_row_stride(p.K);
  p.weights_static = weights_static ? 1 : 0;
  // Stage the activations in shared memory when they fit beside the weights
  // and each warp has many K steps: measured per call, K = 6912 M = 8 went
  // from 9.7 to 8.1 us, while at K = 2560 (5 steps per warp) the up-front copy
  // only adds its latency (M = 32: 6.4 -> 6.8 us).
  const size_t staged = M <= 16 ? smem_bytes<1>(p.K, static_cast<size_t>(M) * K)
                                : smem_bytes<2>(p.K, static_cast<size_t>(M) * K);
  p.x_smem = (K > 4096 && staged <= static_cast<size_t>(kSmemLimit)) ? 1 : 0;
  return M <= 16 ? dispatch_y<1>(p, y_kind, relu2, ctx) : dispatch_y<2>(p, y_kind, relu2, ctx);
}

}  // namespace bitnet
