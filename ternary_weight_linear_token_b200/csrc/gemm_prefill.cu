// gemm_prefill.cu -- BitLinear forward for prefill-sized batches on the
// fifth-generation tensor cores (tcgen05, kind::i8, int32 accumulators in
// tensor memory).  The contraction is a dense int8 x int8 product: xq times
// the ternary weights {-1, 0, +1} held as int8 (BitNet b1.58 2B4T model card,
// 模型详情 -> 量化: W1.58A8; "Microsoft BitNet 深度研究报告", 技术原理 items 2-3).
//
// Tile: 128 tokens x 256 output features per CTA, K in 128-byte stages.
//   warp 0      TMA producer: xq tile [128 x 128 B] with the 128-byte swizzle
//               and the packed weight tile [256 rows x 32 B] (2 bits per
//               weight stay packed all the way from HBM into shared memory).
//   warp 1      allocates 256 TMEM columns; one lane issues 4 MMAs
//               (M=128, N=256, K=32) per stage and commits them to the
//               stage's "empty" barrier.
//   warps 2-9   expand each packed word into 16 int8 weights and store them
//               as the K-major, 128-byte-swizzled B operand; after the K loop
//               the same 8 warps read the accumulator (tcgen05.ld), apply
//               y = acc * (gamma / s_m) and the optional ReLU^2, and store Y.
// A 3-stage ring of mbarriers (TMA full, expansion full, MMA empty) keeps
// TMA, expansion and MMA of different stages in flight at once.  Every wait
// is bounded (see common.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int kStages = 3;
constexpr int kExpWarps = 8;
constexpr int kThreads = 32 * (2 + kExpWarps);
constexpr int kABytes = BM * BK;
constexpr int kBxBytes = BN * BK;
constexpr int kBpBytes = BN * BK / 4;
constexpr int kStageBytes = kABytes + kBxBytes + kBpBytes;
constexpr int kTmemCols = 256;
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + 256;

// Instruction descriptor: s8 x s8 -> s32, both operands K-major, M=128, N=256.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((BN >> 3) << 17) |
                            ((BM >> 4) << 24);

struct PrefillParams {
  const float *s;
  const float *gamma;
  void *Y;
  int *status;
  int64_t M, N, K;
};

template <int YK, bool RELU2>
__device__ __forceinline__ void store16(const PrefillParams &p, int64_t m, int64_t n,
                                        const uint32_t (&v)[16], float r, bool vec_ok) {
  const size_t o = static_cast<size_t>(m) * p.N + n;
  const int valid = static_cast<int>(p.N - n < 16 ? p.N - n : 16);
  if (YK == kI32) {
    int *dst = static_cast<int *>(p.Y) + o;
    if (vec_ok && valid == 16) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<uint4 *>(dst)[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
      for (int e = 0; e < valid; ++e) dst[e] = static_cast<int>(v[e]);
    }
  } else if (YK == kF32) {
    float y[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) y[e] = epilogue_value(static_cast<int>(v[e]), r, RELU2);
    float *dst = static_cast<float *>(p.Y) + o;
    if (vec_ok && valid == 16) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<float4 *>(dst)[q] = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
    } else {
      for (int e = 0; e < valid; ++e) dst[e] = y[e];
    }
  } else {
    uint32_t h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const __nv_bfloat162 b =
          __floats2bfloat162_rn(epilogue_value(static_cast<int>(v[2 * e]), r, RELU2),
                                epilogue_value(static_cast<int>(v[2 * e + 1]), r, RELU2));
      h[e] = *reinterpret_cast<const uint32_t *>(&b);
    }
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.Y) + o;
    if (vec_ok && valid == 16) {
      reinterpret_cast<uint4 *>(dst)[0] = make_uint4(h[0], h[1], h[2], h[3]);
      reinterpret_cast<uint4 *>(dst)[1] = make_uint4(h[4], h[5], h[6], h[7]);
    } else {
      const __nv_bfloat16 *src = reinterpret_cast<const __nv_bfloat16 *>(h);
      for (int e = 0; e < valid; ++e) dst[e] = src[e];
    }
  }
}

template <int YK, bool RELU2>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full_tma = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
  uint64_t *full_x = full_tma + kStages;
  uint64_t *empty = full_x + kStages;
  uint64_t *done = empty + kStages;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int kblocks = static_cast<int>((p.K + BK - 1) / BK);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_x[s], kExpWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_holder;

  // Everything above overlaps the previous kernel; xq and s are its output.
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % kStages, it = kb / kStages;
        if (kb >= kStages && !mbar_wait(&empty[s], (it - 1) & 1, p.status)) break;
        uint8_t *stage = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full_tma[s], kABytes + kBpBytes);
        tma_load_2d(stage, &tmap_a, kb * BK, static_cast<int32_t>(m0), &full_tma[s]);
        tma_load_2d(stage + kABytes + kBxBytes, &tmap_b, kb * (BK / 4), static_cast<int32_t>(n0),
                    &full_tma[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < kblocks && ok; ++kb) {
        const int s = kb % kStages, it = kb / kStages;
        ok = mbar_wait(&full_tma[s], it & 1, p.status) && mbar_wait(&full_x[s], it & 1, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * kStageBytes);
        const uint32_t b_base = a_base + kABytes;
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk)
          mma_i8(tmem_d, smem_desc_sw128(a_base + 32 * kk), smem_desc_sw128(b_base + 32 * kk),
                 kIdesc, (kb | kk) != 0 ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(done);
    }
  } else {
    // ---- expansion: packed [256 rows x 32 B] -> int8 [256 x 128] K-major SW128
    const int et = (warp - 2) * 32 + lane;
    bool ok = true;
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % kStages, it = kb / kStages;
      if (!mbar_wait(&full_tma[s], it & 1, p.status)) {
        ok = false;
        break;
      }
      uint8_t *stage = smem + s * kStageBytes;
      const uint8_t *bp = stage + kABytes + kBxBytes;
      uint8_t *bx = stage + kABytes;
#pragma unroll
      for (int i = 0; i < (BN * BK / 16) / (32 * kExpWarps); ++i) {
        const int wi = et + 32 * kExpWarps * i;
        const int r = wi >> 3, c = wi & 7;
        const uint32_t w = *reinterpret_cast<const uint32_t *>(bp + r * 32 + c * 4);
        const uint4 v = make_uint4(unpack_natural(w, 0), unpack_natural(w, 1),
                                   unpack_natural(w, 2), unpack_natural(w, 3));
        *reinterpret_cast<uint4 *>(bx + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_x[s]);
    }
    // ---- epilogue: TMEM -> registers -> scale -> Y
    if (ok && mbar_wait(done, 0, p.status)) {
      tc_fence_after();
      const int q = warp & 3;                 // TMEM lane quadrant this warp may access
      const int half = (warp - 2) >> 2;       // which 128 columns
      const int64_t m = m0 + q * 32 + lane;
      const float r = (m < p.M) ? __fdiv_rn(*p.gamma, p.s[m]) : 0.0f;
      const bool vec_ok = (YK == kBF16) ? (p.N % 8 == 0) : (p.N % 4 == 0);
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        const int col = half * 128 + cc * 16;
        uint32_t v[16];
        tmem_ld16(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(col), v);
        tmem_wait_ld();
        if (m < p.M && n0 + col < p.N) store16<YK, RELU2>(p, m, n0 + col, v, r, vec_ok);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_d, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int YK, bool RELU2>
cudaError_t go(const CUtensorMap &ta, const CUtensorMap &tb, const PrefillParams &p,
               const LaunchCtx &ctx) {
  auto kern = prefill_kernel<YK, RELU2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(ceil_div(p.N, BN)), static_cast<unsigned>(ceil_div(p.M, BM)));
  return launch_k(kern, grid, dim3(kThreads), kSmemBytes, ctx, ta, tb, p);
}

}  // namespace

bool prefill_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 1 && N >= 1 && K % 64 == 0 && ceil_div(M, BM) < 65536 && ceil_div(N, BN) < (1LL << 31) &&
         encode_fn() != nullptr;
}

cudaError_t launch_prefill(const int8_t *xq, const float *s, const uint8_t *packed,
                           const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2,
                           void *Y, int y_kind, bool /*weights_static*/, const LaunchCtx &ctx) {
  CUtensorMap ta, tb;
  if (!make_map_2d(&ta, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                   static_cast<uint64_t>(K), BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tb, packed, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N),
                   static_cast<uint64_t>(K / 4), BK / 4, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  PrefillParams p;
  p.s = s;
  p.gamma = gamma;
  p.Y = Y;
  p.status = ctx.status;
  p.M = M;
  p.N = N;
  p.K = K;
  if (y_kind == kI32) return go<kI32, false>(ta, tb, p, ctx);
  if (y_kind == kF32) return relu2 ? go<kF32, true>(ta, tb, p, ctx) : go<kF32, false>(ta, tb, p, ctx);
  return relu2 ? go<kBF16, true>(ta, tb, p, ctx) : go<kBF16, false>(ta, tb, p, ctx);
}

}  // namespace bitnet
