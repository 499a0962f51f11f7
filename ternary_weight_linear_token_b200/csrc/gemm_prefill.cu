// gemm_prefill.cu -- BitLinear forward for prefill-sized batches on the
// fifth-generation tensor cores (tcgen05, kind::i8, int32 accumulators in
// tensor memory).  The contraction is a dense int8 x int8 product: xq times
// the ternary weights {-1, 0, +1} held as int8 (BitNet b1.58 2B4T model card,
// 模型详情 -> 量化: W1.58A8; "Microsoft BitNet 深度研究报告", 技术原理 items 2-3).
//
// The int8 weights come from the packed ones by a coalesced expansion pass
// beforehand (launched with the activation quantiser: 4.4 MB in, 17.7 MB out
// for 6912 x 2560), in the K order of the activations.
// prefill_kernel: persistent, K in 128-byte stages, two 256-column int32
// accumulators in TMEM (512 columns) so that tile i's epilogue overlaps tile
// i+1's MMAs.  Two forms:
//   CTA pairs (M > 128; clusters of two CTAs on two SMs, cta_group::2):
//     output tiles of 256 tokens x 256 features taken round-robin by the
//     pairs.  Each CTA's TMA warp (4) loads its own 128 token rows of xq and
//     its own 128 feature rows of the int8 weights (128-byte swizzled, 6-stage
//     ring of 16 + 16 KB); both CTAs' bytes complete on the first CTA's
//     barrier (.cta_group::2 loads, no multicast).  One lane of the first
//     CTA's warp 5 issues 4 pair MMAs (M=256, N=256, K=32) per stage, A and
//     B read from both CTAs' shared memory at the same offsets, and commits
//     with .multicast::cluster to both CTAs' stage-empty and
//     accumulator-full barriers.  D rows 0-127 land in the first CTA's TMEM,
//     128-255 in the second's.
//   single CTAs (M <= 128): tiles of 128 tokens x 256 features, a 4-stage
//     ring of 16 + 32 KB, M=128 MMAs.
//   warps 0-3 (every CTA) epilogue: tcgen05.ld of its 128 accumulator rows,
//     y = acc * (gamma / s_m), optional ReLU^2; bf16 output goes through a
//     128-byte-swizzled shared-memory staging block (32 rows x 64 columns per
//     warp, double-buffered) and a TMA tensor store, so HBM sees whole
//     lines; then the accumulator is released (in a pair, with a
//     cluster-scope arrive on the first CTA's barrier: 8 arrivals).
// Expanding in HBM first keeps shared memory for the tensor core's operands
// only; the pair form halves each SM's share of them to 32 KB of TMA writes
// and 32 KB of operand reads per stage, under what the MMAs take.  Every wait
// is bounded (see common.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "quant_row.cuh"

namespace bitnet {
namespace {

constexpr int BM = 128;                           // token rows per CTA
constexpr int BN = 256;                           // features per accumulator
constexpr int BK = 128;
constexpr int kEpiWarps = 4;
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kThreads = 32 * (kEpiWarps + 2);
// The fused form adds warps that prepare the operands (quantise the token
// rows, expand the packed weight rows) while the pipeline runs.
constexpr int kPrepWarps = 6;
constexpr int kWarpPrep0 = kEpiWarps + 2;
constexpr int kThreadsFused = 32 * (kEpiWarps + 2 + kPrepWarps);
constexpr int kReadyStride = 8;  // readiness counters 32 bytes apart
constexpr int kABytes = BM * BK;
constexpr int kTmemCols = 2 * BN;
constexpr int kStoreRows = 32;                    // epilogue staging block: 32 rows
constexpr int kStoreCols = 64;                    // x 64 bf16 columns = 128-byte rows
constexpr int kStoreBytes = kStoreRows * kStoreCols * 2;
constexpr int kMaxDevices = 64;

// One CTA: a 128 x 256 tile, A 16 KB + B 32 KB per stage, 4 stages.  A pair
// (cta_group::2): a 256 x 256 tile, each CTA holding 128 token rows of A and
// 128 feature rows of B, 16 KB + 16 KB per stage, 6 stages.
template <bool PAIR> struct Cfg {
  static constexpr int kBRows = PAIR ? BN / 2 : BN;
  static constexpr int kStages = PAIR ? 6 : 4;
  static constexpr int kStageBytes = kABytes + kBRows * BK;
  static constexpr int kTileM = PAIR ? 2 * BM : BM;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes +
                                       kEpiWarps * 2 * kStoreBytes + 256;
  // Instruction descriptor: s8 x s8 -> s32, both operands K-major, M = kTileM, N = 256.
  static constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((BN >> 3) << 17) |
                                     ((kTileM >> 4) << 24);
};

struct PrefillParams {
  const float *s;
  const float *gamma;
  void *Y;
  int *status;
  int64_t M, N, K;
  int m_tiles, n_tiles;
  // the fused form: operands prepared inside the kernel.  ready[] counts the
  // rows done per block of a tile's token rows (m_tiles of them), then per
  // 256-row block of weights (n_tiles); a tile's loads wait for both.
  const void *X;        // raw activations (fp32/bf16), or null: xq is given
  int x_kind;
  int8_t *xq;           // where the quantised activations go (TMA source)
  float *s_out;         // their scales (== s)
  const uint8_t *packed;
  int8_t *w8;           // where the expanded weights go (TMA source)
  int expand;           // 0: w8 already holds them
  unsigned *ready;
};

// Rows of token block b (tile_m rows each) and of weight block b (BN rows).
__host__ __device__ inline int block_rows(int64_t total, int64_t rows_per_block, int b) {
  const int64_t r = total - static_cast<int64_t>(b) * rows_per_block;
  return static_cast<int>(r < rows_per_block ? r : rows_per_block);
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Bounded wait (one thread) until a readiness counter reaches `want`, with
// acquire semantics; then the async proxy (the TMA) may read what the
// counted rows' writers stored.  False after recording a timeout.
__device__ __forceinline__ bool wait_ready(const unsigned *ctr, unsigned want, int *status) {
  if (ld_acquire_u32(ctr) != want) {
    const long long t0 = clock64();
    while (ld_acquire_u32(ctr) != want) {
      if (clock64() - t0 > kWaitLimitCycles) {
        record_status(status, kStatusTimeout);
        return false;
      }
    }
  }
  fence_proxy_async_global();
  return true;
}

// The counters of a fused launch: each token block starts at 0 when the
// kernel quantises (else complete), each weight block at 0 when it expands.
__global__ void prep_reset_kernel(unsigned *ready, int m_tiles, int n_tiles, int64_t M, int64_t N,
                                  int tile_m, int quantize, int expand) {
  pdl_launch_dependents();
  pdl_wait();  // the previous kernel may still be reading the counters
  for (int i = threadIdx.x; i < m_tiles + n_tiles; i += blockDim.x) {
    unsigned v;
    if (i < m_tiles)
      v = quantize ? 0u : static_cast<unsigned>(block_rows(M, tile_m, i));
    else
      v = expand ? 0u : static_cast<unsigned>(block_rows(N, BN, i - m_tiles));
    ready[static_cast<size_t>(i) * kReadyStride] = v;
  }
}

// A batch of weight rows expanded by one warp with all of its loads in
// flight at once (kExpandWordsInFlight packed words per lane), then one
// proxy fence per lane and one release count per row.
constexpr int kExpandWordsInFlight = 32;
template <bool PERM>
__device__ __forceinline__ void expand_rows_batch(const PrefillParams &p, int64_t n_first,
                                                  int64_t n_step, int count, int lane) {
  const int words = static_cast<int>(p.K / 16);
  const uint32_t *src = reinterpret_cast<const uint32_t *>(p.packed);
  uint4 *dst = reinterpret_cast<uint4 *>(p.w8);
  uint32_t v[kExpandWordsInFlight];
  // flat index i over (row j, word w) of the batch, lane-strided
  const int total = count * words;
#pragma unroll
  for (int k = 0; k < kExpandWordsInFlight; ++k) {
    const int i = lane + 32 * k;
    v[k] = 0u;
    if (i < total) {
      const int j = i / words, w = i - j * words;
      v[k] = src[(n_first + n_step * j) * words + w];
    }
  }
#pragma unroll
  for (int k = 0; k < kExpandWordsInFlight; ++k) {
    const int i = lane + 32 * k;
    if (i < total) {
      const int j = i / words, w = i - j * words;
      dst[(n_first + n_step * j) * words + w] = expand_word<PERM>(v[k]);
    }
  }
  fence_proxy_async_global();
  __syncwarp();
  if (lane < count)
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(
                     p.ready + static_cast<size_t>(p.m_tiles + (n_first + n_step * lane) / BN) * kReadyStride)
                 : "memory");
}

// One prep warp's share of the operand preparation, in the order the tiles
// need it (tiles go token block by token block, all weight blocks each):
// this CTA's rows of the first three token blocks, then its weight rows,
// then its other token rows.  Row r is this CTA's when r % ctas == cta;
// warp q of the CTA takes every kPrepWarps-th of those.  After each token
// row, and after each batch of weight rows, the warp makes its stores
// visible to the TMA and counts the rows in, with release semantics.
template <int KIND, bool PERM>
__device__ __forceinline__ void prep_work(const PrefillParams &p, int tile_m, int cta, int ctas,
                                          int q, int lane) {
  const int64_t early = static_cast<int64_t>(tile_m) * 3;
  const int64_t step = static_cast<int64_t>(ctas) * kPrepWarps;
  auto tokens = [&](int64_t lo, int64_t hi) {
    if (p.X == nullptr) return;
    for (int64_t m = cta + static_cast<int64_t>(ctas) * q; m < hi; m += step) {
      if (m < lo) continue;
      quantize_row_warp<KIND, PERM>(p.X, m, p.K, lane, p.xq, p.s_out);
      fence_proxy_async_global();
      __syncwarp();
      if (lane == 0)
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(
                         p.ready + static_cast<size_t>(m / tile_m) * kReadyStride)
                     : "memory");
    }
  };
  tokens(0, early < p.M ? early : p.M);
  if (p.expand) {
    const int words = static_cast<int>(p.K / 16);
    int batch = kExpandWordsInFlight * 32 / words;  // rows whose words fit in flight at once
    if (batch > 32) batch = 32;
    if (batch >= 1) {
      for (int64_t n = cta + static_cast<int64_t>(ctas) * q; n < p.N; n += step * batch) {
        const int64_t left = (p.N - 1 - n) / step + 1;
        expand_rows_batch<PERM>(p, n, step, static_cast<int>(left < batch ? left : batch), lane);
      }
    } else {  // long rows: one at a time
      for (int64_t n = cta + static_cast<int64_t>(ctas) * q; n < p.N; n += step) {
        expand_row_warp<PERM>(p.packed, p.w8, n, p.K, lane);
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0)
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(
                           p.ready + static_cast<size_t>(p.m_tiles + n / BN) * kReadyStride)
                       : "memory");
      }
    }
  }
  tokens(early, p.M);
}

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
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (e < valid) dst[e] = static_cast<int>(v[e]);
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
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (e < valid) dst[e] = y[e];
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
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (e < valid) {
          const uint32_t bits = (h[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
          reinterpret_cast<uint16_t *>(dst)[e] = static_cast<uint16_t>(bits);
        }
    }
  }
}

// PAIR: launched as clusters of two CTAs; the first issues the pair MMAs for
// both, each loads its own halves of A and B and writes its own 128 rows.
template <int YK, bool RELU2, bool TMA_Y, bool PAIR, bool FUSED>
__global__ void __launch_bounds__(FUSED ? kThreadsFused : kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ CUtensorMap tmap_y, const PrefillParams p) {
  using C = Cfg<PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;                                   // [stages][A 16 KB | B]
  uint8_t *staging = ring + C::kStages * C::kStageBytes;  // [kEpiWarps][2][32 x 128 B]
  uint64_t *full = reinterpret_cast<uint64_t *>(staging + kEpiWarps * 2 * kStoreBytes);
  uint64_t *empty = full + C::kStages;
  uint64_t *acc_full = empty + C::kStages;
  uint64_t *acc_empty = acc_full + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = static_cast<int>((p.K + BK - 1) / BK);
  const int tiles = p.m_tiles * p.n_tiles;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (warp == kWarpTma && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], PAIR ? 2 * kEpiWarps : kEpiWarps);  // the pair's epilogues
    }
    fence_barrier_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if (TMA_Y) prefetch_tmap(&tmap_y);
  }
  if (warp == kWarpMma) {
    tmem_alloc<PAIR>(tmem_holder, kTmemCols);
    tmem_relinquish<PAIR>();
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();  // both CTAs' barriers and TMEM exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // Everything above overlaps the previous kernel; xq, s and the int8
  // weights are its output.
  pdl_wait();
  pdl_launch_dependents();

  if (warp == kWarpTma) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = unit; tile < tiles && ok; tile += units) {
        const int32_t m0 = (tile / p.n_tiles) * C::kTileM + static_cast<int32_t>(rank) * BM;
        const int32_t n0 = (tile % p.n_tiles) * BN + static_cast<int32_t>(rank) * C::kBRows;
        if (FUSED) {  // the tile's token rows and weight rows are prepared
          const int mb = tile / p.n_tiles, nb = tile % p.n_tiles;
          ok = wait_ready(p.ready + static_cast<size_t>(mb) * kReadyStride,
                          static_cast<unsigned>(block_rows(p.M, C::kTileM, mb)), p.status) &&
               wait_ready(p.ready + static_cast<size_t>(p.m_tiles + nb) * kReadyStride,
                          static_cast<unsigned>(block_rows(p.N, BN, nb)), p.status);
          if (!ok) break;
        }
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::kStages;
          if (it >= C::kStages &&
              !mbar_wait<PAIR>(&empty[s], ((it / C::kStages) - 1) & 1, p.status)) {
            ok = false;
            break;
          }
          uint8_t *stage = ring + s * C::kStageBytes;
          if (PAIR) {
            // both CTAs' halves complete on the first CTA's barrier
            if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::kStageBytes);
            const uint32_t bar0 = mapa_shared(&full[s], 0);
            tma_load_2d_pair(stage, &tmap_a, kb * BK, m0, bar0);
            tma_load_2d_pair(stage + kABytes, &tmap_b, kb * BK, n0, bar0);
          } else {
            mbar_arrive_expect_tx(&full[s], C::kStageBytes);
            tma_load_2d(stage, &tmap_a, kb * BK, m0, &full[s]);
            tma_load_2d(stage + kABytes, &tmap_b, kb * BK, n0, &full[s]);
          }
        }
      }
    }
  } else if (warp == kWarpMma) {
    if (lane == 0 && leader) {
      uint32_t it = 0;
      bool ok = true;
      int tl = 0;
      for (int tile = unit; tile < tiles && ok; tile += units, ++tl) {
        const int acc = tl & 1;
        if (tl >= 2 && !mbar_wait<PAIR>(&acc_empty[acc], ((tl >> 1) - 1) & 1, p.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::kStages;
          ok = mbar_wait<PAIR>(&full[s], (it / C::kStages) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(ring + s * C::kStageBytes);
          const uint32_t b_base = a_base + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t ad = smem_desc_sw128(a_base + 32 * kk);
            const uint64_t bd = smem_desc_sw128(b_base + 32 * kk);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if (PAIR)
              mma_i8_pair(d, ad, bd, C::kIdesc, accum);
            else
              mma_i8(d, ad, bd, C::kIdesc, accum);
          }
          if (PAIR)
            mma_commit_pair(&empty[s]);
          else
            mma_commit(&empty[s]);
        }
        if (PAIR)
          mma_commit_pair(&acc_full[acc]);
        else
          mma_commit(&acc_full[acc]);
      }
    }
  } else if (FUSED && warp >= kWarpPrep0) {
    // ---- prep warps: quantise token rows, expand weight rows
    const int cta = static_cast<int>(blockIdx.x), ctas = static_cast<int>(gridDim.x);
    const int q = warp - kWarpPrep0;
    if (p.x_kind == kF32)
      prep_work<kF32, true>(p, C::kTileM, cta, ctas, q, lane);
    else if (p.x_kind == kBF16)
      prep_work<kBF16, true>(p, C::kTileM, cta, ctas, q, lane);
    else
      prep_work<kBF16, false>(p, C::kTileM, cta, ctas, q, lane);  // int8 given: expansion only
  } else {
    // ---- epilogue warps 0-3: TMEM lane quadrant = warp
    const int q = warp;
    const float gamma = *p.gamma;
    const bool vec_ok = (YK == kBF16) ? (p.N % 8 == 0) : (p.N % 4 == 0);
    uint8_t *my_stage = staging + q * 2 * kStoreBytes;
    // the accumulator is released to the pair's first CTA (its MMA reuses it)
    const uint32_t acc_empty0_a = PAIR ? mapa_shared(&acc_empty[0], 0) : 0u;
    const uint32_t acc_empty0_b = PAIR ? mapa_shared(&acc_empty[1], 0) : 0u;
    int tl = 0, stores = 0;
    for (int tile = unit; tile < tiles; tile += units, ++tl) {
      const int acc = tl & 1;
      if (!mbar_wait<PAIR>(&acc_full[acc], (tl >> 1) & 1, p.status)) break;
      tc_fence_after();
      const int64_t m_base = static_cast<int64_t>(tile / p.n_tiles) * C::kTileM +
                             static_cast<int64_t>(rank) * BM + q * 32;
      const int64_t m = m_base + lane;
      const int64_t n0 = static_cast<int64_t>(tile % p.n_tiles) * BN;
      if (FUSED) {  // the scales come from the prep warps (complete once the tile ran)
        if (lane == 0) (void)ld_acquire_u32(p.ready + static_cast<size_t>(tile / p.n_tiles) * kReadyStride);
        __syncwarp();
      }
      const float r = (m < p.M) ? __fdiv_rn(gamma, p.s[m]) : 0.0f;
      const uint32_t t_row = tmem_base + static_cast<uint32_t>(acc * BN) +
                             (static_cast<uint32_t>(q * 32) << 16);
      if (TMA_Y) {
#pragma unroll 1
        for (int cb = 0; cb < BN / kStoreCols; ++cb, ++stores) {
          uint8_t *buf = my_stage + (stores & 1) * kStoreBytes;
          if (stores >= 2) {  // the store that last used this buffer has read it
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t v[32];
            tmem_ld16(t_row + static_cast<uint32_t>(cb * kStoreCols + 32 * half),
                      *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
            tmem_ld16(t_row + static_cast<uint32_t>(cb * kStoreCols + 32 * half + 16),
                      *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            tmem_wait_ld();
            if (cb == BN / kStoreCols - 1 && half == 1) {  // accumulator fully read
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if (PAIR)
                  mbar_arrive_remote(acc ? acc_empty0_b : acc_empty0_a);
                else
                  mbar_arrive(&acc_empty[acc]);
              }
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {  // 8 columns = 16 bytes per chunk, swizzled
              const int c = 4 * half + c4;
              uint32_t h[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(
                    epilogue_value(static_cast<int>(v[8 * c4 + 2 * e]), r, RELU2),
                    epilogue_value(static_cast<int>(v[8 * c4 + 2 * e + 1]), r, RELU2));
                h[e] = *reinterpret_cast<const uint32_t *>(&b);
              }
              *reinterpret_cast<uint4 *>(buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(h[0], h[1], h[2], h[3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmap_y, buf, static_cast<int32_t>(n0 + cb * kStoreCols),
                         static_cast<int32_t>(m_base));
            bulk_commit();
          }
        }
      } else {
#pragma unroll 1
        for (int cc = 0; cc < BN / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(t_row + static_cast<uint32_t>(cc * 16), v);
          tmem_wait_ld();
          if (m < p.M && n0 + cc * 16 < p.N) store16<YK, RELU2>(p, m, n0 + cc * 16, v, r, vec_ok);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR)
            mbar_arrive_remote(acc ? acc_empty0_b : acc_empty0_a);
          else
            mbar_arrive(&acc_empty[acc]);
        }
      }
    }
    if (TMA_Y && lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  // the other CTA of a pair may still be signalled by (or signal) this one's
  // barriers and TMEM until both are done
  if (PAIR) cluster_sync();
  if (warp == kWarpMma) tmem_dealloc<PAIR>(tmem_base, kTmemCols);
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
                 CUtensorMapSwizzle swz,
                 CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_UINT8) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int YK, bool RELU2, bool TMA_Y, bool PAIR, bool FUSED>
cudaError_t go(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &ty,
               const PrefillParams &p, const LaunchCtx &ctx) {
  using C = Cfg<PAIR>;
  auto kern = prefill_kernel<YK, RELU2, TMA_Y, PAIR, FUSED>;
  const int threads = FUSED ? kThreadsFused : kThreads;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  if (!PAIR) {
    const dim3 grid(static_cast<unsigned>(tiles < ctx.num_sms ? tiles : ctx.num_sms));
    return launch_k(kern, grid, dim3(threads), C::kSmemBytes, ctx, ta, tb, ty, p);
  }
  // as many pairs as the device can hold at once (asked once per device and
  // form); none: the caller runs single CTAs
  static std::atomic<int> resident[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int most = resident[dev].load(std::memory_order_relaxed);
  if (most == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * (ctx.num_sms / 2)));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    most = n > 0 ? n : -1;
    resident[dev].store(most, std::memory_order_relaxed);
  }
  if (most < 1) return cudaErrorInvalidClusterSize;
  int64_t pairs = ctx.num_sms / 2;
  if (pairs > most) pairs = most;
  const dim3 grid(static_cast<unsigned>(2 * (tiles < pairs ? tiles : pairs)));
  return launch_k_cluster(kern, grid, dim3(threads), C::kSmemBytes, 2u, ctx, ta, tb, ty, p);
}

template <bool PAIR, bool FUSED>
cudaError_t go_y(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &ty, bool tma_y,
                 const PrefillParams &p, int y_kind, bool relu2, const LaunchCtx &ctx) {
  if (y_kind == kI32) return go<kI32, false, false, PAIR, FUSED>(ta, tb, ty, p, ctx);
  if (y_kind == kF32)
    return relu2 ? go<kF32, true, false, PAIR, FUSED>(ta, tb, ty, p, ctx)
                 : go<kF32, false, false, PAIR, FUSED>(ta, tb, ty, p, ctx);
  if (tma_y)
    return relu2 ? go<kBF16, true, true, PAIR, FUSED>(ta, tb, ty, p, ctx)
                 : go<kBF16, false, true, PAIR, FUSED>(ta, tb, ty, p, ctx);
  return relu2 ? go<kBF16, true, false, PAIR, FUSED>(ta, tb, ty, p, ctx)
               : go<kBF16, false, false, PAIR, FUSED>(ta, tb, ty, p, ctx);
}

template <bool PAIR>
cudaError_t go_f(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &ty, bool tma_y,
                 const PrefillParams &p, int y_kind, bool relu2, const LaunchCtx &ctx) {
  if (p.ready == nullptr) return go_y<PAIR, false>(ta, tb, ty, tma_y, p, y_kind, relu2, ctx);
  // the counters first: a one-CTA kernel, launched as the fused kernel's predecessor
  const bool quantize = p.X != nullptr;
  const cudaError_t e = launch_k(prep_reset_kernel, dim3(1), dim3(256), 0, ctx, p.ready, p.m_tiles,
                                 p.n_tiles, p.M, p.N, Cfg<PAIR>::kTileM, quantize ? 1 : 0, p.expand);
  if (e != cudaSuccess) return e;
  return go_y<PAIR, true>(ta, tb, ty, tma_y, p, y_kind, relu2, ctx);
}

}  // namespace

bool prefill_shape_ok(int64_t M, int64_t N, int64_t K) {
  return M >= 1 && N >= 1 && K % 64 == 0 && ceil_div(M, BM) * ceil_div(N, BN) < (1LL << 31);
}

bool prefill_supported(int64_t M, int64_t N, int64_t K) {
  return prefill_shape_ok(M, N, K) && encode_fn() != nullptr;
}

size_t prefill_weight_bytes(int64_t N, int64_t K) { return static_cast<size_t>(N) * K; }

size_t prefill_ready_bytes(int64_t M, int64_t N) {
  return static_cast<size_t>(4 * kReadyStride) * static_cast<size_t>(ceil_div(M, BM) + ceil_div(N, BN));
}

cudaError_t launch_prefill(const int8_t *xq, const float *s, const int8_t *w8,
                           const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2,
                           void *Y, int y_kind, const LaunchCtx &ctx, const PrefillPrep *prep) {
  PrefillParams p;
  p.s = s;
  p.gamma = gamma;
  p.Y = Y;
  p.status = ctx.status;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_tiles = static_cast<int>(ceil_div(N, BN));
  p.X = nullptr;
  p.x_kind = kI8;
  p.xq = const_cast<int8_t *>(xq);
  p.s_out = const_cast<float *>(s);
  p.packed = nullptr;
  p.w8 = const_cast<int8_t *>(w8);
  p.expand = 0;
  p.ready = nullptr;
  if (prep != nullptr && (prep->X != nullptr || prep->packed != nullptr)) {
    p.X = prep->X;
    p.x_kind = prep->X != nullptr ? prep->x_kind : kI8;
    p.packed = prep->packed;
    p.expand = prep->packed != nullptr ? 1 : 0;
    p.ready = prep->ready;
  }
  CUtensorMap ta, tb, ty;
  if (!make_map_2d(&ta, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                   static_cast<uint64_t>(K), BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // bf16 output with 16-byte rows goes out through TMA tensor stores
  const bool tma_y = y_kind == kBF16 && N % 8 == 0 &&
                     make_map_2d(&ty, Y, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                                 static_cast<uint64_t>(N) * 2, kStoreCols, kStoreRows,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  if (!tma_y) ty = ta;  // unused by the direct-store kernels
  // more than one 128-token block: CTA pairs on 256-token tiles
  if (M > BM && ctx.num_sms >= 2) {
    if (!make_map_2d(&tb, w8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                     static_cast<uint64_t>(K), BK, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    p.m_tiles = static_cast<int>(ceil_div(M, 2 * BM));
    const cudaError_t e = go_f<true>(ta, tb, ty, tma_y, p, y_kind, relu2, ctx);
    if (e != cudaErrorInvalidClusterSize) return e;  // else: no pair fits, single CTAs
  }
  if (!make_map_2d(&tb, w8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                   static_cast<uint64_t>(K), BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  p.m_tiles = static_cast<int>(ceil_div(M, BM));
  return go_f<false>(ta, tb, ty, tma_y, p, y_kind, relu2, ctx);
}

}  // namespace bitnet
