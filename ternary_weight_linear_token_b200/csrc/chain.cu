// chain.cu -- a chain of M = 1 BitLinear projections in one persistent launch.
//
// A decode step of a BitNet b1.58 model runs its projections one after the
// other, and each takes the previous one's output, re-quantised per token,
// as its input.  Launched one kernel per projection, every link pays a kernel
// launch, a grid-dependency wait and an activation prologue, which at these
// sizes (1.6 to 4.4 MB of packed weights per projection) cost several times
// the weight stream itself.  This kernel walks the whole chain in one
// cooperative launch, one CTA per SM:
//   * Weights do not depend on the activations, so a producer warp streams
//     every projection's packed rows for this CTA into a ring of shared-memory
//     slots (one bulk copy per projection, L2 evict-first) as far ahead as the
//     ring allows, while the consumer warps are still on earlier links.
//   * A link's outputs travel through L2 as tagged 64-bit words (two bf16
//     values and a 32-bit tag unique to this launch, written with one relaxed
//     64-bit store, so data and tag are seen together).  The tag is the
//     launch counter kept in the workspace plus one; the counter advances
//     once every CTA has finished.
//   * Each CTA, once its outputs of a link are out, also publishes two tagged
//     words: the max |y| and the sum of y^2 of its outputs that the next link
//     reads.  They are the CTA's "done" flag, and they are what the next link
//     needs to quantise (s = 127 / max |x|) and, where a layer starts, to
//     normalise (the weightless RMS normalisation).  One warp per CTA polls
//     the records of all CTAs (2 words each), reduces them in a fixed order
//     and computes the scale once; only then do all threads load the data
//     words, once.  So no CTA repeats the reductions over the whole vector,
//     and the polling traffic stays a few KB per round.
//   * Per link, each CTA quantises the whole input to int8 exactly as
//     bitnet_quantize_act does and computes its balanced range of output
//     features with the byte-permute unpack and dp4a, in the same int32
//     arithmetic and with the same epilogue as bitnet_w158a8_matmul.
// Every wait is bounded: a poll, an mbarrier wait or the final counter wait
// that gives up records BITNET_ERR_TIMEOUT and the CTA stops at the next
// step boundary, after its bulk copies in flight have landed.
#include "common.cuh"
#include "internal.h"

namespace bitnet {
namespace {

constexpr int kCWarps = 16;                 // consumer warps
constexpr int kCThreads = 32 * kCWarps;     // consumer threads
constexpr int kThreads = kCThreads + 32;    // + the producer warp
constexpr int kMaxSlots = 8;
constexpr int kMaxCtas = kChainMaxCtas;     // stats records per step
constexpr int kSmemLimit = 227 * 1024;
constexpr int kHeader = 1024;
constexpr int kBarConsumers = 1;            // named barrier of the consumer warps
constexpr uint32_t kTernaryLut = 0xFFFF0100u;  // code 0 -> 0, 1 -> +1, 2 -> -1, 3 -> -1
constexpr int kMaxWordsPerThread = 8;       // K <= 8192: at most 4096 input words

__host__ __device__ constexpr int align128(int n) { return (n + 127) / 128 * 128; }
// Shared-memory copies made once at the start: the step descriptors, every
// step's gamma and this CTA's row range of every step.
__host__ __device__ constexpr int table_bytes(int n_steps) {
  return align128(n_steps * 48) + align128(n_steps * 4) + align128(n_steps * 8);
}

struct __align__(8) StepP {
  const uint8_t *packed;
  const float *gamma;
  uint16_t *Y;       // bf16 [N]
  uint16_t *Xn;      // bf16 [K] normalised input, or null
  int N, K;
  int flags;         // kStepRelu2 | kStepNormIn
  int out_off;       // this step's exchange words, in 64-bit words from xch
};

struct ChainP {
  const uint16_t *x0;
  uint16_t *y_norm;
  unsigned long long *xch;    // [kChainReplicas][xch_words]
  unsigned long long *stats;  // [kChainReplicas][n_steps][kMaxCtas][2]: tagged max |y|, sum y^2
  unsigned int *epoch;
  unsigned int *done;
  int *status;
  int n_steps, ctas, slots, slot_bytes, xq_bytes, ystage_bytes, y_norm_n;
  int xch_words;  // exchange words of one copy
  StepP steps[kChainMaxSteps];
};

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(kBarConsumers), "n"(kCThreads) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// Contiguous global -> shared bulk copy with an L2 cache hint, completed on
// an mbarrier.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Rows [r0, r1) of an N-row projection owned by CTA c: whole pairs of rows
// (one exchange word each), balanced over the CTAs.
__host__ __device__ inline void cta_rows(int N, int c, int ctas, int &r0, int &r1) {
  const long long pairs = (N + 1) / 2;
  r0 = static_cast<int>(2 * (pairs * c / ctas));
  const int e = static_cast<int>(2 * (pairs * (c + 1) / ctas));
  r1 = e < N ? e : N;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t bf16_bits(float y) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(y)));
}
__device__ __forceinline__ float round_bf16(float y) { return __uint_as_float(bf16_bits(y) << 16); }

// Polls this thread's exchange words of one input vector (words tid + i *
// kCThreads below nwords) until each carries `tag`, re-reading only those not
// yet seen, with a short sleep between rounds.  The loads of a round go out
// together and are coalesced across the warp.  Returns false (after
// recording a timeout) if some word never gets there.
__device__ __forceinline__ bool poll_words(const unsigned long long *src, int nwords, int tid,
                                           unsigned tag, uint32_t (&w)[kMaxWordsPerThread],
                                           int *status) {
  uint32_t pending = 0;
#pragma unroll
  for (int i = 0; i < kMaxWordsPerThread; ++i)
    if (tid + i * kCThreads < nwords) pending |= 1u << i;
  long long t0 = 0;
  bool started = false;
  while (pending != 0) {
    unsigned long long got[kMaxWordsPerThread];
#pragma unroll
    for (int i = 0; i < kMaxWordsPerThread; ++i)
      if (pending & (1u << i)) got[i] = ld_relaxed_u64(src + tid + i * kCThreads);
#pragma unroll
    for (int i = 0; i < kMaxWordsPerThread; ++i) {
      if ((pending & (1u << i)) && static_cast<unsigned>(got[i] >> 32) == tag) {
        w[i] = static_cast<uint32_t>(got[i]);
        pending &= ~(1u << i);
      }
    }
    if (pending == 0) break;
    if (!started) {
      started = true;
      t0 = clock64();
    } else if (clock64() - t0 > kWaitLimitCycles) {
      record_status(status, kStatusTimeout);
      return false;
    }
    __nanosleep(32);
  }
  return true;
}

// One warp waits until every CTA has published its record for a step, then
// reduces them in a fixed order (CTA c's record is read by lane c % 32; lane
// sums in order of c, then a butterfly).  a = max |y|, ss = sum y^2 over
// the part of the step's output that the next step reads; lane 0's values
// are the result.  Warp-uniform return; false after recording a timeout.
__device__ __forceinline__ bool poll_stats(const unsigned long long *rec, int ctas, unsigned tag,
                                           int lane, float &a, float &ss, int *status) {
  constexpr int kPer = kMaxCtas / 32;
  unsigned long long m[kPer], q[kPer];
  const long long t0 = clock64();
  while (true) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (lane + 32 * i < ctas) {
        m[i] = ld_relaxed_u64(rec + 2 * (lane + 32 * i));
        q[i] = ld_relaxed_u64(rec + 2 * (lane + 32 * i) + 1);
      }
    }
    bool mine = true;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (lane + 32 * i < ctas)
        mine = mine && static_cast<unsigned>(m[i] >> 32) == tag &&
               static_cast<unsigned>(q[i] >> 32) == tag;
    if (__all_sync(0xffffffffu, mine)) break;
    if (__shfl_sync(0xffffffffu, static_cast<int>(clock64() - t0 > kWaitLimitCycles), 0)) {
      record_status(status, kStatusTimeout);
      return false;
    }
    __nanosleep(256);  // 148 pollers on the same few lines: leave room for the stores
  }
  a = 0.0f;
  ss = 0.0f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    if (lane + 32 * i < ctas) {
      a = fmaxf(a, __uint_as_float(static_cast<uint32_t>(m[i])));
      ss = __fadd_rn(ss, __uint_as_float(static_cast<uint32_t>(q[i])));
    }
  }
  a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
  return true;
}

// Bounded mbarrier wait that also gives up when the CTA is stopping.
__device__ __forceinline__ bool wait_or_stop(uint64_t *bar, uint32_t parity,
                                             const volatile int *stop, int *status) {
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*stop) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      record_status(status, kStatusTimeout);
      return false;
    }
  }
}

// Byte position of element e (0..15) of a 16-element group in the unpack
// order {0,8,1,9}, {2,10,3,11}, {4,12,5,13}, {6,14,7,15}.
__device__ __forceinline__ int unpack_pos(int e) { return ((e & 7) << 1) | (e >> 3); }

// The 16 int8 weights of a packed word as four dp4a operands, in the order
// of the activations in shared memory (selector shifts 0, 16, 2, 18: elements
// {0,8,1,9}, {2,10,3,11}, {4,12,5,13}, {6,14,7,15} of the group).
__device__ __forceinline__ int dot_word(uint32_t w, uint4 x, int acc) {
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, w & 0x3333u)), static_cast<int>(x.x), acc);
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, (w >> 16) & 0x3333u)), static_cast<int>(x.y), acc);
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, (w >> 2) & 0x3333u)), static_cast<int>(x.z), acc);
  acc = __dp4a(static_cast<int>(__byte_perm(kTernaryLut, 0u, (w >> 18) & 0x3333u)), static_cast<int>(x.w), acc);
  return acc;
}

// Dot product of one packed row (words lane, lane + 32, ...) with the int8
// activations, four words per lane in flight; the warp's total.
__device__ __forceinline__ int row_dot(const uint32_t *wrow, const uint4 *x4, int words, int lane) {
  int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
  int w = lane;
  for (; w + 96 < words; w += 128) {
    const uint32_t q0 = wrow[w], q1 = wrow[w + 32], q2 = wrow[w + 64], q3 = wrow[w + 96];
    const uint4 x0 = x4[w], x1 = x4[w + 32], x2 = x4[w + 64], x3 = x4[w + 96];
    a0 = dot_word(q0, x0, a0);
    a1 = dot_word(q1, x1, a1);
    a2 = dot_word(q2, x2, a2);
    a3 = dot_word(q3, x3, a3);
  }
  for (; w < words; w += 32) a0 = dot_word(wrow[w], x4[w], a0);
  return __reduce_add_sync(0xffffffffu, (a0 + a1) + (a2 + a3));
}

// 1 / sqrt(mean(x^2) + 1e-6), the weightless RMS normalisation's factor.
__device__ __forceinline__ float rms_inv(float ss, int K) {
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, static_cast<float>(K)), 1e-6f)));
}

__global__ void __launch_bounds__(kThreads, 1) chain_kernel(const __grid_constant__ ChainP P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);                // [kMaxSlots]
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + 64);          // [kMaxSlots]
  float *red_a = reinterpret_cast<float *>(smem + 128);               // [kCWarps]
  float *red_s = reinterpret_cast<float *>(smem + 192);               // [kCWarps]
  volatile int *stop = reinterpret_cast<volatile int *>(smem + 256);
  int *issued_sh = reinterpret_cast<int *>(smem + 260);
  int *consumed_sh = reinterpret_cast<int *>(smem + 264);
  // `stop` as thread 0 saw it before the last consumer barrier: the value
  // every consumer acts on, so that all of them leave the loop together.
  int *stop_snap = reinterpret_cast<int *>(smem + 268);
  float *par = reinterpret_cast<float *>(smem + 272);                 // scale, gamma/scale, 1/rms
  StepP *tab = reinterpret_cast<StepP *>(smem + kHeader);            // [n_steps]
  float *gam = reinterpret_cast<float *>(smem + kHeader + align128(P.n_steps * 48));
  int2 *rr = reinterpret_cast<int2 *>(smem + kHeader + align128(P.n_steps * 48) +
                                      align128(P.n_steps * 4));       // this CTA's rows
  uint16_t *ystage = reinterpret_cast<uint16_t *>(smem + kHeader + table_bytes(P.n_steps));
  uint8_t *xq = smem + kHeader + table_bytes(P.n_steps) + P.ystage_bytes;  // [xq_bytes]
  uint8_t *slots = xq + P.xq_bytes;                                   // [slots][slot_bytes]
  const uint4 *xq4 = reinterpret_cast<const uint4 *>(xq);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < P.slots; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kCWarps);
    }
    *stop = 0;
    *stop_snap = 0;
    *issued_sh = 0;
    *consumed_sh = 0;
    fence_barrier_init();
  }
  {
    static_assert(sizeof(StepP) == 48, "descriptor size");
    const uint2 *src = reinterpret_cast<const uint2 *>(&P.steps[0]);
    uint2 *dst = reinterpret_cast<uint2 *>(tab);
    for (int i = tid; i < P.n_steps * 6; i += kThreads) dst[i] = src[i];
    for (int i = tid; i < P.n_steps; i += kThreads) {
      gam[i] = *P.steps[i].gamma;
      int r0, r1;
      cta_rows(P.steps[i].N, blockIdx.x, P.ctas, r0, r1);
      rr[i] = make_int2(r0, r1);
    }
  }
  __syncthreads();

  if (warp == kCWarps) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int s = 0, slot = 0;
      uint32_t reuse = 0;  // parity of the slot's release to wait for
      for (; s < P.n_steps; ++s) {
        if (s >= P.slots && !wait_or_stop(empty + slot, reuse, stop, P.status)) {
          *stop = 1;
          break;
        }
        const uint32_t row_bytes = static_cast<uint32_t>(tab[s].K) / 4;
        const int r0 = rr[s].x;
        const uint32_t bytes = static_cast<uint32_t>(rr[s].y - r0) * row_bytes;
        if (bytes > 0) {
          mbar_arrive_expect_tx(full + slot, bytes);
          bulk_g2s_hint(slots + static_cast<size_t>(slot) * P.slot_bytes,
                        tab[s].packed + static_cast<size_t>(r0) * row_bytes, bytes, full + slot, pol);
        } else {
          mbar_arrive(full + slot);
        }
        if (++slot == P.slots) {
          slot = 0;
          if (s >= P.slots) reuse ^= 1u;
        }
      }
      *issued_sh = s;
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- consumers
    const unsigned tag = ld_relaxed_u32(P.epoch) + 1u;
    // the copy of the exchange this CTA reads
    const unsigned long long *my_stats =
        P.stats + static_cast<size_t>(blockIdx.x % kChainReplicas) * P.n_steps * kMaxCtas * 2;
    const unsigned long long *my_xch =
        P.xch + static_cast<size_t>(blockIdx.x % kChainReplicas) * P.xch_words;
    int consumed = 0, slot = 0;
    uint32_t phase = 0;  // parity of the slot's fill to wait for
    for (int s = 0; s < P.n_steps; ++s) {
      const StepP &d = tab[s];
      const int nw = d.K >> 1;  // input words: two bf16 values each
      const bool norm = (d.flags & kStepNormIn) != 0;
      uint32_t w[kMaxWordsPerThread];
#pragma unroll
      for (int i = 0; i < kMaxWordsPerThread; ++i) w[i] = 0u;
      float sc, r, inv = 1.0f;
      if (s == 0) {
        // ---- the chain input: reduce max |x| (and sum x^2) over the CTA
        const uint32_t *src = reinterpret_cast<const uint32_t *>(P.x0);
        float a = 0.0f, ss = 0.0f;
#pragma unroll
        for (int i = 0; i < kMaxWordsPerThread; ++i) {
          if (tid + i * kCThreads >= nw) break;
          w[i] = src[tid + i * kCThreads];
          const float x0 = bf16_lo(w[i]), x1 = bf16_hi(w[i]);
          a = fmaxf(a, fmaxf(fabsf(x0), fabsf(x1)));
          ss = __fmaf_rn(x1, x1, __fmaf_rn(x0, x0, ss));
        }
        a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        if (lane == 0) {
          red_a[warp] = a;
          red_s[warp] = ss;
        }
        if (tid == 0) *stop_snap = *stop;
        consumers_sync();
        if (*stop_snap) break;
        a = red_a[0];
        ss = red_s[0];
#pragma unroll
        for (int i = 1; i < kCWarps; ++i) {
          a = fmaxf(a, red_a[i]);
          ss = __fadd_rn(ss, red_s[i]);
        }
        if (norm) {
          inv = rms_inv(ss, d.K);
          a = round_bf16(__fmul_rn(a, inv));
        }
        sc = act_scale(a);
        r = __fdiv_rn(gam[s], sc);
      } else {
        // ---- warp 0 waits for every CTA's record of the previous step and
        // computes the scale once; then every thread loads its words
        if (warp == 0 && !*stop) {
          float a, ss;
          if (poll_stats(my_stats + static_cast<size_t>(s - 1) * kMaxCtas * 2, P.ctas, tag, lane,
                         a, ss, P.status)) {
            if (lane == 0) {
              float iv = 1.0f;
              if (norm) {
                iv = rms_inv(ss, d.K);
                a = round_bf16(__fmul_rn(a, iv));
              }
              const float scl = act_scale(a);
              par[0] = scl;
              par[1] = __fdiv_rn(gam[s], scl);
              par[2] = iv;
            }
          } else {
            *stop = 1;
          }
        }
        if (tid == 0) *stop_snap = *stop;
        consumers_sync();
        if (*stop_snap) break;
        sc = par[0];
        r = par[1];
        inv = par[2];
        if (!poll_words(my_xch + tab[s - 1].out_off, nw, tid, tag, w, P.status)) {
          *stop = 1;  // acted on at the next step's first barrier
#pragma unroll
          for (int i = 0; i < kMaxWordsPerThread; ++i) w[i] = 0u;
        }
      }
      // ---- (normalise and) quantise: each int8 at its place in the unpack order
#pragma unroll
      for (int i = 0; i < kMaxWordsPerThread; ++i) {
        const int idx = tid + i * kCThreads;
        if (idx >= nw) break;
        if (norm) {
          w[i] = bf16_bits(__fmul_rn(bf16_lo(w[i]), inv)) |
                 (bf16_bits(__fmul_rn(bf16_hi(w[i]), inv)) << 16);
          if (d.Xn != nullptr && blockIdx.x == 0) reinterpret_cast<uint32_t *>(d.Xn)[idx] = w[i];
        }
        const int e = 2 * idx, g = e >> 4, j = e & 15;
        xq[16 * g + unpack_pos(j)] = static_cast<uint8_t>(quant_i8(bf16_lo(w[i]), sc));
        xq[16 * g + unpack_pos(j + 1)] = static_cast<uint8_t>(quant_i8(bf16_hi(w[i]), sc));
      }
      consumers_sync();
      // ---- this CTA's rows: warp w takes rows w, w + 16, ... of its range
      // every lane waits (bounded); the warp goes on only if all of them saw the copy land
      const bool have_w = __all_sync(0xffffffffu, mbar_wait(full + slot, phase, P.status));
      const int r0 = rr[s].x, rows = rr[s].y - r0;
      if (have_w) {
        consumed = s + 1;
        const int words = d.K >> 4;  // packed 32-bit words per row
        const uint32_t *wsl =
            reinterpret_cast<const uint32_t *>(slots + static_cast<size_t>(slot) * P.slot_bytes);
        const bool relu2 = (d.flags & kStepRelu2) != 0;
        for (int rl = warp; rl < rows; rl += kCWarps) {
          const int acc = row_dot(wsl + static_cast<size_t>(rl) * words, xq4, words, lane);
          if (lane == 0) ystage[rl] = static_cast<uint16_t>(bf16_bits(epilogue_value(acc, r, relu2)));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + slot);
      } else {
        *stop = 1;  // acted on at the next step's first barrier
      }
      consumers_sync();
      // ---- warp 0 publishes the CTA's outputs (two per tagged word), then
      // its record: max |y| and sum y^2 over the outputs the next step reads
      if (warp == 0 && !*stop) {
        const int k_next = s + 1 < P.n_steps ? tab[s + 1].K : (P.y_norm != nullptr ? P.y_norm_n : 0);
        float la = 0.0f, ls = 0.0f;
        for (int pl = lane; 2 * pl < rows; pl += 32) {
          const uint32_t ya = ystage[2 * pl];
          const bool has_b = 2 * pl + 1 < rows;
          const uint32_t yb = has_b ? ystage[2 * pl + 1] : 0u;
          const unsigned long long word = (static_cast<unsigned long long>(tag) << 32) | (yb << 16) | ya;
#pragma unroll
          for (int c = 0; c < kChainReplicas; ++c)
            st_relaxed_u64(P.xch + static_cast<size_t>(c) * P.xch_words + d.out_off + (r0 >> 1) + pl, word);
          if (has_b)
            *reinterpret_cast<uint32_t *>(d.Y + r0 + 2 * pl) = (yb << 16) | ya;
          else
            d.Y[r0 + 2 * pl] = static_cast<uint16_t>(ya);
          const int g = r0 + 2 * pl;
          if (g < k_next) {
            const float v = bf16_lo(ya);
            la = fmaxf(la, fabsf(v));
            ls = __fmaf_rn(v, v, ls);
          }
          if (has_b && g + 1 < k_next) {
            const float v = bf16_lo(yb);
            la = fmaxf(la, fabsf(v));
            ls = __fmaf_rn(v, v, ls);
          }
        }
        la = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(la)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ls = __fadd_rn(ls, __shfl_xor_sync(0xffffffffu, ls, o));
        ls = __shfl_sync(0xffffffffu, ls, 0);  // one value for every copy
        if (lane < kChainReplicas) {  // lane c writes copy c
          unsigned long long *rec =
              P.stats + (static_cast<size_t>(lane) * P.n_steps * kMaxCtas + static_cast<size_t>(s) * kMaxCtas +
                         blockIdx.x) * 2;
          st_relaxed_u64(rec, (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(la));
          st_relaxed_u64(rec + 1, (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(ls));
        }
      }
      if (++slot == P.slots) {
        slot = 0;
        phase ^= 1u;
      }
    }
    if (tid == 0) {
      *consumed_sh = consumed;
      *stop_snap = *stop;
    }

    // ---- end of the chain: count this CTA out; CTA 0 normalises the last
    // output (optional) and then advances the launch counter.
    consumers_sync();
    if (tid == 0) {
      __threadfence();
      atomicAdd(P.done, 1u);
    }
    if (blockIdx.x == 0 && !*stop_snap) {
      if (P.y_norm != nullptr) {
        if (warp == 0) {
          float a, ss;
          if (poll_stats(my_stats + static_cast<size_t>(P.n_steps - 1) * kMaxCtas * 2, P.ctas, tag,
                         lane, a, ss, P.status)) {
            if (lane == 0) par[2] = rms_inv(ss, P.y_norm_n);
          } else {
            *stop = 1;
          }
        }
        consumers_sync();
        const int nw = P.y_norm_n >> 1;
        uint32_t w[kMaxWordsPerThread];
        if (!*stop && poll_words(my_xch + tab[P.n_steps - 1].out_off, nw, tid, tag, w, P.status)) {
          const float iv = par[2];
#pragma unroll
          for (int i = 0; i < kMaxWordsPerThread; ++i) {
            const int idx = tid + i * kCThreads;
            if (idx >= nw) break;
            reinterpret_cast<uint32_t *>(P.y_norm)[idx] =
                bf16_bits(__fmul_rn(bf16_lo(w[i]), iv)) | (bf16_bits(__fmul_rn(bf16_hi(w[i]), iv)) << 16);
          }
        }
      }
      if (tid == 0) {
        const unsigned want = tag * static_cast<unsigned>(P.ctas);
        const long long t0 = clock64();
        bool ok = true;
        while (ld_relaxed_u32(P.done) != want) {
          if (clock64() - t0 > kWaitLimitCycles) {
            record_status(P.status, kStatusTimeout);
            ok = false;
            break;
          }
        }
        if (ok) {
          __threadfence();
          atomicExch(P.epoch, tag);
        }
      }
    }
  }

  // ---- leave only once every bulk copy this CTA issued has landed
  __syncthreads();
  if (tid == 0) {
    for (int s = *consumed_sh; s < *issued_sh; ++s)
      mbar_wait(full + s % P.slots, (s / P.slots) & 1, P.status);
  }
}

}  // namespace

// Host side -----------------------------------------------------------------

bool chain_plan(const ChainStep *steps, int n_steps, int num_sms, ChainPlan *plan) {
  const int ctas = num_sms < kMaxCtas ? num_sms : kMaxCtas;
  int64_t slot_bytes = 0, max_rows = 0;
  int max_k = 0;
  for (int s = 0; s < n_steps; ++s) {
    const int64_t pairs = (steps[s].N + 1) / 2;
    const int64_t rows = 2 * ((pairs + ctas - 1) / ctas);
    const int64_t b = rows * (steps[s].K / 4);
    if (b > slot_bytes) slot_bytes = b;
    if (rows > max_rows) max_rows = rows;
    if (steps[s].K > max_k) max_k = static_cast<int>(steps[s].K);
  }
  slot_bytes = (slot_bytes + 127) / 128 * 128;
  const int64_t ystage_bytes = (2 * max_rows + 127) / 128 * 128;
  const int xq_bytes = (max_k + 127) / 128 * 128;
  const int64_t room = kSmemLimit - kHeader - table_bytes(n_steps) - ystage_bytes - xq_bytes;
  int64_t slots = slot_bytes > 0 ? room / slot_bytes : kMaxSlots;
  if (slots > kMaxSlots) slots = kMaxSlots;
  if (slots < 2) return false;
  plan->ctas = ctas;
  plan->slots = static_cast<int>(slots);
  plan->slot_bytes = static_cast<int>(slot_bytes);
  plan->xq_bytes = xq_bytes;
  plan->ystage_bytes = static_cast<int>(ystage_bytes);
  plan->smem = static_cast<size_t>(kHeader) + table_bytes(n_steps) + ystage_bytes + xq_bytes +
               static_cast<size_t>(slots) * slot_bytes;
  return true;
}

int chain_max_k() { return kCThreads * 16; }

cudaError_t launch_chain(const ChainStep *steps, int n_steps, const ChainPlan &plan,
                         const void *x0, void *y_norm, int64_t y_norm_n, void *workspace,
                         const LaunchCtx &ctx) {
  ChainP p;
  p.x0 = static_cast<const uint16_t *>(x0);
  p.y_norm = static_cast<uint16_t *>(y_norm);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  p.epoch = reinterpret_cast<unsigned int *>(ws);
  p.done = reinterpret_cast<unsigned int *>(ws + 128);
  p.stats = reinterpret_cast<unsigned long long *>(ws + kChainWorkspaceHeader);
  p.xch = reinterpret_cast<unsigned long long *>(ws + kChainWorkspaceHeader +
                                                 chain_stats_bytes(n_steps));
  p.status = ctx.status;
  p.n_steps = n_steps;
  p.ctas = plan.ctas;
  p.slots = plan.slots;
  p.slot_bytes = plan.slot_bytes;
  p.xq_bytes = plan.xq_bytes;
  p.ystage_bytes = plan.ystage_bytes;
  p.y_norm_n = static_cast<int>(y_norm_n);
  int64_t off = 0;
  for (int s = 0; s < n_steps; ++s) {
    StepP &d = p.steps[s];
    d.packed = steps[s].packed;
    d.gamma = steps[s].gamma;
    d.Y = static_cast<uint16_t *>(steps[s].Y);
    d.Xn = static_cast<uint16_t *>(steps[s].Xn);
    d.N = static_cast<int>(steps[s].N);
    d.K = static_cast<int>(steps[s].K);
    d.flags = static_cast<int>(steps[s].flags);
    d.out_off = static_cast<int>(off);
    off += chain_xch_words(steps[s].N);
  }
  p.xch_words = static_cast<int>(off);
  cudaError_t e = cudaFuncSetAttribute(chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(plan.smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.ctas));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = ctx.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, chain_kernel, p);
}

}  // namespace bitnet
