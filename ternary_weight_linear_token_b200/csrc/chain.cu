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
//   * A link's outputs go straight to that step's output buffer, each warp
//     storing its finished rows at once.  The values the next step reads are
//     also stored as tagged 32-bit words in the workspace: the bf16 value in
//     the low half, a 16-bit tag of this launch in the high half, one
//     single-copy-atomic store per value.  A word is valid once its tag is
//     this launch's, so the data carries its own readiness: no arrival
//     counter, no fence, no flag to order the data before.
//   * When all its warps have stored their rows (a CTA barrier, so that no
//     warp polls while others of the SM still compute), the CTA hands the
//     weight slot back and starts the next step: every thread loads its part
//     of the tagged input (relaxed loads through L2) and loads again the
//     words whose tag is not yet this launch's, bounded.  Each CTA reduces
//     the max |x| of the whole input itself, and where a layer starts (the
//     weightless RMS normalisation) the fp64 sum of squares, all in the same
//     fixed order in every CTA, so all CTAs quantise identically.
//   * Per link, each CTA quantises the whole input to int8 exactly as
//     bitnet_quantize_act does and computes its balanced range of output
//     features with the byte-permute unpack and dp4a, in the same int32
//     arithmetic and with the same epilogue as bitnet_w158a8_matmul.  Warp
//     w takes rows w, w + 16, ... of the CTA's range, up to 4 at a time: a
//     lane loads each of its activation chunks once per pass and uses it for
//     all of the pass's rows, and stores each row as soon as it is done.
//   * Launch T (T = the launch counter kept in the workspace, plus one) tags
//     its words with (T mod 65535) + 1, never 0 (a zero-filled workspace
//     holds no valid word) and different from the previous launch's tag.
//     After the last step every CTA adds one to a done counter that only
//     grows (release, after a CTA barrier); CTA 0 waits for T * ctas
//     (acquire), normalises the last output (optional) and advances the
//     launch counter, so graph replays and repeated calls need no host
//     action.
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
constexpr int kMaxCtas = kChainMaxCtas;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kHeader = 1024;
constexpr int kBarConsumers = 1;            // named barrier of the consumer warps
constexpr int kChunks = 2;                  // 8-element input chunks per thread: K <= 8192
constexpr int kRowsPerPass = 4;             // rows a warp carries at once in the dot products
constexpr long long kFirstPollDelayCycles = 885;  // before a step's first input loads (450 ns)

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
  int toff;          // first tagged word of this step's output (the part the next step reads)
};

struct ChainP {
  const uint16_t *x0;
  uint16_t *y_norm;
  unsigned *epoch;
  unsigned *done;             // CTAs past the last step, summed over launches
  uint32_t *tagged;           // tag << 16 | bf16 bits, per step from toff
  int *status;
  int n_steps, ctas, slots, slot_bytes, xq_bytes, y_norm_n;
  StepP steps[kChainMaxSteps];
};

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Four tagged words written by other SMs in this launch (each word is read
// single-copy atomic, the four need not be from the same moment).
__device__ __forceinline__ uint4 ld_relaxed_u4(const uint32_t *p) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t *p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// 16 bytes from global memory through L2 only (another SM wrote them in this
// launch; nothing of them may come from this SM's L1).
__device__ __forceinline__ uint4 ld_cg_u4(const void *p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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

// Rows [r0, r1) of an N-row projection owned by CTA c: whole pairs of rows,
// balanced over the CTAs.
__host__ __device__ inline void cta_rows(int N, int c, int ctas, int &r0, int &r1) {
  const long long pairs = (N + 1) / 2;
  r0 = static_cast<int>(2 * (pairs * c / ctas));
  const int e = static_cast<int>(2 * (pairs * (c + 1) / ctas));
  r1 = e < N ? e : N;
}

__device__ __forceinline__ uint32_t bf16_bits(float y) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(y)));
}
__device__ __forceinline__ float round_bf16(float y) { return __uint_as_float(bf16_bits(y) << 16); }

// The 8 bf16 values of a 16-byte chunk as fp32.
__device__ __forceinline__ void chunk_to_float(uint4 u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    v[2 * h] = __uint_as_float(w[h] << 16);
    v[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
  }
}
// True when all four words carry the tag `tb` (already shifted to the high half).
__device__ __forceinline__ bool tagged_ok(uint4 u, uint32_t tb) {
  return (((u.x ^ tb) | (u.y ^ tb) | (u.z ^ tb) | (u.w ^ tb)) >> 16) == 0u;
}

// Bounded wait (one thread) until a counter reaches `target`, polling with
// acquire loads: what every CTA stored before its release add is then
// visible to this thread (and, after a CTA barrier, to the whole CTA).
__device__ __forceinline__ bool wait_count(const unsigned *ctr, unsigned target, int *status) {
  const long long t0 = clock64();
  while (true) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v == target) return true;
    if (clock64() - t0 > kWaitLimitCycles) {
      record_status(status, kStatusTimeout);
      return false;
    }
  }
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

// This thread's part of a step's input from the tagged words `src` (8 values
// per chunk, chunks tid, tid + 512, ...): load every word once, then re-load
// the 4-word groups whose tag is not yet `tb` until all of them carry it.
// Bounded: false (and BITNET_ERR_TIMEOUT recorded) if they never do.
__device__ __forceinline__ bool load_tagged(const uint32_t *src, int nchunks, int tid, uint32_t tb,
                                            float (&v)[kChunks][8], int *status) {
  uint4 t[kChunks][2];
  // The first loads wait about 0.45 us: polling the moment the CTA is done,
  // while the last CTAs still store, slowed every step (30-layer stack: 575
  // us per token without the delay; __nanosleep of 50 / 150 / 300 / 600 /
  // 1000 ns: 548 / 480 / 447 / 462 / 458; sleeping only after a first poll
  // that found missing words: 705).  A spin on the SM clock is exact where
  // the sleep is not: 200 / 300 / 450 / 600 / 800 ns at 1965 MHz gave
  // 472 / 450 / 430 / 434 / 456 us per token.
  {
    const long long t_start = clock64();
    while (clock64() - t_start < kFirstPollDelayCycles) {
    }
  }
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = tid + i * kCThreads;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      t[i][h] = c < nchunks ? ld_relaxed_u4(src + 8 * c + 4 * h) : make_uint4(tb, tb, tb, tb);
  }
  const long long t0 = clock64();
  bool ok = true;
  while (true) {
    bool all = true;
#pragma unroll
    for (int i = 0; i < kChunks; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) all = all && tagged_ok(t[i][h], tb);
    if (all) break;
    if (clock64() - t0 > kWaitLimitCycles) {
      record_status(status, kStatusTimeout);
      ok = false;
      break;
    }
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = tid + i * kCThreads;
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (!tagged_ok(t[i][h], tb)) t[i][h] = ld_relaxed_u4(src + 8 * c + 4 * h);
    }
  }
#pragma unroll
  for (int i = 0; i < kChunks; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w[4] = {t[i][h].x, t[i][h].y, t[i][h].z, t[i][h].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) v[i][4 * h + e] = __uint_as_float(w[e] << 16);
    }
  return ok;
}

// NR rows of a pass (rows w, w + 16, ... from `wr`, each `words` packed
// words long) against the quantised input: lane l takes words l, l + 32, ...
// Two accumulators per row halve the chain of dependent dp4a (integer sums:
// the order does not change the result; 444 -> 436 us per token).
template <int NR>
__device__ __forceinline__ void dot_rows(const uint32_t *wr, int words, const uint4 *xq4, int lane,
                                         int (&acc)[kRowsPerPass]) {
  const size_t stride = static_cast<size_t>(kCWarps) * words;
  int acc2[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) acc2[i] = 0;
  for (int w = lane; w < words; w += 32) {
    const uint4 x = xq4[w];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const Unpacked q = unpack_word(wr[i * stride + w]);
      acc[i] = __dp4a(q.a, static_cast<int>(x.x), acc[i]);
      acc2[i] = __dp4a(q.b, static_cast<int>(x.y), acc2[i]);
      acc[i] = __dp4a(q.c, static_cast<int>(x.z), acc[i]);
      acc2[i] = __dp4a(q.d, static_cast<int>(x.w), acc2[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < NR; ++i) acc[i] += acc2[i];
}

__global__ void __launch_bounds__(kThreads, 1) chain_kernel(const __grid_constant__ ChainP P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);                // [kMaxSlots]
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + 64);          // [kMaxSlots]
  float *red_a = reinterpret_cast<float *>(smem + 128);               // [kCWarps]
  double *red_s = reinterpret_cast<double *>(smem + 192);             // [kCWarps]
  // set by the producer when it gives up, and by consumers when they halt
  volatile int *stop = reinterpret_cast<volatile int *>(smem + 320);
  int *issued_sh = reinterpret_cast<int *>(smem + 324);
  int *consumed_sh = reinterpret_cast<int *>(smem + 328);
  // Set by consumer threads only, each before the consumer barrier after
  // which all of them read it, and not again before all have: every
  // consumer leaves the loop at the same step.  halt_in: an input poll gave
  // up (read after the reduction barrier); halt_w: a weight slot never
  // landed (read after the step's last barrier).
  volatile int *halt_in = reinterpret_cast<volatile int *>(smem + 332);
  volatile int *halt_w = reinterpret_cast<volatile int *>(smem + 336);
  volatile int *fin = reinterpret_cast<volatile int *>(smem + 340);  // CTA 0: every CTA done
  StepP *tab = reinterpret_cast<StepP *>(smem + kHeader);            // [n_steps]
  float *gam = reinterpret_cast<float *>(smem + kHeader + align128(P.n_steps * 48));
  int2 *rr = reinterpret_cast<int2 *>(smem + kHeader + align128(P.n_steps * 48) +
                                      align128(P.n_steps * 4));       // this CTA's rows
  uint8_t *xq = smem + kHeader + table_bytes(P.n_steps);                  // [xq_bytes]
  uint8_t *slots = xq + P.xq_bytes;                                   // [slots][slot_bytes]
  const uint4 *xq4 = reinterpret_cast<const uint4 *>(xq);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < P.slots; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    *stop = 0;
    *halt_in = 0;
    *halt_w = 0;
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
    const uint32_t tb = (tag % 0xFFFFu + 1u) << 16;
    int consumed = 0, slot = 0;
    uint32_t phase = 0;  // parity of the slot's fill to wait for
    for (int s = 0; s < P.n_steps; ++s) {
      const StepP &d = tab[s];
      const int nchunks = d.K >> 3;  // 8 bf16 values per chunk
      const bool norm = (d.flags & kStepNormIn) != 0;
      // ---- the input: x0, or the previous step's tagged output
      float v[kChunks][8];
      if (s == 0) {
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
          const int c = tid + i * kCThreads;
          chunk_to_float(c < nchunks ? *reinterpret_cast<const uint4 *>(P.x0 + 8 * c)
                                     : make_uint4(0u, 0u, 0u, 0u),
                         v[i]);
        }
      } else {
        if (*halt_w) break;
        if (!load_tagged(P.tagged + tab[s - 1].toff, nchunks, tid, tb, v, P.status)) *halt_in = 1;
      }
      float la = 0.0f;
      double ss = 0.0;
#pragma unroll
      for (int i = 0; i < kChunks; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          la = fmaxf(la, fabsf(v[i][e]));
          if (norm) ss = add_sq(ss, v[i][e]);  // fp64, the same order in every CTA
        }
      la = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(la)));
      if (norm) ss = warp_sum_f64(ss);
      if (lane == 0) {
        red_a[warp] = la;
        red_s[warp] = ss;
      }
      consumers_sync();
      if (*halt_in) break;
      float a = __uint_as_float(
          __reduce_max_sync(0xffffffffu, __float_as_uint(lane < kCWarps ? red_a[lane] : 0.0f)));
      float inv = 1.0f;
      if (norm) {
        inv = rms_factor(warp_sum_f64(lane < kCWarps ? red_s[lane] : 0.0), d.K);
        // rounding x * inv to bf16 is monotone in |x|: the max of the
        // normalised values is the normalised max
        a = round_bf16(__fmul_rn(a, inv));
      }
      const float sc = act_scale(a);
      const float r = __fdiv_rn(gam[s], sc);
      // ---- (normalise and) quantise: each int8 at its place in the unpack order
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int c0 = i * kCThreads;
        if (c0 >= nchunks) break;  // uniform over the CTA
        const int c = c0 + tid;
        if (norm) {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[i][e] = round_bf16(__fmul_rn(v[i][e], inv));
          if (d.Xn != nullptr && blockIdx.x == 0 && c < nchunks) {
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h)
              o[h] = (__float_as_uint(v[i][2 * h]) >> 16) | (__float_as_uint(v[i][2 * h + 1]) & 0xFFFF0000u);
            *reinterpret_cast<uint4 *>(d.Xn + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        store_half_group(xq, c, v[i], sc, c < nchunks);
      }
      consumers_sync();
      // ---- this CTA's rows: warp w takes rows w, w + 16, ... of its range
      // every lane waits (bounded); the warp goes on only if all of them saw the copy land
      const bool have_w = __all_sync(0xffffffffu, mbar_wait(full + slot, phase, P.status));
      const int r0 = rr[s].x, rows = rr[s].y - r0;
      const int words = d.K >> 4;  // packed 32-bit words per row
      const bool last = s + 1 == P.n_steps;
      const int k_next = last ? 0 : tab[s + 1].K;
      uint32_t *tout = P.tagged + d.toff;
      const bool relu2 = (d.flags & kStepRelu2) != 0;
      if (have_w) {
        consumed = s + 1;
        const uint32_t *wsl =
            reinterpret_cast<const uint32_t *>(slots + static_cast<size_t>(slot) * P.slot_bytes);
        for (int rb = warp; rb < rows; rb += kCWarps * kRowsPerPass) {
          int acc[kRowsPerPass] = {0, 0, 0, 0};
          const uint32_t *wr = wsl + static_cast<size_t>(rb) * words;
          const int nr = (rows - rb + kCWarps - 1) / kCWarps;  // rows in this pass (warp-uniform)
          if (nr >= kRowsPerPass) dot_rows<kRowsPerPass>(wr, words, xq4, lane, acc);
          else if (nr == 3) dot_rows<3>(wr, words, xq4, lane, acc);
          else if (nr == 2) dot_rows<2>(wr, words, xq4, lane, acc);
          else dot_rows<1>(wr, words, xq4, lane, acc);
#pragma unroll
          for (int i = 0; i < kRowsPerPass; ++i) {
            const int rl = rb + i * kCWarps;
            if (rl < rows) {  // the same for the whole warp
              const int v = __reduce_add_sync(0xffffffffu, acc[i]);
              if (lane == i) {  // the row is complete: lane i stores it now
                const int row = r0 + rl;
                const uint32_t y = bf16_bits(epilogue_value(v, r, relu2));
                d.Y[row] = static_cast<uint16_t>(y);
                if (row < k_next) st_relaxed_u32(tout + row, tb | y);
              }
            }
          }
        }
      } else {
        *halt_w = 1;  // acted on when the step ends
      }
      if (!last) {
        // every warp is past its reads of the slot and has stored its rows;
        // no warp polls the next input while others still compute
        consumers_sync();
        if (tid == 0 && !*halt_w) mbar_arrive(empty + slot);
      }
      if (++slot == P.slots) {
        slot = 0;
        phase ^= 1u;
      }
    }
    // ---- end of the chain: every CTA counts itself in for the last step
    // once all its warps have stored their rows (release, after a CTA
    // barrier); CTA 0 waits for all of them (acquire), normalises the last
    // output (optional) and then advances the launch counter.
    consumers_sync();
    const bool halted = *halt_in != 0 || *halt_w != 0;
    if (tid == 0) {
      *consumed_sh = consumed;
      if (halted) *stop = 1;  // the producer stops waiting for slots
      else red_release_add(P.done, 1u);
    }
    if (blockIdx.x == 0 && !halted) {
      if (tid == 0) *fin = wait_count(P.done, tag * static_cast<unsigned>(P.ctas), P.status);
      consumers_sync();
      if (*fin) {
        if (P.y_norm != nullptr) {
          const uint16_t *src = tab[P.n_steps - 1].Y;
          const int nchunks = P.y_norm_n >> 3;
          uint4 raw[kChunks];
          double ss = 0.0;
#pragma unroll
          for (int i = 0; i < kChunks; ++i) {
            const int c = tid + i * kCThreads;
            raw[i] = c < nchunks ? ld_cg_u4(src + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
            float f[8];
            chunk_to_float(raw[i], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = add_sq(ss, f[e]);
          }
          ss = warp_sum_f64(ss);
          if (lane == 0) red_s[warp] = ss;
          consumers_sync();
          const float iv = rms_factor(warp_sum_f64(lane < kCWarps ? red_s[lane] : 0.0), P.y_norm_n);
#pragma unroll
          for (int i = 0; i < kChunks; ++i) {
            const int c = tid + i * kCThreads;
            if (c >= nchunks) break;
            float f[8];
            chunk_to_float(raw[i], f);
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h)
              o[h] = bf16_bits(__fmul_rn(f[2 * h], iv)) | (bf16_bits(__fmul_rn(f[2 * h + 1], iv)) << 16);
            *reinterpret_cast<uint4 *>(P.y_norm + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        if (tid == 0) atomicExch(P.epoch, tag);
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
  int64_t slot_bytes = 0;
  int max_k = 0;
  for (int s = 0; s < n_steps; ++s) {
    const int64_t pairs = (steps[s].N + 1) / 2;
    const int64_t rows = 2 * ((pairs + ctas - 1) / ctas);
    const int64_t b = rows * (steps[s].K / 4);
    if (b > slot_bytes) slot_bytes = b;
    if (steps[s].K > max_k) max_k = static_cast<int>(steps[s].K);
  }
  slot_bytes = (slot_bytes + 127) / 128 * 128;
  const int xq_bytes = (max_k + 127) / 128 * 128;
  const int64_t room = kSmemLimit - kHeader - table_bytes(n_steps) - xq_bytes;
  int64_t slots = slot_bytes > 0 ? room / slot_bytes : kMaxSlots;
  if (slots > kMaxSlots) slots = kMaxSlots;
  if (slots < 2) return false;
  plan->ctas = ctas;
  plan->slots = static_cast<int>(slots);
  plan->slot_bytes = static_cast<int>(slot_bytes);
  plan->xq_bytes = xq_bytes;
  plan->smem = static_cast<size_t>(kHeader) + table_bytes(n_steps) + xq_bytes +
               static_cast<size_t>(slots) * slot_bytes;
  return true;
}

int chain_max_k() { return kCThreads * 8 * kChunks; }

cudaError_t launch_chain(const ChainStep *steps, int n_steps, const ChainPlan &plan,
                         const void *x0, void *y_norm, int64_t y_norm_n, void *workspace,
                         const LaunchCtx &ctx) {
  ChainP p;
  p.x0 = static_cast<const uint16_t *>(x0);
  p.y_norm = static_cast<uint16_t *>(y_norm);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  p.epoch = reinterpret_cast<unsigned *>(ws);
  p.done = reinterpret_cast<unsigned *>(ws + kChainDoneOffset);
  p.tagged = reinterpret_cast<uint32_t *>(ws + kChainWorkspaceHeader);
  p.status = ctx.status;
  p.n_steps = n_steps;
  p.ctas = plan.ctas;
  p.slots = plan.slots;
  p.slot_bytes = plan.slot_bytes;
  p.xq_bytes = plan.xq_bytes;
  p.y_norm_n = static_cast<int>(y_norm_n);
  int64_t toff = 0;
  for (int s = 0; s < n_steps; ++s) {
    StepP &d = p.steps[s];
    d.packed = steps[s].packed;
    d.gamma = steps[s].gamma;
    d.Y = static_cast<uint16_t *>(steps[s].Y);
    d.Xn = static_cast<uint16_t *>(steps[s].Xn);
    d.N = static_cast<int>(steps[s].N);
    d.K = static_cast<int>(steps[s].K);
    d.flags = static_cast<int>(steps[s].flags);
    d.toff = static_cast<int>(toff);
    if (s + 1 < n_steps) toff += chain_tag_words(steps[s + 1].K);
  }
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
