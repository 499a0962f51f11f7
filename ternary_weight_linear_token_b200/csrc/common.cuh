// common.cuh -- device helpers shared by the BitLinear kernels (sm_100a).
//
// Thin inline-PTX wrappers: mbarriers, bulk and tensor (TMA) copies,
// programmatic dependent launch, tcgen05 (TMEM allocation, MMA, commit,
// loads), plus the bit-exact arithmetic of the quantisers.  Every wait on
// an mbarrier is bounded: when it gives up it records BITNET_ERR_TIMEOUT in
// the device status word and returns false, so no kernel can spin forever.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnet {

constexpr int kStatusTimeout = 5;  // == BITNET_ERR_TIMEOUT

// ------------------------------------------------------------ status word
__device__ __forceinline__ void record_status(int *status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------ PDL
// Wait until the grids this one depends on (programmatic dependent launch)
// have completed and their memory is visible; a no-op without such a grid.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next grid in the stream to start launching.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ shared memory
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// CLUSTER: acquire at cluster scope, for barriers that threads or tensor
// cores of the other CTA of a pair arrive on.
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  if (CLUSTER)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  return ok != 0;
}

// About two seconds at the B200 boost clock: far beyond any legitimate wait.
constexpr long long kWaitLimitCycles = 4000000000LL;

// Bounded wait for the phase with the given parity to complete.  Returns
// false (after recording a timeout) if it did not complete within the limit.
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status) {
  if (mbar_try_wait<CLUSTER>(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait<CLUSTER>(bar, parity)) return true;
    if (clock64() - t0 > kWaitLimitCycles) {
      record_status(status, kStatusTimeout);
      return false;
    }
  }
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy reads (TMA, tensor core) of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ bulk copies
// Contiguous global -> shared copy completed on an mbarrier (transaction
// bytes).  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tensor (TMA) load of one box into shared memory; c0 is the innermost
// coordinate in elements (bytes here: all our maps are over 8-bit data).
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int32_t c0, int32_t c1,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------ CTA pairs
// A cluster of two CTAs on two SMs sharing tcgen05 work (cta_group::2).
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of every CTA of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// shared::cluster address of this CTA's shared variable at `p` as it sits in
// CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on an mbarrier of any CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// 2-D TMA load into this CTA's shared memory, completion (transaction bytes)
// signalled on an mbarrier of either CTA of the pair.  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const void *tmap, int32_t c0,
                                                 int32_t c1, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(bar_cluster)
      : "memory");
}

// 2-D tensor (TMA) store of one box from shared memory, tracked in this
// thread's bulk async-group.  c0 is the innermost coordinate in elements.
__device__ __forceinline__ void tma_store_2d(const void *tmap, const void *src, int32_t c0,
                                             int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap),
      "r"(c0), "r"(c1), "r"(smem_u32(src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all of this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ------------------------------------------------------------ tcgen05
// PAIR: cta_group::2, issued by one warp in each CTA of the pair, which then
// hold the same columns.
template <bool PAIR = false>
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  if (PAIR)
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
template <bool PAIR = false>
__device__ __forceinline__ void tmem_relinquish() {
  if (PAIR)
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  else
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
template <bool PAIR = false>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  if (PAIR)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32, one CTA.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The pair form (issued by the pair's first CTA): A is 256 rows, 128 in each
// CTA's shared memory, B's N columns half in each, at the same offsets; D's
// rows 0-127 land in this CTA's TMEM, rows 128-255 in the other's.
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (once) on the mbarrier at this offset in both CTAs of the pair when
// the pair MMAs issued so far have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}

// Arrive (once) on an mbarrier when all previously issued MMAs of this
// thread have completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  const uint64_t lo = ((saddr & 0x3FFFFu) >> 4) | (1u << 16);            // start, LBO = 16 B
  const uint64_t hi = (1024u >> 4) | (1u << 14) | (2u << 29);            // SBO, version, SW128
  return lo | (hi << 32);
}

// ------------------------------------------------------------ arithmetic
// Per-token scale s = 127 / amax (IEEE fp32 division); 1 for an all-zero row.
// The weightless RMS normalisation's factor 1 / sqrt(ss / K + 1e-6) for a
// token whose squares sum to ss.  ss is accumulated in fp64, where the square
// of an fp32 (or bf16) value is exact, and the factor is computed in fp64 and
// rounded once to fp32: the operations of the plain definition, so the
// factor differs from it only where the fp64 sums, taken in another order,
// straddle an fp32 rounding boundary of the factor (about one token in 10^7).
__device__ __forceinline__ float rms_factor(double ss, int64_t K) {
  const double q = __dadd_rn(__ddiv_rn(ss, static_cast<double>(K)), 1e-6);
  return __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(q)));
}
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// x^2 added to an fp64 sum (the product is exact in fp64).
__device__ __forceinline__ double add_sq(double ss, float x) {
  const double d = static_cast<double>(x);
  return __fma_rn(d, d, ss);
}

__device__ __forceinline__ float act_scale(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(127.0f, amax);
}
// clamp(round_half_away(x * s), -127, 127), exactly, on the FMA and ALU
// pipes only (no float-to-int conversion): adding 1.5 * 2^23 to a float of
// magnitude below 2^22 leaves its nearest integer (ties to even, the IEEE
// rounding of the add) as the low bits of the sum.  Subtracting it back gives
// that integer as a float; a tie (the remainder is exactly +-0.5) is then
// moved away from zero, and the clamped integer is read from the low bits of
// a second add.  Checked against the plain definition for every float of
// magnitude up to 128; an in-contract x * s never exceeds 127.00003.
__device__ __forceinline__ int quant_i8(float x, float s) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23, bit pattern 0x4B400000
  const float v = __fmul_rn(x, s);
  float r = __fsub_rn(__fadd_rn(v, kMagic), kMagic);
  if (fabsf(__fsub_rn(v, r)) == 0.5f) r = __fadd_rn(v, copysignf(0.5f, v));
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return static_cast<int>(__float_as_uint(__fadd_rn(r, kMagic)) - 0x4B400000u);
}
// quant_i8 for 16 activations of one row, for the throughput-bound
// quantiser.  Within the quantiser's contract (finite x, s = 127 / max|x|
// finite) |x * s| <= 127 * (1 + 2^-24) rounds to at most 127.0000077, so the
// clamp never binds and is left out.  Adding 1.5 * 2^23 rounds v = x * s to
// the nearest integer, ties to even, which the sum's low bits hold; r = that
// sum minus 1.5 * 2^23 is the same integer as a float, and d = v - r is
// exact, |d| <= 1/2.  A tie (|d| = 1/2) that went toward zero -- d has the
// sign of v; with q != 0 that is the sign of q, with q = 0 (v = +-1/2) it
// always is -- moves one step away.  Ties are rare: they are found by the
// chunk's largest |d| and fixed in a branch.  Checked against the plain
// definition for every float |v| <= 127.00002.  The three roundings are the
// explicit _rn intrinsics, which the compiler never contracts: a fused
// x * s + 1.5 * 2^23 would round the exact product instead of v and break
// ties such as v = 63.5 (the paired f32x2 instructions did exactly that).
__device__ __forceinline__ void quant16(const float (&x)[16], float s, int (&q)[16]) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23, bit pattern 0x4B400000
  float d[16];
  float dmax = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float v = __fmul_rn(x[e], s);
    const float t = __fadd_rn(v, kMagic);
    q[e] = static_cast<int>(__float_as_uint(t) - 0x4B400000u);
    d[e] = __fsub_rn(v, __fsub_rn(t, kMagic));
    dmax = fmaxf(dmax, fabsf(d[e]));
  }
  if (dmax == 0.5f) {
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if (fabsf(d[e]) == 0.5f && (q[e] == 0 || (d[e] > 0.0f) == (q[e] > 0)))
        q[e] += d[e] > 0.0f ? 1 : -1;
  }
}

// y = (float)acc * (gamma / s), then optionally ReLU^2.
__device__ __forceinline__ float epilogue_value(int acc, float r, bool relu2) {
  float y = __fmul_rn(__int2float_rn(acc), r);
  if (relu2) {
    y = y > 0.0f ? y : 0.0f;
    y = __fmul_rn(y, y);
  }
  return y;
}

// Four int8 lanes of 2-bit codes -> int8 ternary values {0, +1, -1}, natural
// order: lane i of the result is element 4j + i of the 16-element group held
// by word w (layout: element 16g + 4j + i at bits 8i + 2j).
__device__ __forceinline__ uint32_t unpack_natural(uint32_t w, int j) {
  const uint32_t c = (w >> (2 * j)) & 0x03030303u;        // codes in byte lanes
  const uint32_t h = (w >> (2 * j + 1)) & 0x01010101u;    // 1 where the code is 2
  return c + h * 0xFDu;                                   // 2 -> 0xFF (-1), no carries
}

// Four int8 values into one 32-bit word, first value in the lowest byte.
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(b), 0x0040u);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(c), static_cast<uint32_t>(d), 0x0040u);
  return __byte_perm(lo, hi, 0x5410u);
}

// 16 int8 activations of one 16-element group, stored in the order in which
// the byte-permute unpack produces the weights of the matching packed word:
// elements {0,8,1,9}, {4,12,5,13}, {2,10,3,11}, {6,14,7,15}.
__device__ __forceinline__ uint4 pack_permuted(const int (&q)[16]) {
  uint4 o;
  o.x = pack4(q[0], q[8], q[1], q[9]);
  o.y = pack4(q[4], q[12], q[5], q[13]);
  o.z = pack4(q[2], q[10], q[3], q[11]);
  o.w = pack4(q[6], q[14], q[7], q[15]);
  return o;
}

// 16 int8 weights {0, +1, -1} of one packed word.  PERM: in the K order of
// pack_permuted, by four byte-permute lookups in a 4-entry table held in a
// register (code 0 -> 0x00, 1 -> 0x01, 2 and 3 -> 0xFF), 3 instructions per 4
// weights; else natural order (shift/mask/multiply).
template <bool PERM>
__device__ __forceinline__ uint4 expand_word(uint32_t w) {
  constexpr uint32_t kLut = 0xFFFF0100u;
  if (PERM)
    return make_uint4(__byte_perm(kLut, 0u, w & 0x3333u), __byte_perm(kLut, 0u, (w >> 2) & 0x3333u),
                      __byte_perm(kLut, 0u, (w >> 16) & 0x3333u),
                      __byte_perm(kLut, 0u, (w >> 18) & 0x3333u));
  return make_uint4(unpack_natural(w, 0), unpack_natural(w, 1), unpack_natural(w, 2),
                    unpack_natural(w, 3));
}


// ------------------------------------------------------------ decode dot products
// The unpack order of one 16-element group of int8 activations in shared
// memory (16 bytes): the elements that the byte-permute unpack below pairs
// with selector shifts 0, 16, 2, 18 -- {0,8,1,9}, {2,10,3,11}, {4,12,5,13},
// {6,14,7,15} -- so elements 0..7 of the group fill bytes 0..7 with the help
// of 4 bytes from elements 8..11, and vice versa.
constexpr uint32_t kTernaryLut = 0xFFFF0100u;  // code 0 -> 0, 1 -> +1, 2 -> -1, 3 -> -1

// clamp(round_half_away(x * s), -127, 127) of 8 values, packed as 8 int8
// in their order (two words, first value in the lowest byte), on the FMA and
// ALU pipes: the nearest integer (ties to even, the IEEE rounding of the add)
// is the low byte of x * s + 1.5 * 2^23; a remainder of exactly one half (a
// tie, found as the chunk's largest |v - r|, which is at most 1/2) is moved
// away from zero in a rarely taken branch.  The same arithmetic as quant16:
// within the contract (finite x, s = 127 / max |x|) |x * s| rounds to at
// most 127, so the clamp never binds and is left out.
__device__ __forceinline__ uint2 quant8_packed(const float (&x)[8], float s) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23, bit pattern 0x4B400000
  uint32_t t[8];
  float d[8];
  float dmax = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float v = __fmul_rn(x[e], s);
    const float tf = __fadd_rn(v, kMagic);
    t[e] = __float_as_uint(tf);
    d[e] = __fsub_rn(v, __fsub_rn(tf, kMagic));
    dmax = fmaxf(dmax, fabsf(d[e]));
  }
  if (dmax == 0.5f) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int q = static_cast<int>(t[e] - 0x4B400000u);
      if (fabsf(d[e]) == 0.5f && (q == 0 || (d[e] > 0.0f) == (q > 0))) t[e] += d[e] > 0.0f ? 1u : ~0u;
    }
  }
  return make_uint2(__byte_perm(__byte_perm(t[0], t[1], 0x0040u), __byte_perm(t[2], t[3], 0x0040u), 0x5410u),
                    __byte_perm(__byte_perm(t[4], t[5], 0x0040u), __byte_perm(t[6], t[7], 0x0040u), 0x5410u));
}

// Quantise one 8-element half-group and store it, with the partner lane's
// help, in the unpack order.  Both lanes of a pair must call this together
// (the shuffle needs the whole warp); `active` is false past the end of K.
__device__ __forceinline__ void store_half_group(uint8_t *xrow, int chunk, const float (&v)[8],
                                                 float sm, bool active) {
  const uint2 ab = active ? quant8_packed(v, sm) : make_uint2(0u, 0u);
  const bool lo = (chunk & 1) == 0;  // elements 0..7 of the group (else 8..15)
  const uint32_t a = ab.x, b = ab.y;
  // low half sends elements 4..7, high half sends elements 8..11
  const uint32_t other = __shfl_xor_sync(0xffffffffu, lo ? b : a, 1);
  if (!active) return;
  uint2 o;
  if (lo) {  // bytes 0..7: {0,8,1,9}, {2,10,3,11}
    o.x = __byte_perm(a, other, 0x5140);
    o.y = __byte_perm(a, other, 0x7362);
  } else {   // bytes 8..15: {4,12,5,13}, {6,14,7,15}
    o.x = __byte_perm(other, b, 0x5140);
    o.y = __byte_perm(other, b, 0x7362);
  }
  *reinterpret_cast<uint2 *>(xrow + 8 * chunk) = o;
}

// The 16 int8 weights of a packed word, as four dp4a operands in the
// shared-memory K order (selector shifts 0, 16, 2, 18).
struct Unpacked {
  int a, b, c, d;
};
// The byte permute reads only the low 16 bits of its selector, so one mask
// of the whole word serves two selectors (shift 0 and 16; shift 2 and 18).
__device__ __forceinline__ Unpacked unpack_word(uint32_t w) {
  const uint32_t m0 = w & 0x33333333u, m1 = (w >> 2) & 0x33333333u;
  return {static_cast<int>(__byte_perm(kTernaryLut, 0u, m0)),
          static_cast<int>(__byte_perm(kTernaryLut, 0u, m0 >> 16)),
          static_cast<int>(__byte_perm(kTernaryLut, 0u, m1)),
          static_cast<int>(__byte_perm(kTernaryLut, 0u, m1 >> 16))};
}
__device__ __forceinline__ int dot_word(const Unpacked &q, uint4 x, int acc) {
  acc = __dp4a(q.a, static_cast<int>(x.x), acc);
  acc = __dp4a(q.b, static_cast<int>(x.y), acc);
  acc = __dp4a(q.c, static_cast<int>(x.z), acc);
  acc = __dp4a(q.d, static_cast<int>(x.w), acc);
  return acc;
}

}  // namespace bitnet
