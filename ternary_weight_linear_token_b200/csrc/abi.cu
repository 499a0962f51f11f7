// abi.cu -- the C ABI (include/bitnet158.h): argument checks on the host,
// choice of kernel path, launches on the caller's stream.
//
// Every check runs before any CUDA call, so a rejected call has no side
// effect and needs no GPU.  Paths of bitnet_w158a8_matmul:
//   rows     M <= 3 (M <= 8 when K % 64 != 0): one fused low-latency kernel
//            (warp per output feature, dp4a; activation quantisation inside).
//   mmv      4 <= M <= 32, K % 64 == 0, fp32/bf16 input: bitnet_quantize_act
//            into the workspace, then the int8 mma.sync kernel with the
//            tokens as the A operand.
//   decode   9 <= M <= 32, K % 64 == 0, int8 input (natural K order): the
//            int8 mma.sync kernel with the weights as the A operand.
//   prefill  otherwise, K % 64 == 0: bitnet_quantize_act into the workspace
//            (unless xq is given), the weights expanded to int8 into the
//            workspace, then the tcgen05 tensor-core kernel.
//   generic  K % 64 != 0: quantise into the workspace, then the dp4a kernel.
#include <cuda_runtime.h>

#include <mutex>
#include <new>

#include "../../include/bitnet158.h"
#include "internal.h"

namespace bitnet {

__device__ int g_device_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxK = int64_t(1) << 24;
constexpr int64_t kMaxRows = (int64_t(1) << 31) - 1;

struct DeviceInfo {
  int *status = nullptr;
  int num_sms = 0;
  bool ready = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

bitnet_status device_ctx(bitnet_stream_t stream, LaunchCtx *ctx) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BITNET_ERR_CUDA;
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!d.ready) {
      void *addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess) return BITNET_ERR_CUDA;
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BITNET_ERR_CUDA;
      d.status = static_cast<int *>(addr);
      d.num_sms = sms;
      d.ready = true;
    }
  }
  ctx->stream = reinterpret_cast<cudaStream_t>(stream);
  ctx->status = d.status;
  ctx->num_sms = d.num_sms;
  ctx->pdl = true;
  return BITNET_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t elem_size(bitnet_dtype t) {
  switch (t) {
    case BITNET_F32: return 4;
    case BITNET_BF16: return 2;
    case BITNET_I8: return 1;
    case BITNET_I32: return 4;
  }
  return 0;
}

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na > 0 && nb > 0 && x < y + nb && y < x + na;
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

bitnet_status check_k(int64_t K) {
  if (K <= 0) return BITNET_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK) return BITNET_ERR_UNSUPPORTED_SHAPE;
  return BITNET_OK;
}

bitnet_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA; }

// From here on quantise-then-mma.sync beats the fused dp4a kernel (measured
// per call on the decode projections, dependent calls: at M = 2 the fused
// kernel, 3.7 us for 2560 x 2560 against about 5.5 us; at M = 4 the
// mma.sync path, which stays near 5.5 us up to M = 32).
constexpr int64_t kMmvMinM = 4;

// The fused one-launch kernel serves this call (int8 input in natural K
// order always takes it when it can: the mma.sync kernel wants the
// quantiser's unpack order).
bool use_rows(int64_t M, int64_t N, int64_t K, bitnet_dtype x_dtype) {
  return rows_supported(M, N, K) &&
         (x_dtype == BITNET_I8 || M < kMmvMinM || !mmv_supported(M, N, K));
}

// The tensor-core path serves this call (by shape; at run time it also
// needs the driver's tensor-map encoder, else the generic kernel runs, whose
// scratch is a prefix of this path's).
bool use_prefill(int64_t M, int64_t N, int64_t K, bitnet_dtype x_dtype) {
  if (use_rows(M, N, K, x_dtype)) return false;
  if (x_dtype == BITNET_I8 ? decode_supported(M, N, K) : mmv_supported(M, N, K)) return false;
  return prefill_shape_ok(M, N, K);
}

// Scratch the matmul needs, in this order: int8 xq [M][K] and fp32 s [M]
// whenever the activation quantiser runs as its own kernel (float input,
// every path but the fused one), then the int8 weights [N][K] on the
// tensor-core path.  Pure arithmetic: no CUDA call.
size_t act_scratch(int64_t M, int64_t K) {
  return align256(static_cast<size_t>(M) * static_cast<size_t>(K)) +
         align256(4 * static_cast<size_t>(M));
}
size_t matmul_workspace(int64_t M, int64_t N, int64_t K, bitnet_dtype x_dtype) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  if (use_rows(M, N, K, x_dtype)) return 0;
  const size_t act = x_dtype == BITNET_I8 ? 0 : act_scratch(M, K);
  return act + (use_prefill(M, N, K, x_dtype) ? align256(prefill_weight_bytes(N, K)) +
                                                    align256(prefill_ready_bytes(M, N))
                                              : 0);
}

// Argument checks of bitnet_w158a8_matmul (and of its normalising variant,
// which passes s = NULL): BITNET_OK or the status to return.  OK for an
// empty call whatever the pointers.
bitnet_status check_matmul(const void *X, bitnet_dtype x_dtype, const float *s,
                           const uint8_t *packed, const float *gamma, int64_t M, int64_t N,
                           int64_t K, bitnet_epilogue epi, const void *Y, bitnet_dtype y_dtype,
                           const void *workspace, size_t workspace_bytes, uint32_t flags,
                           bool norm_in, bool check_workspace = true) {
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16 && x_dtype != BITNET_I8)
    return BITNET_ERR_INVALID_ARG;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16 && y_dtype != BITNET_I32)
    return BITNET_ERR_INVALID_ARG;
  if (epi != BITNET_EPI_NONE && epi != BITNET_EPI_RELU2) return BITNET_ERR_INVALID_ARG;
  if (y_dtype == BITNET_I32 && epi != BITNET_EPI_NONE) return BITNET_ERR_INVALID_ARG;
  if ((flags & ~(BITNET_FLAG_WEIGHTS_STATIC | BITNET_FLAG_WEIGHTS_EXPANDED |
                 BITNET_FLAG_TABLE_LOOKUP | BITNET_FLAG_PREP_IN_KERNEL)) != 0)
    return BITNET_ERR_INVALID_ARG;
  if ((flags & BITNET_FLAG_TABLE_LOOKUP) != 0 && norm_in) return BITNET_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || M > kMaxRows || N > kMaxRows) return BITNET_ERR_INVALID_ARG;
  if (bitnet_status st = check_k(K)) return st;
  if (M == 0 || N == 0) return BITNET_OK;
  if (X == nullptr || packed == nullptr || gamma == nullptr || Y == nullptr)
    return BITNET_ERR_INVALID_ARG;
  if ((x_dtype == BITNET_I8) != (s != nullptr)) return BITNET_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(packed, 16) || !aligned(Y, 16) || !aligned(gamma, 4) ||
      (s != nullptr && !aligned(s, 4)))
    return BITNET_ERR_MISALIGNED;
  if (overlap(X, static_cast<size_t>(M) * K * elem_size(x_dtype), Y,
              static_cast<size_t>(M) * N * elem_size(y_dtype)))
    return BITNET_ERR_INVALID_ARG;
  // the normalising variant runs the fused kernel, with no scratch, whenever it can
  if ((flags & BITNET_FLAG_TABLE_LOOKUP) != 0)  // the comparison kernel: no scratch
    return lut_supported(M, N, K) ? BITNET_OK : BITNET_ERR_UNSUPPORTED_SHAPE;
  if (!check_workspace) return BITNET_OK;
  const size_t need = norm_in && rows_supported(M, N, K) ? 0 : matmul_workspace(M, N, K, x_dtype);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need) return BITNET_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  }
  return BITNET_OK;
}

// Kernel choice and launches of bitnet_w158a8_matmul once its arguments are
// checked.
bitnet_status run_matmul(const void *X, bitnet_dtype x_dtype, const float *s,
                         const uint8_t *packed, const float *gamma, int64_t M, int64_t N,
                         int64_t K, bool relu2, void *Y, bitnet_dtype y_dtype, void *workspace,
                         bool wstatic, bool expanded, bool prep_in_kernel, const LaunchCtx &ctx) {
  if (use_rows(M, N, K, x_dtype))
    return from_cuda(launch_rows(X, x_dtype, s, packed, gamma, M, N, K, relu2, Y, y_dtype,
                                 wstatic, false, nullptr, ctx));
  const bool from_float = x_dtype != BITNET_I8;
  const bool mmv = from_float && mmv_supported(M, N, K);
  const bool decode = !from_float && decode_supported(M, N, K);  // caller's int8, 9..32 tokens
  const bool prefill = use_prefill(M, N, K, x_dtype) && prefill_supported(M, N, K);
  const int8_t *xq = static_cast<const int8_t *>(X);
  const float *sq = s;
  int8_t *wxq = static_cast<int8_t *>(workspace);
  float *ws = from_float ? reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                                     align256(static_cast<size_t>(M) * K))
                         : nullptr;
  // the tensor-core path's int8 weights follow the activation scratch, then
  // the readiness counters of its in-kernel form
  int8_t *w8 = prefill ? static_cast<int8_t *>(workspace) + (from_float ? act_scratch(M, K) : 0)
                       : nullptr;
  if (prefill && prep_in_kernel) {
    // The tensor-core kernel prepares its own operands while it runs: it
    // quantises fp32/bf16 activations into the workspace (in the K order of
    // its weight unpack) and expands the packed weights after them (unless
    // the caller vouches for an earlier expansion).
    PrefillPrep prep;
    if (from_float) {
      prep.X = X;
      prep.x_kind = x_dtype;
      xq = wxq;
      sq = ws;
    }
    if (!expanded) prep.packed = packed;
    prep.ready = reinterpret_cast<unsigned *>(w8 + align256(prefill_weight_bytes(N, K)));
    return from_cuda(launch_prefill(xq, sq, w8, gamma, M, N, K, relu2, Y, y_dtype, ctx, &prep));
  }
  ExpandJob expand;  // the tensor-core path's weight expansion, unless the caller vouches for one
  if (prefill) {
    expand.packed = packed;
    expand.w8 = w8;
    expand.words = expanded ? 0 : N * (K / 16);
  }
  if (from_float) {
    // The prefill and mmv kernels take the quantiser's output in the K order
    // of their fast weight unpack; the generic kernel wants natural order.
    // The weight expansion rides in the quantiser's launch.
    cudaError_t e = launch_quantize_act(X, x_dtype, M, K, wxq, ws, prefill || mmv, ctx, expand);
    if (e != cudaSuccess) return BITNET_ERR_CUDA;
    xq = wxq;
    sq = ws;
  } else if (prefill && expand.words > 0) {
    // the caller's int8 activations are in natural K order
    if (launch_expand_weights(expand, false, ctx) != cudaSuccess) return BITNET_ERR_CUDA;
  }
  if (prefill)
    return from_cuda(launch_prefill(xq, sq, w8, gamma, M, N, K, relu2, Y, y_dtype, ctx));
  if (mmv)
    return from_cuda(launch_mmv(xq, sq, packed, gamma, M, N, K, relu2, Y, y_dtype, wstatic, ctx));
  if (decode)
    return from_cuda(launch_decode(xq, BITNET_I8, sq, packed, gamma, M, N, K, relu2, Y, y_dtype,
                                   wstatic, ctx));
  return from_cuda(launch_generic(xq, sq, packed, gamma, M, N, K, relu2, Y, y_dtype, ctx));
}

static_assert(kStepRelu2 == BITNET_STEP_RELU2 && kStepNormIn == BITNET_STEP_NORM_IN,
              "step flags");
static_assert(kChainMaxSteps == BITNET_CHAIN_MAX_STEPS, "chain length");

// Checks one chain descriptor list; BITNET_OK or the status to return.
bitnet_status check_chain(const bitnet_chain_step *steps, int n_steps) {
  if (steps == nullptr || n_steps < 1 || n_steps > BITNET_CHAIN_MAX_STEPS)
    return BITNET_ERR_INVALID_ARG;
  for (int s = 0; s < n_steps; ++s) {
    const bitnet_chain_step &d = steps[s];
    if (d.packed == nullptr || d.gamma == nullptr || d.Y == nullptr) return BITNET_ERR_INVALID_ARG;
    if ((d.flags & ~(BITNET_STEP_RELU2 | BITNET_STEP_NORM_IN)) != 0) return BITNET_ERR_INVALID_ARG;
    if (d.X_normed != nullptr && (d.flags & BITNET_STEP_NORM_IN) == 0) return BITNET_ERR_INVALID_ARG;
    if (d.N < 1 || d.K < 1) return BITNET_ERR_INVALID_ARG;
    if (d.N > (int64_t(1) << 22) || d.K % 64 != 0 || d.K < 64 || d.K > chain_max_k())
      return BITNET_ERR_UNSUPPORTED_SHAPE;
    if (s > 0 && d.K > steps[s - 1].N) return BITNET_ERR_INVALID_ARG;
    if (!aligned(d.packed, 16) || !aligned(d.gamma, 4) || !aligned(d.Y, 16) ||
        (d.X_normed != nullptr && !aligned(d.X_normed, 16)))
      return BITNET_ERR_MISALIGNED;
  }
  return BITNET_OK;
}

size_t chain_workspace(const bitnet_chain_step *steps, int n_steps) {
  int64_t words = 0;
  for (int s = 1; s < n_steps; ++s) words += chain_tag_words(steps[s].K);
  return align256(kChainWorkspaceHeader + 4 * static_cast<size_t>(words));
}

}  // namespace

// The argument checks of bitnet_w158a8_matmul without the workspace ones
// (for the entry point that brings its own scratch).
int matmul_args_status(const void *X, int x_dtype, const float *s, const uint8_t *packed,
                       const float *gamma, int64_t M, int64_t N, int64_t K, int epi,
                       const void *Y, int y_dtype, uint32_t flags) {
  return check_matmul(X, static_cast<bitnet_dtype>(x_dtype), s, packed, gamma, M, N, K,
                      static_cast<bitnet_epilogue>(epi), Y, static_cast<bitnet_dtype>(y_dtype),
                      nullptr, 0, flags, false, false);
}

}  // namespace bitnet

using namespace bitnet;

namespace {

// The argument checks of bitnet_w158a8_matmul_host (also those of a plan).
bitnet_status check_host_call(const void *X_host, bitnet_dtype x_dtype, void *X_dev,
                              const uint8_t *packed, const float *gamma, int64_t M, int64_t N,
                              int64_t K, bitnet_epilogue epi, void *Y_dev, void *Y_host,
                              bitnet_dtype y_dtype, void *workspace, size_t workspace_bytes,
                              uint32_t flags) {
  if (x_dtype == BITNET_I8) return BITNET_ERR_INVALID_ARG;
  if (bitnet_status st = check_matmul(X_dev, x_dtype, nullptr, packed, gamma, M, N, K, epi, Y_dev,
                                      y_dtype, workspace, workspace_bytes, flags, false))
    return st;
  if (M == 0 || N == 0) return BITNET_OK;
  if (X_host == nullptr || Y_host == nullptr) return BITNET_ERR_INVALID_ARG;
  return BITNET_OK;
}

// Copy in, the product, copy out, all on ctx.stream (no wait).
bitnet_status enqueue_host_call(const void *X_host, bitnet_dtype x_dtype, void *X_dev,
                                const uint8_t *packed, const float *gamma, int64_t M, int64_t N,
                                int64_t K, bitnet_epilogue epi, void *Y_dev, void *Y_host,
                                bitnet_dtype y_dtype, void *workspace, uint32_t flags,
                                const LaunchCtx &ctx) {
  const size_t x_bytes = static_cast<size_t>(M) * K * elem_size(x_dtype);
  const size_t y_bytes = static_cast<size_t>(M) * N * elem_size(y_dtype);
  // a few KB (decode): a copy kernel chained to the product; more: the copy engine
  const cudaError_t in =
      small_copy_ok(X_host, X_dev, x_bytes)
          ? launch_small_copy(X_host, X_dev, x_bytes, ctx)
          : cudaMemcpyAsync(X_dev, X_host, x_bytes, cudaMemcpyHostToDevice, ctx.stream);
  if (in != cudaSuccess) return BITNET_ERR_CUDA;
  const bool relu2 = epi == BITNET_EPI_RELU2, wstatic = (flags & BITNET_FLAG_WEIGHTS_STATIC) != 0;
  const bitnet_status st =
      (flags & BITNET_FLAG_TABLE_LOOKUP) != 0
          ? from_cuda(launch_lut(X_dev, x_dtype, nullptr, packed, gamma, M, N, K, relu2, Y_dev,
                                 y_dtype, wstatic, ctx))
          : run_matmul(X_dev, x_dtype, nullptr, packed, gamma, M, N, K, relu2, Y_dev, y_dtype,
                       workspace, wstatic, (flags & BITNET_FLAG_WEIGHTS_EXPANDED) != 0,
                       (flags & BITNET_FLAG_PREP_IN_KERNEL) != 0, ctx);
  if (st != BITNET_OK) return st;
  const cudaError_t out =
      small_copy_ok(Y_host, Y_dev, y_bytes)
          ? launch_small_copy(Y_dev, Y_host, y_bytes, ctx)
          : cudaMemcpyAsync(Y_host, Y_dev, y_bytes, cudaMemcpyDeviceToHost, ctx.stream);
  return out == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

// The same work for a large call on the tensor-core path, as a pipeline of
// token chunks over three streams: chunk c + 1 is copied in (stream `in`)
// while chunk c is computed (ctx.stream) and the finished chunks are copied
// out (stream `out`), so that the two copy directions and the product
// overlap.  Every chunk but the last has the same number of tokens, so the
// int8 weights the first chunk expanded into the workspace sit where the
// next equal chunks look for them (BITNET_FLAG_WEIGHTS_EXPANDED); the last,
// smaller chunk expands them again.  Only recorded into a plan's graph: the
// streams and events are the capture's and are released after it.
constexpr int64_t kPipeChunks = 8;
constexpr int64_t kPipeMinTokens = 256;
constexpr size_t kPipeMinBytes = size_t(4) << 20;

bool pipeline_fits(bitnet_dtype x_dtype, int64_t M, int64_t N, int64_t K, bitnet_dtype y_dtype,
                   uint32_t flags) {
  if ((flags & ~BITNET_FLAG_WEIGHTS_STATIC) != 0) return false;
  if (M < kPipeMinTokens || !use_prefill(M, N, K, x_dtype) || !prefill_supported(M, N, K))
    return false;
  return static_cast<size_t>(M) * (K * elem_size(x_dtype) + N * elem_size(y_dtype)) >=
         kPipeMinBytes;
}

// Side streams and events of a pipelined capture, made before it and
// released after it ends (a stream that joined a capture must not go away
// while the capture is open).
struct PipeRes {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t ev[2 * kPipeChunks + 3] = {};
  bool make() {
    if (cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking) != cudaSuccess)
      return false;
    for (cudaEvent_t &e : ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
  void release() {
    for (cudaEvent_t &e : ev)
      if (e != nullptr) cudaEventDestroy(e);
    if (in != nullptr) cudaStreamDestroy(in);
    if (out != nullptr) cudaStreamDestroy(out);
  }
};

bitnet_status enqueue_host_pipeline(const void *X_host, bitnet_dtype x_dtype, void *X_dev,
                                    const uint8_t *packed, const float *gamma, int64_t M,
                                    int64_t N, int64_t K, bitnet_epilogue epi, void *Y_dev,
                                    void *Y_host, bitnet_dtype y_dtype, void *workspace,
                                    uint32_t flags, const PipeRes &r, const LaunchCtx &ctx) {
  const int64_t per = ceil_div(ceil_div(M, kPipeChunks), int64_t(128)) * 128;  // whole row tiles
  const int64_t chunks = ceil_div(M, per);  // <= kPipeChunks
  const size_t xrow = static_cast<size_t>(K) * elem_size(x_dtype);
  const size_t yrow = static_cast<size_t>(N) * elem_size(y_dtype);
  // fork: both side streams join the capture after the main stream's start
  if (cudaEventRecord(r.ev[0], ctx.stream) != cudaSuccess ||
      cudaStreamWaitEvent(r.in, r.ev[0], 0) != cudaSuccess ||
      cudaStreamWaitEvent(r.out, r.ev[0], 0) != cudaSuccess)
    return BITNET_ERR_CUDA;
  bitnet_status st = BITNET_OK;
  const bool relu2 = epi == BITNET_EPI_RELU2, wstatic = (flags & BITNET_FLAG_WEIGHTS_STATIC) != 0;
  for (int64_t c = 0; st == BITNET_OK && c < chunks; ++c) {
    const int64_t m0 = c * per, mc = M - m0 < per ? M - m0 : per;
    uint8_t *xd = static_cast<uint8_t *>(X_dev) + static_cast<size_t>(m0) * xrow;
    uint8_t *yd = static_cast<uint8_t *>(Y_dev) + static_cast<size_t>(m0) * yrow;
    const cudaEvent_t in_done = r.ev[1 + 2 * c], y_done = r.ev[2 + 2 * c];
    if (cudaMemcpyAsync(xd, static_cast<const uint8_t *>(X_host) + static_cast<size_t>(m0) * xrow,
                        static_cast<size_t>(mc) * xrow, cudaMemcpyHostToDevice, r.in) != cudaSuccess ||
        cudaEventRecord(in_done, r.in) != cudaSuccess ||
        cudaStreamWaitEvent(ctx.stream, in_done, 0) != cudaSuccess) {
      st = BITNET_ERR_CUDA;
      break;
    }
    const bool reuse = c > 0 && mc == per;  // the first chunk's expansion, at the same offset
    st = run_matmul(xd, x_dtype, nullptr, packed, gamma, mc, N, K, relu2, yd, y_dtype, workspace,
                    wstatic, reuse, false, ctx);
    if (st != BITNET_OK) break;
    if (cudaEventRecord(y_done, ctx.stream) != cudaSuccess ||
        cudaStreamWaitEvent(r.out, y_done, 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t *>(Y_host) + static_cast<size_t>(m0) * yrow, yd,
                        static_cast<size_t>(mc) * yrow, cudaMemcpyDeviceToHost, r.out) != cudaSuccess)
      st = BITNET_ERR_CUDA;
  }
  // join (also after an error, so that the capture can end): the main
  // stream ends after both side streams
  const cudaEvent_t join_in = r.ev[2 * kPipeChunks + 1], join_out = r.ev[2 * kPipeChunks + 2];
  if (cudaEventRecord(join_in, r.in) != cudaSuccess ||
      cudaStreamWaitEvent(ctx.stream, join_in, 0) != cudaSuccess ||
      cudaEventRecord(join_out, r.out) != cudaSuccess ||
      cudaStreamWaitEvent(ctx.stream, join_out, 0) != cudaSuccess)
    st = BITNET_ERR_CUDA;
  return st;
}

}  // namespace

// A host-to-host call captured once as a CUDA graph.
struct bitnet_host_plan_s {
  cudaGraphExec_t exec;
  cudaStream_t stream;
};

extern "C" {

int bitnet_version(void) { return BITNET_VERSION; }

const char *bitnet_status_string(bitnet_status status) {
  switch (status) {
    case BITNET_OK: return "ok";
    case BITNET_ERR_INVALID_ARG: return "invalid argument";
    case BITNET_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BITNET_ERR_MISALIGNED: return "misaligned pointer";
    case BITNET_ERR_CUDA: return "CUDA error";
    case BITNET_ERR_TIMEOUT: return "device wait timed out";
    case BITNET_ERR_RANGE: return "input outside the numeric contract";
    case BITNET_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

size_t bitnet_quantize_weights_workspace_size(int64_t N, int64_t K) {
  (void)K;
  return N > 0 ? align256(8 * static_cast<size_t>(N)) : 0;
}

bitnet_status bitnet_quantize_weights(const void *W, bitnet_dtype w_dtype, int64_t N, int64_t K,
                                      uint8_t *packed, float *gamma, void *workspace,
                                      size_t workspace_bytes, bitnet_stream_t stream) {
  if (W == nullptr || packed == nullptr || gamma == nullptr) return BITNET_ERR_INVALID_ARG;
  if (w_dtype != BITNET_F32 && w_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (N <= 0 || N > kMaxRows) return BITNET_ERR_INVALID_ARG;
  if (bitnet_status st = check_k(K)) return st;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(gamma, 4)) return BITNET_ERR_MISALIGNED;
  const size_t need = bitnet_quantize_weights_workspace_size(N, K);
  if (workspace == nullptr || workspace_bytes < need) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  if (overlap(W, static_cast<size_t>(N) * K * elem_size(w_dtype), packed,
              static_cast<size_t>(N) * (K / 4)))
    return BITNET_ERR_INVALID_ARG;
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  return from_cuda(launch_quantize_weights(W, w_dtype, N, K, packed, gamma,
                                           static_cast<double *>(workspace), ctx));
}

bitnet_status bitnet_quantize_act(const void *X, bitnet_dtype x_dtype, int64_t M, int64_t K,
                                  int8_t *xq, float *s, bitnet_stream_t stream) {
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (M < 0 || M > kMaxRows) return BITNET_ERR_INVALID_ARG;
  if (bitnet_status st = check_k(K)) return st;
  if (M == 0) return BITNET_OK;  // empty: pointers may be NULL
  if (X == nullptr || xq == nullptr || s == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(xq, 16) || !aligned(s, 4)) return BITNET_ERR_MISALIGNED;
  if (overlap(X, static_cast<size_t>(M) * K * elem_size(x_dtype), xq, static_cast<size_t>(M) * K))
    return BITNET_ERR_INVALID_ARG;
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  return from_cuda(launch_quantize_act(X, x_dtype, M, K, xq, s, false, ctx));
}

size_t bitnet_w158a8_matmul_workspace_size(int64_t M, int64_t N, int64_t K, bitnet_dtype x_dtype) {
  return matmul_workspace(M, N, K, x_dtype);
}

bitnet_status bitnet_w158a8_matmul_host(const void *X_host, bitnet_dtype x_dtype, void *X_dev,
                                        const uint8_t *packed, const float *gamma, int64_t M,
                                        int64_t N, int64_t K, bitnet_epilogue epi, void *Y_dev,
                                        void *Y_host, bitnet_dtype y_dtype, void *workspace,
                                        size_t workspace_bytes, uint32_t flags,
                                        bitnet_stream_t stream) {
  if (bitnet_status st = check_host_call(X_host, x_dtype, X_dev, packed, gamma, M, N, K, epi, Y_dev,
                                         Y_host, y_dtype, workspace, workspace_bytes, flags))
    return st;
  if (M == 0 || N == 0) return BITNET_OK;
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  if (bitnet_status st = enqueue_host_call(X_host, x_dtype, X_dev, packed, gamma, M, N, K, epi,
                                           Y_dev, Y_host, y_dtype, workspace, flags, ctx))
    return st;
  return cudaStreamSynchronize(ctx.stream) == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

bitnet_status bitnet_host_plan_create(const void *X_host, bitnet_dtype x_dtype, void *X_dev,
                                      const uint8_t *packed, const float *gamma, int64_t M,
                                      int64_t N, int64_t K, bitnet_epilogue epi, void *Y_dev,
                                      void *Y_host, bitnet_dtype y_dtype, void *workspace,
                                      size_t workspace_bytes, uint32_t flags,
                                      bitnet_stream_t stream, bitnet_host_plan *plan) {
  if (plan == nullptr) return BITNET_ERR_INVALID_ARG;
  *plan = nullptr;
  if (bitnet_status st = check_host_call(X_host, x_dtype, X_dev, packed, gamma, M, N, K, epi, Y_dev,
                                         Y_host, y_dtype, workspace, workspace_bytes, flags))
    return st;
  if (M == 0 || N == 0) return BITNET_ERR_INVALID_ARG;
  // the graph's copies need page-locked host memory
  for (const void *h : {X_host, static_cast<const void *>(Y_host)}) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, h) != cudaSuccess) {
      (void)cudaGetLastError();
      return BITNET_ERR_INVALID_ARG;
    }
    if (a.type != cudaMemoryTypeHost) return BITNET_ERR_INVALID_ARG;
  }
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  // Captured on a stream of its own (the caller's may be the legacy default
  // stream, which cannot be captured), launched later on the caller's.
  cudaStream_t cap = nullptr;
  if (cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking) != cudaSuccess) return BITNET_ERR_CUDA;
  LaunchCtx cctx = ctx;
  cctx.stream = cap;
  cudaGraph_t graph = nullptr;
  bitnet_status st = BITNET_OK;
  const bool pipe = pipeline_fits(x_dtype, M, N, K, y_dtype, flags);
  PipeRes res;
  if (pipe && !res.make()) st = BITNET_ERR_CUDA;
  if (st == BITNET_OK && cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    st = BITNET_ERR_CUDA;
  else if (st == BITNET_OK) {
    st = pipe ? enqueue_host_pipeline(X_host, x_dtype, X_dev, packed, gamma, M, N, K, epi, Y_dev,
                                      Y_host, y_dtype, workspace, flags, res, cctx)
              : enqueue_host_call(X_host, x_dtype, X_dev, packed, gamma, M, N, K, epi, Y_dev,
                                  Y_host, y_dtype, workspace, flags, cctx);
    // always end the capture, also after a failed enqueue
    if (cudaStreamEndCapture(cap, &graph) != cudaSuccess && st == BITNET_OK) st = BITNET_ERR_CUDA;
  }
  res.release();
  cudaGraphExec_t exec = nullptr;
  if (st == BITNET_OK &&
      (graph == nullptr || cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess))
    st = BITNET_ERR_CUDA;
  // uploaded now, on the caller's stream, so that the first run costs what
  // every later one does
  if (st == BITNET_OK && cudaGraphUpload(exec, ctx.stream) != cudaSuccess) st = BITNET_ERR_CUDA;
  if (graph != nullptr) cudaGraphDestroy(graph);
  cudaStreamDestroy(cap);
  if (st != BITNET_OK) {
    (void)cudaGetLastError();
    if (exec != nullptr) cudaGraphExecDestroy(exec);
    return st;
  }
  bitnet_host_plan made = new (std::nothrow) bitnet_host_plan_s{exec, ctx.stream};
  if (made == nullptr) {  // no exception crosses the C boundary
    cudaGraphExecDestroy(exec);
    return BITNET_ERR_CUDA;
  }
  *plan = made;
  return BITNET_OK;
}

bitnet_status bitnet_host_plan_run(bitnet_host_plan plan) {
  if (plan == nullptr) return BITNET_ERR_INVALID_ARG;
  if (cudaGraphLaunch(plan->exec, plan->stream) != cudaSuccess) return BITNET_ERR_CUDA;
  return cudaStreamSynchronize(plan->stream) == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

void bitnet_host_plan_destroy(bitnet_host_plan plan) {
  if (plan == nullptr) return;
  cudaGraphExecDestroy(plan->exec);
  delete plan;
}

bitnet_path bitnet_w158a8_matmul_path(int64_t M, int64_t N, int64_t K, bitnet_dtype x_dtype) {
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16 && x_dtype != BITNET_I8)
    return BITNET_PATH_NONE;
  if (M <= 0 || N <= 0 || M > kMaxRows || N > kMaxRows || check_k(K) != BITNET_OK)
    return BITNET_PATH_NONE;
  if (use_rows(M, N, K, x_dtype)) return BITNET_PATH_ROWS;
  if (x_dtype != BITNET_I8 && mmv_supported(M, N, K)) return BITNET_PATH_MMA_TOKENS;
  if (x_dtype == BITNET_I8 && decode_supported(M, N, K)) return BITNET_PATH_MMA_WEIGHTS;
  // the same decision run_matmul takes, the encoder lookup included
  if (use_prefill(M, N, K, x_dtype) && prefill_supported(M, N, K)) return BITNET_PATH_TENSOR_CORE;
  return BITNET_PATH_GENERIC;
}

bitnet_status bitnet_w158a8_matmul(const void *X, bitnet_dtype x_dtype, const float *s,
                                   const uint8_t *packed, const float *gamma, int64_t M,
                                   int64_t N, int64_t K, bitnet_epilogue epi, void *Y,
                                   bitnet_dtype y_dtype, void *workspace, size_t workspace_bytes,
                                   uint32_t flags, bitnet_stream_t stream) {
  if (bitnet_status st = check_matmul(X, x_dtype, s, packed, gamma, M, N, K, epi, Y, y_dtype,
                                      workspace, workspace_bytes, flags, false))
    return st;
  if (M == 0 || N == 0) return BITNET_OK;  // empty: pointers may be NULL
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  if ((flags & BITNET_FLAG_TABLE_LOOKUP) != 0)
    return from_cuda(launch_lut(X, x_dtype, s, packed, gamma, M, N, K, epi == BITNET_EPI_RELU2, Y,
                                y_dtype, (flags & BITNET_FLAG_WEIGHTS_STATIC) != 0, ctx));
  return run_matmul(X, x_dtype, s, packed, gamma, M, N, K, epi == BITNET_EPI_RELU2, Y, y_dtype,
                    workspace, (flags & BITNET_FLAG_WEIGHTS_STATIC) != 0,
                    (flags & BITNET_FLAG_WEIGHTS_EXPANDED) != 0,
                    (flags & BITNET_FLAG_PREP_IN_KERNEL) != 0, ctx);
}

bitnet_status bitnet_rms_norm_w158a8_matmul(const void *X, bitnet_dtype x_dtype, void *X_normed,
                                            const uint8_t *packed, const float *gamma,
                                            int64_t M, int64_t N, int64_t K,
                                            bitnet_epilogue epi, void *Y, bitnet_dtype y_dtype,
                                            void *workspace, size_t workspace_bytes,
                                            uint32_t flags, bitnet_stream_t stream) {
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (bitnet_status st = check_matmul(X, x_dtype, nullptr, packed, gamma, M, N, K, epi, Y, y_dtype,
                                      workspace, workspace_bytes, flags, true))
    return st;
  if (M == 0 || N == 0) return BITNET_OK;
  const size_t x_bytes = static_cast<size_t>(M) * K * elem_size(x_dtype);
  const bool fused = rows_supported(M, N, K);  // the NORM variant of the fused kernel, M <= 8
  if (!fused && X_normed == nullptr) return BITNET_ERR_INVALID_ARG;  // needed as the matmul input
  if (X_normed != nullptr) {
    if (!aligned(X_normed, 16)) return BITNET_ERR_MISALIGNED;
    if (overlap(X, x_bytes, X_normed, x_bytes) ||
        overlap(Y, static_cast<size_t>(M) * N * elem_size(y_dtype), X_normed, x_bytes))
      return BITNET_ERR_INVALID_ARG;
  }
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  const bool relu2 = epi == BITNET_EPI_RELU2;
  const bool wstatic = (flags & BITNET_FLAG_WEIGHTS_STATIC) != 0;
  if (fused)
    return from_cuda(launch_rows(X, x_dtype, nullptr, packed, gamma, M, N, K, relu2, Y, y_dtype,
                                 wstatic, true, X_normed, ctx));
  if (launch_rms_norm(X, x_dtype, M, K, X_normed, x_dtype, ctx) != cudaSuccess) return BITNET_ERR_CUDA;
  return run_matmul(X_normed, x_dtype, nullptr, packed, gamma, M, N, K, relu2, Y, y_dtype,
                    workspace, wstatic, (flags & BITNET_FLAG_WEIGHTS_EXPANDED) != 0,
                    (flags & BITNET_FLAG_PREP_IN_KERNEL) != 0, ctx);
}

bitnet_status bitnet_rms_norm(const void *X, bitnet_dtype x_dtype, int64_t M, int64_t K, void *Y,
                              bitnet_dtype y_dtype, bitnet_stream_t stream) {
  if ((x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) ||
      (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16))
    return BITNET_ERR_INVALID_ARG;
  if (M < 0 || M > kMaxRows) return BITNET_ERR_INVALID_ARG;
  if (bitnet_status st = check_k(K)) return st;
  if (M == 0) return BITNET_OK;  // empty: pointers may be NULL
  if (X == nullptr || Y == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Y, 16)) return BITNET_ERR_MISALIGNED;
  if (X != Y && overlap(X, static_cast<size_t>(M) * K * elem_size(x_dtype), Y,
                        static_cast<size_t>(M) * K * elem_size(y_dtype)))
    return BITNET_ERR_INVALID_ARG;
  if (X == Y && x_dtype != y_dtype) return BITNET_ERR_INVALID_ARG;
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  return from_cuda(launch_rms_norm(X, x_dtype, M, K, Y, y_dtype, ctx));
}

size_t bitnet_decode_chain_workspace_size(const bitnet_chain_step *steps, int n_steps) {
  if (check_chain(steps, n_steps) != BITNET_OK) return 0;
  return chain_workspace(steps, n_steps);
}

bitnet_status bitnet_decode_chain(const bitnet_chain_step *steps, int n_steps, const void *x0,
                                  void *y_norm, void *workspace, size_t workspace_bytes,
                                  bitnet_stream_t stream) {
  if (bitnet_status st = check_chain(steps, n_steps)) return st;
  if (x0 == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x0, 16) || (y_norm != nullptr && !aligned(y_norm, 16))) return BITNET_ERR_MISALIGNED;
  const int64_t n_last = steps[n_steps - 1].N;
  if (y_norm != nullptr && (n_last % 16 != 0 || n_last > chain_max_k()))
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  // x0 is read by every CTA during the first step: no output may overlap it
  const size_t x0_bytes = 2 * static_cast<size_t>(steps[0].K);
  for (int s = 0; s < n_steps; ++s) {
    if (overlap(x0, x0_bytes, steps[s].Y, 2 * static_cast<size_t>(steps[s].N)) ||
        (steps[s].X_normed != nullptr &&
         overlap(x0, x0_bytes, steps[s].X_normed, 2 * static_cast<size_t>(steps[s].K))))
      return BITNET_ERR_INVALID_ARG;
  }
  if (y_norm != nullptr && overlap(x0, x0_bytes, y_norm, 2 * static_cast<size_t>(n_last)))
    return BITNET_ERR_INVALID_ARG;
  const size_t need = chain_workspace(steps, n_steps);
  if (workspace == nullptr || workspace_bytes < need) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return BITNET_ERR_MISALIGNED;
  LaunchCtx ctx;
  if (bitnet_status st = device_ctx(stream, &ctx)) return st;
  ChainStep cs[kChainMaxSteps];
  for (int s = 0; s < n_steps; ++s)
    cs[s] = ChainStep{steps[s].packed, steps[s].gamma, steps[s].N, steps[s].K, steps[s].flags,
                      steps[s].Y, steps[s].X_normed};
  ChainPlan plan;
  if (!chain_plan(cs, n_steps, ctx.num_sms, &plan)) return BITNET_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_chain(cs, n_steps, plan, x0, y_norm, n_last, workspace, ctx));
}

bitnet_status bitnet_get_device_status(bitnet_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BITNET_ERR_CUDA;
  int value = 0;
  if (cudaMemcpyFromSymbol(&value, g_device_status, sizeof(int)) != cudaSuccess)
    return BITNET_ERR_CUDA;
  if (value != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
      return BITNET_ERR_CUDA;
  }
  return static_cast<bitnet_status>(value);
}

}  // extern "C"
