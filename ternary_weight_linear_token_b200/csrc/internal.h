// internal.h -- host-side launchers shared between the C-ABI file and the
// kernel files.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace bitnet {

// Element kinds used by the kernels (mirror bitnet_dtype values).
enum Kind : int { kF32 = 0, kBF16 = 1, kI8 = 2, kI32 = 3 };

struct LaunchCtx {
  cudaStream_t stream;
  int *status;      // device status word of the current device
  int num_sms;
  bool pdl;         // launch with programmatic stream serialization
};

// quant_weights.cu
cudaError_t launch_quantize_weights(const void *W, int w_kind, int64_t N, int64_t K,
                                    uint8_t *packed, float *gamma, double *row_sums,
                                    const LaunchCtx &ctx);

// quant_act.cu
// permuted: store each 16-element group of xq in the order the byte-permute
// weight unpack produces (internal layout of the prefill kernel's A operand).
// The packed weights [N][K/4] expanded to int8 [N][K] (scratch of the
// tensor-core path): words = N * K / 16 packed words, 0 for none.
struct ExpandJob {
  const uint8_t *packed = nullptr;
  int8_t *w8 = nullptr;
  int64_t words = 0;
};
cudaError_t launch_quantize_act(const void *X, int x_kind, int64_t M, int64_t K, int8_t *xq,
                                float *s, bool permuted, const LaunchCtx &ctx,
                                const ExpandJob &expand = ExpandJob{});
// The expansion alone (int8 activations given by the caller).
cudaError_t launch_expand_weights(const ExpandJob &job, bool permuted, const LaunchCtx &ctx);
cudaError_t launch_rms_norm(const void *X, int x_kind, int64_t M, int64_t K, void *Y, int y_kind,
                            const LaunchCtx &ctx);

// gemv_rows.cu: lowest-latency kernel for 1 <= M <= 8 tokens, any K % 16 == 0.
// norm (float input only): RMS-normalise each token first; CTA 0 writes the
// normalised input to Xn when it is not null.
bool rows_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_rows(const void *X, int x_kind, const float *s, const uint8_t *packed,
                        const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2, void *Y,
                        int y_kind, bool weights_static, bool norm, void *Xn,
                        const LaunchCtx &ctx);

// gemv_lut.cu: table-lookup comparison kernel for 1 <= M <= 8 tokens, K % 16 == 0.
bool lut_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_lut(const void *X, int x_kind, const float *s, const uint8_t *packed,
                       const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2, void *Y,
                       int y_kind, bool weights_static, const LaunchCtx &ctx);

// gemv_decode.cu: fused decode kernel, M <= 32, K % 64 == 0.
bool decode_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_decode(const void *X, int x_kind, const float *s, const uint8_t *packed,
                          const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2,
                          void *Y, int y_kind, bool weights_static, const LaunchCtx &ctx);

// gemv_mma.cu: int8 mma.sync with the tokens as the A operand, M <= 32,
// K % 64 == 0; xq from launch_quantize_act(permuted = true).
bool mmv_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_mmv(const int8_t *xq, const float *s, const uint8_t *packed, const float *gamma,
                       int64_t M, int64_t N, int64_t K, bool relu2, void *Y, int y_kind,
                       bool weights_static, const LaunchCtx &ctx);

// gemm_generic.cu: any M, K % 16 == 0, int8 activations already quantised.
cudaError_t launch_generic(const int8_t *xq, const float *s, const uint8_t *packed,
                           const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2,
                           void *Y, int y_kind, const LaunchCtx &ctx);

// gemm_prefill.cu: the tcgen05 tensor-core kernel on int8 xq and int8
// weights w8 [N][K] (expanded beforehand, in xq's K order); K % 64 == 0.
// prefill_shape_ok is the shape rule alone (no CUDA call);
// prefill_supported also needs the driver's tensor-map encoder.
bool prefill_shape_ok(int64_t M, int64_t N, int64_t K);
bool prefill_supported(int64_t M, int64_t N, int64_t K);
size_t prefill_weight_bytes(int64_t N, int64_t K);
// Operands the tensor-core kernel prepares itself while it runs (the fused
// form): the raw activations X (quantised, in xq's K order, into xq and s),
// and/or the packed weights (expanded into w8).  `ready` is scratch of
// prefill_ready_bytes(M, N) bytes for its per-block readiness counters.
struct PrefillPrep {
  const void *X = nullptr;        // null: xq and s are given
  int x_kind = 0;
  const uint8_t *packed = nullptr;  // null: w8 is given
  unsigned *ready = nullptr;
};
size_t prefill_ready_bytes(int64_t M, int64_t N);
cudaError_t launch_prefill(const int8_t *xq, const float *s, const int8_t *w8,
                           const float *gamma, int64_t M, int64_t N, int64_t K, bool relu2,
                           void *Y, int y_kind, const LaunchCtx &ctx,
                           const PrefillPrep *prep = nullptr);

// host_copy.cu: small copies between page-locked host memory and the device
// by a kernel (16-byte pieces, programmatic dependent launch).  small_copy_ok:
// bytes <= kSmallCopyMax, a multiple of 16, both pointers 16-byte aligned and
// `host` page-locked memory the device addresses at the same address.
constexpr size_t kSmallCopyMax = 64 * 1024;
bool small_copy_ok(const void *host, const void *dev, size_t bytes);
cudaError_t launch_small_copy(const void *src, void *dst, size_t bytes, const LaunchCtx &ctx);

// chain.cu: persistent M = 1 chain of BitLinear projections (one
// cooperative launch).  Step flags mirror BITNET_STEP_*.
constexpr int kChainMaxSteps = 256;
constexpr int kStepRelu2 = 1;
constexpr int kStepNormIn = 2;
constexpr int kChainMaxCtas = 256;              // CTAs of one chain launch, at most
// Workspace: the launch counter at byte 0, the done counter at byte 128,
// then for every step but the last the tagged words of the part of its
// output the next step reads (its K values), each step's run a whole number
// of 128-byte lines.
constexpr size_t kChainWorkspaceHeader = 256;
constexpr size_t kChainDoneOffset = 128;
inline int64_t chain_tag_words(int64_t k_next) { return (k_next + 31) / 32 * 32; }
struct ChainStep {
  const uint8_t *packed;
  const float *gamma;
  int64_t N, K;
  uint32_t flags;
  void *Y;
  void *Xn;
};
struct ChainPlan {
  int ctas, slots, slot_bytes, xq_bytes;
  size_t smem;
};
int chain_max_k();
bool chain_plan(const ChainStep *steps, int n_steps, int num_sms, ChainPlan *plan);
cudaError_t launch_chain(const ChainStep *steps, int n_steps, const ChainPlan &plan,
                         const void *x0, void *y_norm, int64_t y_norm_n, void *workspace,
                         const LaunchCtx &ctx);

// abi.cu: the argument checks of bitnet_w158a8_matmul without the workspace
// ones, as a bitnet_status value (0 = OK).
int matmul_args_status(const void *X, int x_dtype, const float *s, const uint8_t *packed,
                       const float *gamma, int64_t M, int64_t N, int64_t K, int epi,
                       const void *Y, int y_dtype, uint32_t flags);

// Launch helper: cudaLaunchKernelEx with the PDL attribute when ctx.pdl.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     const LaunchCtx &ctx, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ctx.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ctx.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The same launch as clusters of `cluster_x` CTAs along x (gridDim.x a
// multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_k_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             unsigned cluster_x, const LaunchCtx &ctx, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ctx.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ctx.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace bitnet
