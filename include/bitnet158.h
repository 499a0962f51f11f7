/*
 * bitnet158.h -- C ABI of the B200 (sm_100a) BitLinear forward of BitNet b1.58
 * (W1.58A8: ternary weights, 8-bit activations).
 *
 * The operation (sources are web pages on BitNet b1.58, cited by title and
 * section):
 *
 *   weights     gamma = mean |W| over the whole [N, K] matrix;
 *               Q(w)  = round(clamp(w / gamma, -1, 1)) in {-1, 0, +1};
 *               stored as the 2-bit value {0 -> 0, +1 -> 1, -1 -> 2}.
 *               ("Microsoft BitNet 深度研究报告", 技术原理 item 2, AbsMean 量化)
 *               Four 2-bit values per byte.  (Write-up of the BitNet b1.58
 *               2B4T technical report, "GPU端：CUDA内核的定制魔法".)
 *   activations per token m: s_m = 127 / max_k |x_mk|;
 *               xq = clamp(round(x * s_m), -127, 127) as int8.
 *               (BitNet b1.58 2B4T model card, 模型详情 -> 量化: per-token
 *               absmax 8-bit activations.)
 *   product     acc[m][n] = sum_k xq[m][k] * Q(W)[n][k], exact in int32
 *               (the add/subtract form of item 3 of the research report);
 *               y[m][n] = (float)acc * (gamma / s_m), then optionally ReLU^2
 *               (model card, 架构: squared ReLU in the FFN; no bias terms).
 *
 * Readings where the pages say nothing (the same in the CPU oracle):
 *   round = half away from zero; gamma is summed in fp64, each row in k
 *   order, then the rows in n order, and rounded once to fp32; gamma == 0
 *   gives all-zero codes; an all-zero activation row gives s = 1 and xq = 0;
 *   y = (float)acc * (gamma / s) with one fp32 division and one fp32
 *   multiply; bf16 outputs round to nearest even.
 *   Packed layout: row-major [N][K/4] bytes.  Inside each group of 16
 *   consecutive elements of a row one little-endian 32-bit word holds
 *   element 16g + 4j + i at bits [8i + 2j, 8i + 2j + 2), i, j in 0..3 (so
 *   byte i of the word holds elements i, i+4, i+8, i+12).  Code 3 is never
 *   written; packed input containing it gives unspecified results.
 *
 * Conventions for every entry point:
 *   - Every array argument is a DEVICE pointer owned by the caller; the
 *     library keeps no pointer after the call returns and allocates no
 *     device memory (scratch comes from the caller's workspace argument).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; gamma and s stay on the device.
 *   - Arguments are checked on the host before anything is launched; a
 *     failed check returns an error status and launches nothing.  Errors are
 *     return codes only: no exception, abort or device trap.
 *   - Arrays are dense row-major.  X, xq, Y and packed must be 16-byte
 *     aligned; s and gamma 4-byte aligned; workspaces 256-byte aligned.
 *   - M == 0 or N == 0 is an empty call that returns BITNET_OK and launches
 *     nothing; its array pointers may then be NULL.  K must be a positive multiple of 16 (one packed word) and at
 *     most 2^24 (so |acc| <= 127 * K stays inside int32).
 *   - A kernel that gives up a bounded wait records BITNET_ERR_TIMEOUT in a
 *     device status word; bitnet_get_device_status() reads and clears it.
 */
#ifndef BITNET158_H
#define BITNET158_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t (declared here without the CUDA headers). */
typedef struct CUstream_st *bitnet_stream_t;

typedef enum bitnet_status {
    BITNET_OK = 0,
    BITNET_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size, aliasing */
    BITNET_ERR_UNSUPPORTED_SHAPE = 2, /* K not a positive multiple of 16, or K > 2^24    */
    BITNET_ERR_MISALIGNED = 3,        /* a pointer breaks the alignment rule above       */
    BITNET_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed            */
    BITNET_ERR_TIMEOUT = 5,           /* a device-side bounded wait gave up              */
    BITNET_ERR_RANGE = 6,             /* reserved: input outside the numeric contract    */
    BITNET_ERR_WORKSPACE = 7          /* workspace missing or smaller than required      */
} bitnet_status;

typedef enum bitnet_dtype {
    BITNET_F32 = 0,
    BITNET_BF16 = 1,
    BITNET_I8 = 2,
    BITNET_I32 = 3
} bitnet_dtype;

typedef enum bitnet_epilogue {
    BITNET_EPI_NONE = 0,
    BITNET_EPI_RELU2 = 1  /* y = max(y, 0)^2, the FFN activation of the model card */
} bitnet_epilogue;

/* Flag for bitnet_w158a8_matmul: `packed` and `gamma` are not written by the
 * kernel that precedes this call on `stream`.  With it the kernel may start
 * streaming the weights from HBM before the preceding kernel has finished
 * (programmatic dependent launch); the activations are still read, and Y
 * written, only after the preceding kernel has completed.  Without it the
 * weights are also read only after that point. */
#define BITNET_FLAG_WEIGHTS_STATIC 1u

/* Flag for bitnet_w158a8_matmul: the workspace already holds the int8 copy
 * of these packed weights that the tensor-core path makes, written by an
 * earlier call with the same `packed`, N, K and the same kind of input
 * (int8 activations, or fp32/bf16 ones: the two keep the copy in different
 * K orders), on this workspace, and nothing has written that part of the
 * workspace since.  The call then skips the expansion and only quantises
 * the activations (fp32/bf16 input) and runs the tensor-core kernel.  For a
 * prefill that reuses one weight matrix over many calls (token blocks of a
 * long prompt, several prompts in turn) this saves N*K/4 bytes read and N*K
 * written per call.  Calls on the other paths keep no weight copy and
 * ignore the flag (bitnet_w158a8_matmul_path tells which path a call
 * takes).  A wrong promise gives wrong results, not an error. */
#define BITNET_FLAG_WEIGHTS_EXPANDED 2u

/* Flag for bitnet_w158a8_matmul: run the table-lookup kernel instead, the
 * GPU form of the CPU kernels that "Microsoft BitNet 深度研究报告" describes
 * (技术原理 item 3, 查找表优化; the TL1/TL2 rows of its bitnet.cpp kernel
 * table): per token, every sum that two ternary weights (one 4-bit nibble of
 * the packed layout) can select from two activations is tabulated, and each
 * packed byte then costs two table reads.  Same results, bit for bit, as the
 * other kernels; kept as a measured comparison (it is slower here: every CTA
 * builds the whole table for its few rows).  1 <= M <= 8 tokens, any input
 * dtype, no workspace; shapes whose tables of one token do not fit in shared
 * memory (K above about 10000) return BITNET_ERR_UNSUPPORTED_SHAPE.  Not
 * accepted by bitnet_rms_norm_w158a8_matmul. */
#define BITNET_FLAG_TABLE_LOOKUP 4u

/* Flag for bitnet_w158a8_matmul: on the tensor-core path, let the tensor-core
 * kernel prepare its operands itself while its tiles run (extra warps
 * quantise the token rows and expand the weight rows, block by block; a
 * tile's loads wait for its blocks), instead of the separate quantiser
 * launch that precedes it by default.  Same results, bit for bit.  Kept as a
 * measured comparison: on B200 it is slower (a handful of preparing warps
 * per SM cannot stream the operands as fast as a dedicated launch over the
 * whole GPU, so the tiles wait).  Ignored on the other paths. */
#define BITNET_FLAG_PREP_IN_KERNEL 8u

/* ----------------------------------------------------------------------
 * Weight quantisation: absmean ternary codes, packed four per byte.
 * ("Microsoft BitNet 深度研究报告", 技术原理 item 2; 2B4T report write-up,
 * GPU kernel section.)
 *
 *   W        [N][K] fp32 or bf16 (w_dtype = BITNET_F32 | BITNET_BF16), finite.
 *   packed   [N][K/4] bytes, written (layout above).
 *   gamma    one fp32, written: mean |W| (fp64 sum in the fixed order above).
 *   workspace at least bitnet_quantize_weights_workspace_size(N, K) bytes of
 *            device scratch (fp64 row sums); contents on entry don't matter.
 * N must be positive (the mean of an empty matrix is undefined).
 * ---------------------------------------------------------------------- */
size_t bitnet_quantize_weights_workspace_size(int64_t N, int64_t K);

bitnet_status bitnet_quantize_weights(const void *W, bitnet_dtype w_dtype, int64_t N, int64_t K,
                                      uint8_t *packed, float *gamma, void *workspace,
                                      size_t workspace_bytes, bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * Per-token absmax activation quantisation.  (Model card of BitNet b1.58
 * 2B4T, 模型详情 -> 量化.)
 *
 *   X    [M][K] fp32 or bf16 (x_dtype), finite.
 *   xq   [M][K] int8, written: clamp(round_half_away(x * s_m), -127, 127).
 *   s    [M] fp32, written: 127 / max_k |x_mk| (fp32 division); 1 for an
 *        all-zero row.
 * K here may be any positive value up to 2^24 that keeps the rows 16-byte
 * aligned (K % 16 == 0 for int8 rows).
 * ---------------------------------------------------------------------- */
bitnet_status bitnet_quantize_act(const void *X, bitnet_dtype x_dtype, int64_t M, int64_t K,
                                  int8_t *xq, float *s, bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * The W1.58A8 BitLinear product y = Q(W) applied to x, with the rescale by
 * gamma / s and the optional ReLU^2.  (Research report 技术原理 items 2-3;
 * model card 模型详情; 2B4T report write-up, GPU kernel section.)
 *
 *   X        x_dtype = BITNET_F32 | BITNET_BF16: [M][K] raw activations; the
 *            per-token quantisation runs inside the call (bit-identical to
 *            bitnet_quantize_act) and `s` must be NULL.
 *            x_dtype = BITNET_I8: [M][K] xq from bitnet_quantize_act, and `s`
 *            its [M] scales.
 *   packed, gamma  from bitnet_quantize_weights for the [N][K] weight.
 *   epi      BITNET_EPI_NONE or BITNET_EPI_RELU2.
 *   Y        [M][N], y_dtype = BITNET_F32 | BITNET_BF16, or BITNET_I32 for
 *            the raw int32 accumulators (epi must then be NONE; the scale is
 *            not applied).  Y must not overlap X.
 *   workspace at least bitnet_w158a8_matmul_workspace_size(M, N, K, x_dtype)
 *            bytes (may be NULL when that is 0).  Contents on entry don't
 *            matter; the call may overwrite all of it.
 *   flags    0, or any of BITNET_FLAG_WEIGHTS_STATIC, BITNET_FLAG_WEIGHTS_EXPANDED,
 *            BITNET_FLAG_TABLE_LOOKUP, BITNET_FLAG_PREP_IN_KERNEL.
 * Up to 3 tokens (8 when K % 64 != 0) run one fused kernel and need no
 * workspace.  Otherwise fp32/bf16 input is first quantised into the
 * workspace by the activation quantiser (M*K bytes + 4*M, each rounded up to
 * 256); then 4..32 tokens run an int8 mma.sync kernel and larger M the
 * tcgen05 tensor-core kernel, which first expands the packed weights to int8
 * in the workspace (N*K more bytes, rounded up to 256; needed for int8 input
 * too), followed by the readiness counters of BITNET_FLAG_PREP_IN_KERNEL
 * (32 bytes per 128 tokens and per 256 output features, rounded up to 256).
 * The weights in HBM stay packed; the int8 copy is scratch of the call.
 * ---------------------------------------------------------------------- */
size_t bitnet_w158a8_matmul_workspace_size(int64_t M, int64_t N, int64_t K, bitnet_dtype x_dtype);

bitnet_status bitnet_w158a8_matmul(const void *X, bitnet_dtype x_dtype, const float *s,
                                   const uint8_t *packed, const float *gamma, int64_t M,
                                   int64_t N, int64_t K, bitnet_epilogue epi, void *Y,
                                   bitnet_dtype y_dtype, void *workspace, size_t workspace_bytes,
                                   uint32_t flags, bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * bitnet_w158a8_matmul from host memory to host memory, in one call: the
 * activations are copied from X_host to the caller's device buffer X_dev,
 * the product runs on the device (exactly bitnet_w158a8_matmul with X_dev,
 * same results), the output is copied from the caller's device buffer Y_dev
 * to Y_host, and the call returns once Y_host holds it (it synchronises
 * `stream`).  For a caller whose activations and results live on the host:
 * one C call per forward instead of a copy, a launch, a copy and a wait.
 *   X_host   [M][K] fp32 or bf16 (x_dtype), host memory; page-locked
 *            (cudaHostAlloc / cudaHostRegister) for the copy to be
 *            asynchronous, else it is staged by the driver.
 *   Y_host   [M][N] of y_dtype, host memory (page-locked likewise).
 *   X_dev, Y_dev  device buffers of those sizes, 16-byte aligned.
 * Everything else as bitnet_w158a8_matmul (int8 input is not accepted here:
 * its scales would need a copy of their own).  Errors: the argument checks
 * of bitnet_w158a8_matmul on X_dev and Y_dev, BITNET_ERR_INVALID_ARG for a
 * null host pointer, BITNET_ERR_CUDA when a copy or the synchronisation
 * fails.
 * ---------------------------------------------------------------------- */
bitnet_status bitnet_w158a8_matmul_host(const void *X_host, bitnet_dtype x_dtype, void *X_dev,
                                        const uint8_t *packed, const float *gamma, int64_t M,
                                        int64_t N, int64_t K, bitnet_epilogue epi, void *Y_dev,
                                        void *Y_host, bitnet_dtype y_dtype, void *workspace,
                                        size_t workspace_bytes, uint32_t flags,
                                        bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * The same host-to-host call, over fixed buffers, as a plan: for a
 * projection that runs again and again with the same buffers (a decode
 * loop), bitnet_host_plan_create checks the arguments once, records the
 * copy in, the product's kernels and the copy out as one CUDA graph and
 * uploads it to the device (it runs nothing; the upload is enqueued on
 * `stream`); bitnet_host_plan_run launches that graph on `stream` and
 * returns once Y_host holds the result (it synchronises `stream`), one
 * submission instead of three.  A large call on the tensor-core path is
 * recorded as a pipeline of token chunks over three streams, so that the
 * copies in and out overlap the product (same results).  The caller refills
 * X_host before a run and reads Y_host after it.
 *   Arguments as bitnet_w158a8_matmul_host, plus:
 *   X_host, Y_host  page-locked host memory (cudaHostAlloc /
 *            cudaHostRegister), else BITNET_ERR_INVALID_ARG.
 *   plan     receives the plan (NULL on error).  Caller-owned: free it with
 *            bitnet_host_plan_destroy.  Every buffer, the weights and the
 *            stream must stay valid and in place while the plan is used;
 *            run it on the device that was current at creation.
 * Errors: those of bitnet_w158a8_matmul_host; BITNET_ERR_INVALID_ARG for a
 * null `plan`, an empty call (M or N = 0) or pageable host memory;
 * BITNET_ERR_CUDA when capturing or instantiating the graph fails.
 * bitnet_host_plan_run: BITNET_ERR_INVALID_ARG for a null plan,
 * BITNET_ERR_CUDA when the launch or the synchronisation fails.
 * ---------------------------------------------------------------------- */
typedef struct bitnet_host_plan_s *bitnet_host_plan;

bitnet_status bitnet_host_plan_create(const void *X_host, bitnet_dtype x_dtype, void *X_dev,
                                      const uint8_t *packed, const float *gamma, int64_t M,
                                      int64_t N, int64_t K, bitnet_epilogue epi, void *Y_dev,
                                      void *Y_host, bitnet_dtype y_dtype, void *workspace,
                                      size_t workspace_bytes, uint32_t flags,
                                      bitnet_stream_t stream, bitnet_host_plan *plan);
bitnet_status bitnet_host_plan_run(bitnet_host_plan plan);
/* Frees the plan (NULL: nothing).  Not while a run of it is in flight. */
void bitnet_host_plan_destroy(bitnet_host_plan plan);

/* ----------------------------------------------------------------------
 * Which kernel path bitnet_w158a8_matmul takes for these sizes on the
 * current device (the paths are listed in the comment above).  Pure host
 * logic, except that the tensor-core path also needs the driver's
 * tensor-map encoder (cuTensorMapEncodeTiled), looked up once it is found:
 * when the driver does not provide it, calls of the tensor-core shape run
 * the much slower dp4a kernel instead, and this query returns
 * BITNET_PATH_GENERIC for them, so that a caller can tell.  Returns
 * BITNET_PATH_NONE for invalid sizes or dtypes, or an empty call.
 * ---------------------------------------------------------------------- */
typedef enum bitnet_path {
    BITNET_PATH_NONE = 0,
    BITNET_PATH_ROWS = 1,        /* 1..3 tokens (8 when K % 64 != 0): fused dp4a kernel        */
    BITNET_PATH_MMA_TOKENS = 2,  /* 4..32 tokens, fp32/bf16 input: quantiser + int8 mma.sync  */
    BITNET_PATH_MMA_WEIGHTS = 3, /* 9..32 tokens, int8 input: int8 mma.sync, weights as A     */
    BITNET_PATH_TENSOR_CORE = 4, /* more tokens: weight expansion + tcgen05 kernel             */
    BITNET_PATH_GENERIC = 5      /* K % 64 != 0, or no tensor-map encoder: dp4a fallback      */
} bitnet_path;

bitnet_path bitnet_w158a8_matmul_path(int64_t M, int64_t N, int64_t K, bitnet_dtype x_dtype);

/* ----------------------------------------------------------------------
 * Y = BitLinear(rms_norm(X)): the weightless RMS normalisation of
 * bitnet_rms_norm applied to each token of X, rounded to X's dtype, and then
 * exactly what bitnet_w158a8_matmul computes for that normalised input.  In
 * a decode stack it joins a layer's input normalisation (the model card's
 * "subln", 模型详情 -> 架构; no formula on the pages, this is the plain
 * stand-in) to the projection that reads it, saving one launch per layer.
 *   X        [M][K] F32 | BF16 (no int8: the normalisation needs the values).
 *   X_normed [M][K] of X's dtype, or NULL when M <= 8.  Receives the
 *            normalised input that was quantised (every link can be
 *            checked).  For M > 8 it is required: the normalisation then
 *            runs as its own kernel into it, and the matmul reads it.  Must
 *            not overlap X or Y.
 * Everything else as bitnet_w158a8_matmul.  Workspace: none when M <= 8 and
 * K % 16 == 0 fit the fused kernel, otherwise
 * bitnet_w158a8_matmul_workspace_size(M, N, K, x_dtype) bytes.  The
 * normalisation's fp32 sum may be ordered differently from bitnet_rms_norm's
 * (not part of the bit-exact contract).
 * ---------------------------------------------------------------------- */
bitnet_status bitnet_rms_norm_w158a8_matmul(const void *X, bitnet_dtype x_dtype, void *X_normed,
                                            const uint8_t *packed, const float *gamma,
                                            int64_t M, int64_t N, int64_t K,
                                            bitnet_epilogue epi, void *Y, bitnet_dtype y_dtype,
                                            void *workspace, size_t workspace_bytes,
                                            uint32_t flags, bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * bitnet_w158a8_matmul for callers that cannot allocate device memory.
 * (The pages on BitNet b1.58 have no counterpart of this entry point; it is
 * a service of this library.)
 *
 * Some callers cannot give the library a workspace: a plugin inside a host
 * framework that owns all device memory and hands out none, or a serving
 * loop that must never call cudaMalloc because cudaMalloc can block until
 * the whole device is idle.  This entry point takes the arguments of
 * bitnet_w158a8_matmul without the workspace and uses a scratch array built
 * into the library instead: BITNET_STATIC_SCRATCH_BYTES of device memory on
 * every GPU that loads the library, held until the process exits.  It
 * allocates nothing.
 *   - A call whose scratch need, bitnet_w158a8_matmul_workspace_size(M, N,
 *     K, x_dtype), is larger than BITNET_STATIC_SCRATCH_BYTES returns
 *     BITNET_ERR_WORKSPACE and launches nothing.  The need is 0 for up to
 *     3 tokens, about M*K bytes for 4..32 tokens, and about (M + N)*K bytes
 *     on the tensor-core path (M*K of them only for fp32/bf16 input).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, which keeps whatever the
 *     last call left in it; nothing in it needs to start at zero.
 *     BITNET_FLAG_WEIGHTS_EXPANDED refers to that array here: it holds only
 *     when the previous tensor-core-path call on the device used the same
 *     weights and kind of input.  Calls
 *     whose kernels overlap on the GPU (different streams or threads) race
 *     on the array: keep them on one stream or otherwise serialised.
 * ---------------------------------------------------------------------- */
#define BITNET_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

bitnet_status bitnet_w158a8_matmul_noalloc(const void *X, bitnet_dtype x_dtype, const float *s,
                                           const uint8_t *packed, const float *gamma, int64_t M,
                                           int64_t N, int64_t K, bitnet_epilogue epi, void *Y,
                                           bitnet_dtype y_dtype, uint32_t flags,
                                           bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * Weightless per-token RMS normalisation, y = x / sqrt(mean_k(x^2) + 1e-6),
 * fp32 arithmetic, bf16 or fp32 in and out.  Glue between chained
 * BitLinears: the model card names "subln" normalisation (模型详情 -> 架构)
 * without a formula, and this is the plain stand-in used by the decode
 * chain.  Not part of the bit-exact BitLinear contract.
 *   X [M][K] (x_dtype F32 | BF16), Y [M][K] (y_dtype F32 | BF16); may alias.
 * ---------------------------------------------------------------------- */
bitnet_status bitnet_rms_norm(const void *X, bitnet_dtype x_dtype, int64_t M, int64_t K, void *Y,
                              bitnet_dtype y_dtype, bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * A chain of M = 1 BitLinear projections in one launch.
 *
 * A decode step of BitNet b1.58 (the model card, 模型详情 -> 架构: a
 * Transformer whose linear layers are all BitLinear, ReLU^2 in the FFN,
 * a "subln" normalisation) runs its projections one after the other, each
 * on the previous one's output re-quantised per token (the technical
 * report's W1.58A8 BitLinear; 技术原理 of "Microsoft BitNet 深度研究报告").
 * This call runs such a chain for one token in a single cooperative launch
 * with one CTA per SM.  Every step computes exactly what
 * bitnet_w158a8_matmul computes for M = 1 with bf16 input and bf16 output:
 * same int8 activations and scale, same int32 accumulators, same epilogue.
 *
 * Step s reads the first K values of step s-1's output (of x0 for s = 0).
 * With BITNET_STEP_NORM_IN it first applies the weightless RMS
 * normalisation of bitnet_rms_norm to those K values, rounds them to bf16,
 * and quantises that; X_normed (optional) receives them, so every link can
 * be checked.  The normalisation's fp32 sum may be ordered differently from
 * bitnet_rms_norm's (not part of the bit-exact contract).
 *
 *   steps      host array of n_steps descriptors (1 <= n_steps <=
 *              BITNET_CHAIN_MAX_STEPS); read during the call only.
 *   x0         bf16 [steps[0].K], device, 16-byte aligned.  Must not
 *              overlap any output.
 *   y_norm     bf16 [steps[n-1].N] or NULL: the RMS normalisation of the
 *              last step's output (N % 16 == 0 and N <= 8192 when given).
 *   workspace  >= bitnet_decode_chain_workspace_size(steps, n_steps) bytes
 *              (256 + 4 * the sum of K over steps 1 .. n_steps-1, rounded
 *              up to 256), 16-byte aligned.  ZERO-FILLED before the first
 *              call; then passed unchanged to every later call of a chain
 *              (the library keeps a launch counter and a done counter in it,
 *              which only grow, and every link's values tagged with the
 *              launch they belong to).  After a call that reported
 *              BITNET_ERR_TIMEOUT, zero it again.
 *              Two chains must not run concurrently on one workspace.
 * Per step: packed [N][K/4] and gamma as from bitnet_quantize_weights
 * (packed 16-byte aligned); Y bf16 [N], 16-byte aligned; 1 <= N <= 2^22;
 * K % 64 == 0, 64 <= K <= 8192 and K <= the previous step's N.  Shapes whose
 * per-SM share of a step's packed rows does not fit twice in shared memory
 * return BITNET_ERR_UNSUPPORTED_SHAPE.
 * Every wait in the kernel is bounded; one that gives up records
 * BITNET_ERR_TIMEOUT (read it with bitnet_get_device_status).
 * ---------------------------------------------------------------------- */
#define BITNET_CHAIN_MAX_STEPS 256
#define BITNET_STEP_RELU2 1u   /* ReLU^2 epilogue */
#define BITNET_STEP_NORM_IN 2u /* RMS-normalise the input before quantising it */

typedef struct bitnet_chain_step {
  const uint8_t *packed; /* [N][K/4] packed ternary codes, device */
  const float *gamma;    /* device, 1 float */
  int64_t N;             /* output features */
  int64_t K;             /* input features */
  uint32_t flags;        /* BITNET_STEP_RELU2 | BITNET_STEP_NORM_IN */
  void *Y;               /* bf16 [N] output of this step, device */
  void *X_normed;        /* bf16 [K] normalised input (NORM_IN steps only), or NULL */
} bitnet_chain_step;

/* 0 if the descriptors are invalid. */
size_t bitnet_decode_chain_workspace_size(const bitnet_chain_step *steps, int n_steps);

bitnet_status bitnet_decode_chain(const bitnet_chain_step *steps, int n_steps, const void *x0,
                                  void *y_norm, void *workspace, size_t workspace_bytes,
                                  bitnet_stream_t stream);

/* ----------------------------------------------------------------------
 * Status and diagnostics.
 * ---------------------------------------------------------------------- */
/* Static English text for a status code (never NULL). */
const char *bitnet_status_string(bitnet_status status);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device: BITNET_OK, or the first error a kernel recorded
 * (BITNET_ERR_TIMEOUT after a bounded wait gave up). */
bitnet_status bitnet_get_device_status(bitnet_stream_t stream);

/* ABI version of this header: major * 10000 + minor * 100 + patch.  1.1:
 * the path query, the host-to-host call and its plans; the chain workspace
 * holds tagged link values (its size from bitnet_decode_chain_workspace_size). */
#define BITNET_VERSION 10100
int bitnet_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET158_H */
