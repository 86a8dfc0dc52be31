/*
 * fnl -- fused pre-norm linear layer for NVIDIA B200 (sm_100a).
 *
 * One call runs, on one GPU and in one pass over the weights:
 *   residual add  ->  LayerNorm or RMSNorm  ->  bf16 projection GEMM with fp32
 *   accumulation on the tcgen05 tensor cores  ->  a fused epilogue
 * with the normalised activations built in shared memory only (never written
 * to global memory). The three epilogues are the three fusions the pages
 * describe:
 *   fnl_add_norm_qkv        LayerNorm + QKV projection fused into one kernel,
 *                           q/k/v written directly (TensorRT-LLM 深度工程实践,
 *                           §2.3 跨算子融合, "LayerNorm + QKV Projection 融合"),
 *                           with the GQA head grouping of §2.2 图构建与算子映射;
 *   fnl_add_norm_swiglu     gate/up GEMM with SiLU(gate) * up done in registers
 *                           and one write-back (same page, §2.3 "GEMM + 激活融合
 *                           （SwiGLU）");
 *   fnl_add_bias_norm_gelu  Add -> Bias -> LayerNorm -> Linear -> GELU as one
 *                           kernel (trt-llm-deep-dive, "3. Layer Fusion" figure
 *                           and the 面试视角 answer on kernel fusion).
 * Residual + LayerNorm fusion and the RMSNorm op are named in TensorRT-LLM 简介
 * (the four-layer architecture: 模型定义层, 图优化层).
 *
 * Notation: M tokens (rows), K hidden size, N rows of W (= output columns
 * before the epilogue). All matrices are row-major bf16 (raw 16-bit patterns,
 * fnl_bf16), all pointers are DEVICE pointers of the handle's device, owned by
 * the caller and left untouched after the call returns (results are written
 * asynchronously on `stream`).
 *   x, residual   [M, K]
 *   residual_out  [M, K]   = bf16_rne(x + residual (+ bias_in)); must not
 *                          overlap x, residual or bias_in
 *   gamma         [K]      norm scale
 *   beta          [K]      LayerNorm shift, NULL = 0; must be NULL for RMSNorm
 *   W             [N, K]   projection weight, row n = output column n
 * Statistics use h = x + residual (+ bias_in) in fp32 before rounding:
 *   LayerNorm  mean = sum(h)/K, var = sum((h-mean)^2)/K, rstd = 1/sqrt(var+eps),
 *              a = (h - mean) * rstd * gamma + beta
 *   RMSNorm    rstd = 1/sqrt(sum(h^2)/K + eps), a = h * rstd * gamma
 * a is rounded to bf16 for the tensor cores (see fnl_precision); y = a W^T
 * accumulates in fp32.
 * mean_out / rstd_out (fp32 [M], nullable) receive the statistics; mean_out
 * must be NULL for RMSNorm.
 *
 * Requirements (checked on the host before any launch):
 *   - every bf16 pointer 16-byte aligned, fp32 outputs 4-byte aligned;
 *   - K, N (and D, I) multiples of 8; 1 <= K <= 32768; M >= 0 (M = 0 is a no-op);
 *     N <= 65535 * 128;
 *   - eps > 0 and finite (with eps = 0 a constant row would divide by zero);
 *   - outputs overlap neither each other nor any input;
 *   - the handle is used by one host thread / one stream at a time (its
 *     workspace is shared by its calls);
 *   - W is not written by the kernel enqueued on `stream` immediately before
 *     the call: the GEMM kernel is a programmatic dependent of that kernel and
 *     the large-M kernels fetch their first weight tiles before waiting for it
 *     (activations, statistics, workspace and outputs are touched only after
 *     the wait). Not checkable on the host; a weight produced by the previous
 *     kernel needs any other stream operation in between.
 * Calls are asynchronous: they enqueue one or two kernels on `stream` and
 * return. They never synchronise, except the first call whose shape needs more
 * workspace than the handle holds: that call synchronises `stream`, then
 * reallocates (create the handle with fnl_options.max_tokens / max_n to
 * reserve it up front, e.g. before capturing the calls in a CUDA graph).
 * Error behaviour: argument errors return FNL_ERR_* without touching the GPU;
 * launch errors return FNL_ERR_CUDA; fnl_last_error() gives the text. Device
 * waits inside the kernels are bounded: a wait that gives up records a code
 * that fnl_check() reports as FNL_ERR_DEVICE_STATUS.
 */
#ifndef FNL_H_
#define FNL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t fnl_bf16;                 /* raw bfloat16 bits */
typedef struct CUstream_st* fnl_stream;    /* same type as cudaStream_t; NULL = default stream */
typedef struct fnl_handle fnl_handle;      /* opaque: device, workspace, last error */

typedef enum {
  FNL_OK = 0,
  FNL_ERR_INVALID_ARG = 1,    /* NULL where required, bad size, bad enum, eps <= 0 or not finite */
  FNL_ERR_ALIGNMENT = 2,      /* pointer or leading dimension not aligned */
  FNL_ERR_ALIAS = 3,          /* an output overlaps an input or another output */
  FNL_ERR_UNSUPPORTED = 4,    /* shape outside what the kernels handle (K > 32768, ...) */
  FNL_ERR_CUDA = 5,           /* CUDA runtime/driver error (allocation, launch) */
  FNL_ERR_DEVICE_STATUS = 6   /* a kernel's bounded wait gave up (see fnl_check) */
} fnl_status;

typedef enum { FNL_NORM_LAYERNORM = 0, FNL_NORM_RMSNORM = 1 } fnl_norm;

typedef enum {
  FNL_PATH_AUTO = 0,          /* M <= 128: small-M split-K kernel (cluster form when it fits); else a tile kernel */
  FNL_PATH_TILE = 1,          /* force the large-M persistent kernel, 128 x 256 tiles */
  FNL_PATH_SPLITK = 2,        /* force the small-M split-K kernel, stream-K form (requires M <= 128) */
  FNL_PATH_TILE_WIDE = 3,     /* force the large-M persistent kernel, 128 x 512 tiles */
  FNL_PATH_SPLITK_CLUSTER = 4, /* force the small-M kernel's cluster form (M <= 128; FNL_ERR_UNSUPPORTED when
                                  the tiles cannot all run at once as clusters of 2..8 CTAs) */
  FNL_PATH_TILE_PAIR = 5,      /* force the large-M kernel on CTA pairs (tcgen05 cta_group::2), 256 x 512 tiles */
  FNL_PATH_TILE_PAIR_SPLIT = 6 /* the pair kernel's stream-K form: whole waves of tiles as above, the tiles left
                                  over dealt to all pairs as (tile, k-block) units; a fix-up kernel launched
                                  after it adds each split tile's partial sums in a fixed order and runs the
                                  epilogue (AUTO takes it when the last wave is less than about half full) */
} fnl_path;

/* How the normalised activation a is rounded for the bf16 tensor cores.
 * A single bf16 rounding of a perturbs each output by ~2^-9 |a| |W_n|; SwiGLU
 * multiplies that error by SiLU(gate) (up to ~5x at |gate| ~ 5), which exceeds
 * 1e-2 + 1e-2 |out| on Llama-sized MLPs. SPLIT writes a = hi + lo (both bf16)
 * and accumulates hi W^T + lo W^T in the same fp32 accumulator (twice the
 * tensor-core work, no extra memory traffic). */
typedef enum {
  FNL_PRECISION_DEFAULT = 0,  /* SPLIT for SwiGLU, SINGLE for QKV and GELU */
  FNL_PRECISION_SPLIT = 1,    /* hi + lo operand for every epilogue */
  FNL_PRECISION_SINGLE = 2    /* one bf16 rounding for every epilogue */
} fnl_precision;

typedef struct {
  int max_tokens;   /* reserve workspace for M up to this (0: grow on demand) */
  int max_n;        /* reserve workspace for N up to this (0: grow on demand) */
  int path;         /* fnl_path */
  int max_ctas;     /* cap on persistent CTAs (0: one per SM) -- for tests */
  int precision;    /* fnl_precision */
  long long wait_ns;      /* limit of the kernels' main-loop waits in ns (0: 4 s). A wait that
                             runs out aborts its CTA and records a code for fnl_check. */
  int debug_stall_calls;  /* fault injection for tests of the status path: the next this-many
                             calls withhold one weight copy in their first CTA, so a wait for it
                             runs out after wait_ns (their outputs are then incomplete and
                             fnl_check reports FNL_ERR_DEVICE_STATUS). 0 in normal use. */
  int tune;               /* 1: shape auto-tuning (TensorRT-LLM 深度工程实践, §2.4 内核自动调优:
                             candidate kernels run on the target GPU, the fastest is kept). With
                             path = FNL_PATH_AUTO, the first call of each shape (op, norm, N, K, and
                             M up to its 16-row padding at M <= 128 or its count of 128-row
                             blocks above) times every candidate plan on `stream` (the small-M
                             kernel's stream-K form and each cluster size whose clusters fit, the
                             128x256 and 128x512 tile kernels) and keeps the fastest for the
                             handle's later calls of that shape. Each candidate is timed on
                             launches that follow a write of twice the L2 size (weights cold in
                             L2, as in a model's layer loop). That first call allocates the
                             write buffer for its duration and synchronises `stream`; inside a
                             stream capture no tuning happens (the untuned plan is used and
                             nothing is cached). 0: the untuned plan. */
} fnl_options;

/* Create a handle on `device` (cudaSetDevice is called). opt may be NULL. */
fnl_status fnl_create(fnl_handle** out, int device, const fnl_options* opt);

/* Free the handle's workspace. Synchronises the device first. NULL is a no-op. */
fnl_status fnl_destroy(fnl_handle* h);

/* Static text of a status code. */
const char* fnl_status_string(fnl_status s);

/* Text of the handle's last error ("" if none). Valid until the next call. */
const char* fnl_last_error(const fnl_handle* h);

/* Text of the plan of the handle's last call ("" if none): the kernel, its
 * form and grid, and whether it was tuned. Valid until the next call. */
const char* fnl_last_plan(const fnl_handle* h);

/* Synchronise `stream`, read and clear the device status word. Returns
 * FNL_ERR_DEVICE_STATUS if a kernel since the last check gave up a wait
 * (device codes 1-7) or, in the debug build libfnl_debug.so (compiled with
 * FNL_DEBUG_CHECKS), skipped an output store that would have left its buffer
 * (device code 8); fnl_last_error() names the code. The outputs of the calls
 * since the last check are then not to be trusted. It
 * also resets the handle's split-K arrival counters (an aborted CTA leaves its
 * tiles' counters part-way), so later calls on the handle compute correctly. */
fnl_status fnl_check(fnl_handle* h, fnl_stream stream);

/* Residual add -> norm -> QKV projection -> head-major GQA split.
 * N = (Hq + 2*Hkv) * D; W rows [0, Hq*D) are the query heads, the next Hkv*D
 * the key heads, the last Hkv*D the value heads, D consecutive rows per head.
 * bias: nullable [N]. Outputs q [Hq, M, D], k [Hkv, M, D], v [Hkv, M, D]
 * with q[h, m, d] = y[m, h*D + d] (and likewise after the Q block).
 * Hq must be a multiple of Hkv. */
fnl_status fnl_add_norm_qkv(fnl_handle* h, fnl_stream stream,
                            const fnl_bf16* x, const fnl_bf16* residual, fnl_bf16* residual_out,
                            const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm, float eps,
                            const fnl_bf16* W, const fnl_bf16* bias,
                            int M, int K, int Hq, int Hkv, int D,
                            fnl_bf16* q, fnl_bf16* k, fnl_bf16* v,
                            float* mean_out, float* rstd_out);

/* Residual add -> norm -> gate/up projection -> SiLU(gate) * up.
 * W is [2I, K]: rows [0, I) gate, rows [I, 2I) up. bias: nullable [2I].
 * out [M, I] = SiLU(y[:, :I]) * y[:, I:], SiLU(g) = g / (1 + exp(-g)). */
fnl_status fnl_add_norm_swiglu(fnl_handle* h, fnl_stream stream,
                               const fnl_bf16* x, const fnl_bf16* residual, fnl_bf16* residual_out,
                               const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm, float eps,
                               const fnl_bf16* W, const fnl_bf16* bias,
                               int M, int K, int I,
                               fnl_bf16* out, float* mean_out, float* rstd_out);

/* Residual add + bias_in -> norm -> projection + bias_out -> GELU (tanh form).
 * bias_in: nullable [K], added to every row before the norm (and included in
 * residual_out). bias_out: nullable [N]. out [M, N] = GELU(y + bias_out),
 * GELU(z) = 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))). */
fnl_status fnl_add_bias_norm_gelu(fnl_handle* h, fnl_stream stream,
                                  const fnl_bf16* x, const fnl_bf16* residual, const fnl_bf16* bias_in,
                                  fnl_bf16* residual_out,
                                  const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm, float eps,
                                  const fnl_bf16* W, const fnl_bf16* bias_out,
                                  int M, int K, int N,
                                  fnl_bf16* out, float* mean_out, float* rstd_out);

/* Tensor-parallel all-reduce of the row-parallel projection's partial
 * outputs, the input of the next fused op (TensorRT-LLM 深度工程实践, §4.1
 * Tensor Parallelism: the output and down projections are split by rows, and
 * the ranks' partial results are summed before the next add + norm).
 * out[i] = bf16(sum over p = 0..P-1 of parts[p][i]), the sum in fp32 in rank
 * order (every rank that runs it gets the same bits), one round-to-nearest-even.
 * parts: host array of P device pointers, each n bf16 (16-byte aligned); on a
 * node they are the P ranks' buffers, the peers' mapped into this device's
 * address space (CUDA IPC / peer access), read with plain loads. The call does
 * not wait for the other ranks: order it after every partial is complete (a
 * host barrier or stream events). out: n bf16 (16-byte aligned), then passed as
 * x to fnl_add_norm_* with the residual stream as residual. 1 <= P <= 16.
 * Errors: FNL_ERR_INVALID_ARG (P out of range, n < 0, NULL), FNL_ERR_ALIGNMENT,
 * FNL_ERR_ALIAS (out overlaps a part). */
fnl_status fnl_tp_allreduce(fnl_handle* h, fnl_stream stream, const fnl_bf16* const* parts, int P, fnl_bf16* out,
                            long long n);

/* FP8 (W8A8) form of fnl_add_norm_qkv for decode-sized batches (M <= 128),
 * on the e4m3 tensor cores (tcgen05.mma kind::f8f6f4). TensorRT-LLM
 * 深度工程实践, §3.3 FP4/FP8 动态量化加速: W8A8_FP8 with activation ranges taken
 * from runtime statistics (no calibration). Per token m, the normalised row a
 * (as in fnl_add_norm_qkv, in fp32) is quantised with its own scale,
 * s_a[m] = max_k |a[m, k]| / 448, codes e4m3(a * 448 / max|a|) (round to
 * nearest even, saturating at +-448); W is given as e4m3 codes Wq [N, K] (one
 * byte each, K-contiguous) with one scale per row, w_scale [N] (fp32, see
 * fnl_quantize_weight_fp8), and
 *   y[m, n] = s_a[m] w_scale[n] sum_k code_a[m, k] Wq[n, k] (+ bias[n]),
 * accumulated in fp32, then the QKV split as in fnl_add_norm_qkv. Two kernels
 * per call: a pre-pass (one CTA per token: residual_out, the statistics and
 * the token's amax) and the small-M split-K kernel's FP8 form. Requirements as
 * for fnl_add_norm_qkv plus: K a multiple of 16, Wq 16-byte aligned, w_scale
 * 16-byte aligned; M > 128 or a forced tile path -> FNL_ERR_UNSUPPORTED. */
fnl_status fnl_add_norm_qkv_fp8(fnl_handle* h, fnl_stream stream,
                                const fnl_bf16* x, const fnl_bf16* residual, fnl_bf16* residual_out,
                                const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm, float eps,
                                const uint8_t* Wq, const float* w_scale, const fnl_bf16* bias,
                                int M, int K, int Hq, int Hkv, int D,
                                fnl_bf16* q, fnl_bf16* k, fnl_bf16* v,
                                float* mean_out, float* rstd_out);

/* FP8 (W8A8) forms of fnl_add_norm_swiglu and fnl_add_bias_norm_gelu (M <= 128),
 * with the same quantisation as fnl_add_norm_qkv_fp8: Wq [2I, K] (gate rows,
 * then up rows) or [N, K] e4m3 codes with one fp32 scale per row, the
 * normalised activations coded per token; the epilogue dequantises, then
 * applies SiLU(gate) * up, or GELU(y + bias_out). bias_in (GELU form) enters h
 * as in the bf16 op. Requirements and errors as for fnl_add_norm_qkv_fp8. */
fnl_status fnl_add_norm_swiglu_fp8(fnl_handle* h, fnl_stream stream,
                                   const fnl_bf16* x, const fnl_bf16* residual, fnl_bf16* residual_out,
                                   const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm, float eps,
                                   const uint8_t* Wq, const float* w_scale, const fnl_bf16* bias,
                                   int M, int K, int I,
                                   fnl_bf16* out, float* mean_out, float* rstd_out);
fnl_status fnl_add_bias_norm_gelu_fp8(fnl_handle* h, fnl_stream stream,
                                      const fnl_bf16* x, const fnl_bf16* residual, const fnl_bf16* bias_in,
                                      fnl_bf16* residual_out,
                                      const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm, float eps,
                                      const uint8_t* Wq, const float* w_scale, const fnl_bf16* bias_out,
                                      int M, int K, int N,
                                      fnl_bf16* out, float* mean_out, float* rstd_out);

/* Static per-output-channel FP8 quantisation of a bf16 weight W [N, K] for
 * the FP8 form: w_scale[n] = max_k |W[n, k]| / 448 (1 for an all-zero row) and
 * Wq[n, k] = e4m3(W[n, k] / w_scale[n]), both divisions IEEE fp32, round to
 * nearest even, saturating. One CTA per row on `stream`. K a multiple of 8;
 * W 16-byte, Wq 8-byte, w_scale 4-byte aligned; outputs must not overlap W. */
fnl_status fnl_quantize_weight_fp8(fnl_handle* h, fnl_stream stream, const fnl_bf16* W, int N, int K,
                                   uint8_t* Wq, float* w_scale);

/* Residual-stream projection: the layer's output projection (attention o_proj
 * or MLP down_proj) with the residual add fused into its epilogue, which closes
 * the layer's residual loop. These are the row-split projections of
 * TensorRT-LLM 深度工程实践, §4.1 Tensor Parallelism; the residual connection
 * they feed is the residual add that the graph-optimisation layer fuses
 * (TensorRT-LLM 简介, 图优化层).
 *   out[m, n] = bf16_rne(residual[m, n] + sum_k a[m, k] W[n, k] (+ bias[n]))
 * with the sum accumulated in fp32 on the tensor cores (a is bf16 already: no
 * norm, no operand rounding).
 *   a         [M, K]  the sublayer's activation (attention or SwiGLU output)
 *   W         [N, K]  projection weight, row n = output column n
 *   bias      [N]     nullable
 *   residual  [M, N]  the residual stream
 *   out       [M, N]  the updated residual stream; may be the same buffer as
 *                     residual (in-place update: each element is read, then
 *                     written, by one thread); any other overlap of out with
 *                     an input is FNL_ERR_ALIAS.
 * Requirements, asynchrony and errors as for the fused ops (K, N multiples of
 * 8, 16-byte aligned pointers, K <= 32768). M <= 128 runs the small-M split-K
 * kernel, larger M a tile kernel; fnl_options.path forces one as for the
 * fused ops. */
fnl_status fnl_linear_add_residual(fnl_handle* h, fnl_stream stream, const fnl_bf16* a, const fnl_bf16* W,
                                   const fnl_bf16* bias, const fnl_bf16* residual, fnl_bf16* out, int M, int K,
                                   int N);

/* Allocation-free variant of fnl_add_norm_qkv for decode-sized batches.
 * The pages have no counterpart to this entry point. It is for callers that
 * cannot call cudaMalloc on the call path: plugins inside an inference engine
 * that owns all device memory through its own static memory plan, and
 * latency-critical decode loops that must never pay cudaMalloc/cudaFree's
 * implicit device synchronisation. fnl_create allocates a workspace, so this
 * entry point takes no handle. It computes the same function as
 * fnl_add_norm_qkv (same arguments, same meaning, same layouts) on the calling
 * thread's current device, with the same kernel as FNL_PATH_SPLITK (the
 * small-M kernel's stream-K form over all SMs): its results are bitwise equal
 * to those of a handle created with path = FNL_PATH_SPLITK. A handle in
 * FNL_PATH_AUTO may pick the cluster form, whose fp32 partial sums are added
 * in another order, so the two agree within rounding but not always bitwise.
 * Scratch: a file-scope device array of 16 MiB inside the library, held by
 * every GPU that loads it until the process exits. Calls allocate nothing and
 * share that array: it keeps the last call's contents, and each call first
 * clears the split-K arrival counters on `stream`. Calls that overlap on one
 * GPU (several streams or host threads at once) race on the array and must be
 * serialised by the caller.
 * Limits: M <= 128 (FNL_ERR_UNSUPPORTED otherwise), and the split-K partial
 * sums must fit the array (about T * segments * roundup16(M) * 516 bytes with
 * T = ceil(N/128); e.g. N = 10240, M = 128 fits, N = 65536, M = 128 does not:
 * FNL_ERR_UNSUPPORTED). Other errors as for fnl_add_norm_qkv (status code only:
 * there is no handle to hold the text). A wait that runs out inside the kernel
 * is recorded in the array's status word, which fnl_check_static reads.
 * The first call on each device resolves the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture. */
fnl_status fnl_add_norm_qkv_static(fnl_stream stream,
                                   const fnl_bf16* x, const fnl_bf16* residual, fnl_bf16* residual_out,
                                   const fnl_bf16* gamma, const fnl_bf16* beta, fnl_norm norm, float eps,
                                   const fnl_bf16* W, const fnl_bf16* bias,
                                   int M, int K, int Hq, int Hkv, int D,
                                   fnl_bf16* q, fnl_bf16* k, fnl_bf16* v,
                                   float* mean_out, float* rstd_out);

/* Status check of fnl_add_norm_qkv_static on the current device: synchronise
 * `stream` (the stream of the static calls), read the status word of the
 * static array and clear it. Returns FNL_ERR_DEVICE_STATUS if a static call
 * since the last check gave up a bounded wait (its outputs are then not to be
 * trusted), FNL_OK otherwise. Allocates nothing. */
fnl_status fnl_check_static(fnl_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FNL_H_ */
