"""CPU oracle for the fused pre-norm linear layer: plain, slow, fp64.

TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the
benchmark's CPU-baseline / reference leg may import or call this package; the
CUDA library and its Python binding never do, and this package imports neither
of them. It shares no code, constant or helper with the CUDA path. Inputs come
from the seeded generator (``synthetic.py``) as bf16 values widened to float64.

What is computed, and where the pages say so:

* residual add -- the graph-optimisation layer fuses the residual add with the
  LayerNorm that follows it (TensorRT-LLM 简介, the four-layer architecture,
  图优化层); the GPT-style
  chain Input -> Add -> Bias -> LayerNorm -> GELU is the Layer Fusion figure of
  "TRT-LLM 编译优化管线 / 构建阶段详解 / 3. Layer Fusion" (trt-llm-deep-dive).
* LayerNorm statistics in the order mean -> variance -> rsqrt(var + eps) ->
  gamma * (x - mean) * rsqrt + beta, then a dot with the QKV weight written to
  separate q/k/v outputs: the fused_layernorm_qkv kernel of TensorRT-LLM 深度工程实践,
  §2.3 跨算子融合 ("LayerNorm + QKV Projection 融合").
* RMSNorm is named as a model-definition op (TensorRT-LLM 简介, 模型定义层); the
  pages give no formula, so the textbook one is used (reading R3 below).
* SwiGLU: y = SiLU(x @ gate) * (x @ up), TensorRT-LLM 深度工程实践, §2.3
  ("GEMM + 激活融合（SwiGLU）").
* LayerNorm + Linear + GELU into one kernel: trt-llm-deep-dive, the 面试视角 answer
  on kernel fusion beyond the standard patterns.
* QKV projection + reshape + GQA grouping: TensorRT-LLM 深度工程实践, §2.2 图构建与
  算子映射; GQA/MQA head counts come from the model config (§2.1).
* FP8 W8A8 quantisation of the fused op: TensorRT-LLM 深度工程实践, §3.3 FP4/FP8
  动态量化加速 (W8A8_FP8, dynamic activation ranges, no calibration for FP8).
* Residual-stream projection: the attention output projection and the MLP's
  down projection are the row-split GEMMs of TensorRT-LLM 深度工程实践, §4.1
  Tensor Parallelism; the residual connection they feed is the residual add
  that the graph-optimisation layer fuses (TensorRT-LLM 简介, 图优化层).

Readings taken where the pages are silent:
  R1 variance is the population variance (divide by K), two passes about the mean.
  R2 eps sits inside the square root: rstd = (var + eps)^(-1/2).
  R3 RMSNorm: a = h * gamma / sqrt(mean(h^2) + eps); no mean, no beta.
  R4 statistics use the unrounded h = x + residual (+ bias_in), exact in fp64.
  R5 bias_in (GELU variant) is a [K] vector added before the norm; bias_out is
     added before GELU: out = GELU_tanh(y + bias_out).
  R6 GELU is the tanh form 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).
  R7 W is [N, K] like a linear layer's weight; QKV columns are ordered
     [Q heads | K heads | V heads], D contiguous columns per head, stored
     head-major Q[h, m, d] = y[m, h*D + d]. SwiGLU's W stacks gate rows [0, I)
     over up rows [I, 2I).
  R8 residual_out is h rounded once to bf16, round-to-nearest-even.
  R11 FP8 W8A8 (the pages name the W8A8_FP8 scheme and say its activation
     ranges adapt online from runtime statistics, no calibration; they give
     no granularity): e4m3 codes (round to nearest, ties to even, saturating at
     +-448); weights get one static scale per output channel, s_w[n] =
     max_k |W[n, k]| / 448; activations one dynamic scale per token, taken on
     the normalised row, s_a[m] = max_k |a[m, k]| / 448; y = s_a s_w sum of
     code products. Every decision that picks a code is taken in fp32, the
     kernel's precision, with the kernel's formula: weights e4m3(w / s_w);
     activations formed in fp32 from the statistics, t = (h - mean) rstd,
     a = t gamma + beta, then e4m3(a * (448 / amax)). RMSNorm's 1/rms is a
     positive per-token factor: its codes are decided on h * gamma and rstd
     joins the token's scale. The statistics, the sums of code products and
     the dequantisation are fp64.
  R9 the residual-stream projection adds the residual after the projection and
     its bias: out = residual + a W^T + bias, with residual [M, N] (N = the
     hidden size the projection returns to); the stored result is out rounded
     once to bf16. The pages name the row-split output and down projections
     but give no formula for the residual connection; this is the pre-norm
     transformer's plain reading.

  R13 tensor parallelism (the pages split the output and down projections by
     rows and all-reduce their partial outputs; they give no precision): the
     P ranks' bf16 partial activations are summed exactly and rounded once to
     bf16, and that sum is the x of the next fused add + norm + projection.

Parity pins live in tests/test_oracle_pins.py; every function here is pinned.
"""
from .core import (  # noqa: F401
    bf16_round,
    residual_add,
    layernorm,
    rmsnorm,
    normalize,
    projection,
    split_qkv_head_major,
    silu,
    swiglu,
    gelu_tanh,
    add_norm_qkv,
    add_norm_swiglu,
    add_bias_norm_gelu,
    linear_add_residual,
    tp_allreduce,
    add_norm_qkv_tp,
    E4M3_MAX,
    e4m3_round,
    fp8_row_scale_and_codes,
    fp8_activation_codes,
    fp8_h32,
    fp8_normalised32,
    quantize_weight_fp8,
    fp8_linear,
    fp8_projection,
    add_norm_qkv_fp8,
    add_norm_swiglu_fp8,
    add_bias_norm_gelu_fp8,
    run,
)
