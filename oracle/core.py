"""fp64 reference arithmetic of the fused pre-norm linear layer (test infrastructure).

Each function follows one step of the pages' description in their order; the
package docstring gives the citations and the readings R1..R8. No blocking, no
fusion, no reordering: numpy's float64 matmul is the only library primitive.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def bf16_round(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16, ties to even (reading R8).

    bfloat16 keeps 8 significant bits. With v = m * 2**e and 0.5 <= |m| < 1,
    m * 2**8 is an exact float64 and np.rint rounds half to even, so the result
    is the correctly rounded bf16 value (normal range; the workloads never
    leave it)."""
    v = _f64(v)
    m, e = np.frexp(v)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def residual_add(x, residual, bias_in=None) -> np.ndarray:
    """h = x + residual (+ bias_in broadcast over rows), exact in fp64 (R4, R5)."""
    h = _f64(x) + _f64(residual)
    if bias_in is not None:
        h = h + _f64(bias_in)[None, :]
    return h


def layernorm(h, gamma, beta, eps):
    """LayerNorm of each row of h, in the fused_layernorm_qkv order:
    mean, then variance about it (R1), then rsqrt(var + eps) (R2), then
    gamma * (h - mean) * rstd + beta. Returns (a, mean, rstd)."""
    h = _f64(h)
    K = h.shape[1]
    mean = h.sum(axis=1) / K
    d = h - mean[:, None]
    var = (d * d).sum(axis=1) / K
    rstd = 1.0 / np.sqrt(var + eps)
    g = _f64(gamma)[None, :]
    b = np.zeros_like(g) if beta is None else _f64(beta)[None, :]
    a = g * d * rstd[:, None] + b
    return a, mean, rstd


def rmsnorm(h, gamma, eps):
    """RMSNorm of each row (R3): a = h * rstd * gamma, rstd = (mean(h^2)+eps)^-1/2.
    Returns (a, rstd)."""
    h = _f64(h)
    K = h.shape[1]
    ms = (h * h).sum(axis=1) / K
    rstd = 1.0 / np.sqrt(ms + eps)
    a = h * rstd[:, None] * _f64(gamma)[None, :]
    return a, rstd


def normalize(h, gamma, beta, norm: str, eps: float):
    """Dispatch on the norm kind. Returns (a, mean or None, rstd)."""
    if norm == "layernorm":
        return layernorm(h, gamma, beta, eps)
    if norm == "rmsnorm":
        a, rstd = rmsnorm(h, gamma, eps)
        return a, None, rstd
    raise ValueError(f"unknown norm {norm!r}")


def projection(a, W, bias=None) -> np.ndarray:
    """y[m, n] = sum_k a[m, k] * W[n, k] (+ bias[n]); W is [N, K] (R7)."""
    y = _f64(a) @ _f64(W).T
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return y


def split_qkv_head_major(y, Hq, Hkv, D):
    """Columns [0, Hq*D) are Q, the next Hkv*D are K, the last Hkv*D are V;
    each is returned head-major [H, M, D] (R7)."""
    y = _f64(y)
    M, N = y.shape
    if N != (Hq + 2 * Hkv) * D:
        raise ValueError("N must equal (Hq + 2*Hkv) * D")
    q = y[:, : Hq * D].reshape(M, Hq, D).transpose(1, 0, 2)
    k = y[:, Hq * D:(Hq + Hkv) * D].reshape(M, Hkv, D).transpose(1, 0, 2)
    v = y[:, (Hq + Hkv) * D:].reshape(M, Hkv, D).transpose(1, 0, 2)
    return np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v)


def silu(z) -> np.ndarray:
    """SiLU(z) = z / (1 + exp(-z)) in fp64."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu(y, I) -> np.ndarray:
    """SiLU(gate) * up with gate = y[:, :I] and up = y[:, I:2I] (R7)."""
    y = _f64(y)
    return silu(y[:, :I]) * y[:, I:2 * I]


def gelu_tanh(z) -> np.ndarray:
    """GELU, tanh form (R6)."""
    z = _f64(z)
    return 0.5 * z * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (z + 0.044715 * z ** 3)))


def _stats(out: dict, mean, rstd) -> dict:
    if mean is not None:
        out["mean"] = mean
    out["rstd"] = rstd
    return out


def add_norm_qkv(x, residual, gamma, beta, norm, eps, W, bias, Hq, Hkv, D) -> dict:
    """Residual add -> norm -> QKV projection -> head-major Q/K/V split."""
    h = residual_add(x, residual)
    a, mean, rstd = normalize(h, gamma, beta, norm, eps)
    y = projection(a, W, bias)
    q, k, v = split_qkv_head_major(y, Hq, Hkv, D)
    return _stats({"residual_out": bf16_round(h), "q": q, "k": k, "v": v}, mean, rstd)


def add_norm_swiglu(x, residual, gamma, beta, norm, eps, W, bias, I) -> dict:
    """Residual add -> norm -> gate/up projection -> SiLU(gate) * up."""
    h = residual_add(x, residual)
    a, mean, rstd = normalize(h, gamma, beta, norm, eps)
    y = projection(a, W, bias)
    return _stats({"residual_out": bf16_round(h), "out": swiglu(y, I)}, mean, rstd)


def add_bias_norm_gelu(x, residual, bias_in, gamma, beta, norm, eps, W, bias_out) -> dict:
    """Residual add + bias_in -> norm -> projection + bias_out -> GELU_tanh."""
    h = residual_add(x, residual, bias_in)
    a, mean, rstd = normalize(h, gamma, beta, norm, eps)
    z = projection(a, W, bias_out)
    return _stats({"residual_out": bf16_round(h), "out": gelu_tanh(z)}, mean, rstd)


def tp_allreduce(parts) -> np.ndarray:
    """Tensor-parallel all-reduce of the row-parallel projection's partial
    outputs (TensorRT-LLM 深度工程实践, §4.1 Tensor Parallelism: the output and
    down projections are split by rows, and each rank's partial result is
    summed across ranks before the next add and norm). Reading R13: the P
    ranks' bf16 partials summed exactly, then rounded once to bf16, because the
    reduced tensor is bf16 like its inputs."""
    return bf16_round(np.sum(np.stack([_f64(v) for v in parts]), axis=0))


def add_norm_qkv_tp(parts, residual, gamma, beta, norm, eps, W, bias, Hq, Hkv, D) -> dict:
    """The fused QKV op fed by the all-reduce: x = tp_allreduce(parts), then
    add_norm_qkv(x, residual, ...) (reading R13)."""
    return add_norm_qkv(tp_allreduce(parts), residual, gamma, beta, norm, eps, W, bias, Hq, Hkv, D)


def linear_add_residual(a, W, bias, residual) -> dict:
    """Residual-stream projection (o_proj / down_proj) with the residual add
    fused after it: out = residual + a W^T (+ bias), in fp64 (reading R9).
    a [M, K] is the sublayer's activation (attention output or SwiGLU output),
    W [N, K], residual [M, N] the residual stream."""
    return {"out": _f64(residual) + projection(a, W, bias)}


# ---------------------------------------------------------------- FP8 (W8A8)
E4M3_MAX = 448.0   # largest finite value of the e4m3 format (1 sign, 4 exponent bits with bias 7, 3 mantissa bits)


def e4m3_round(v) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to even, saturating at +-448
    (reading R11). Normal binades [2^e, 2^(e+1)) for e >= -6 have 8 steps of
    2^(e-3); below 2^-6 the subnormal step is 2^-9."""
    v = _f64(v)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)                       # subnormals share the 2^-9 step of e = -6
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.rint(a / quantum) * quantum            # np.rint: halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(a > 0, np.sign(v) * q, 0.0)


def _f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32)


def fp8_row_scale_and_codes(v32):
    """Per-row symmetric e4m3 quantisation of a weight row (R11), every step
    in fp32: amax = max |v| of the row, s = amax / 448 (1 for an all-zero
    row), code = e4m3(v / s). Returns (codes as fp64 values, s as fp32)."""
    v32 = _f32(v32)
    amax = np.max(np.abs(v32), axis=1)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = e4m3_round((v32 / s[:, None]).astype(np.float32))
    return q, s


def fp8_activation_codes(a32):
    """Per-token dynamic quantisation of the normalised activation (R11), the
    decision in fp32 as the kernel takes it: amax = max_k |a|, code =
    e4m3(a * (448 / amax)), dequantisation scale s_a = amax / 448 (448 / amax
    and s_a are 1 for an all-zero row). Returns (codes as fp64 values, s_a)."""
    a32 = _f32(a32)
    amax = np.max(np.abs(a32), axis=1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    inv = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
    s = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = e4m3_round((a32 * inv[:, None]).astype(np.float32))
    return q, s


def quantize_weight_fp8(W):
    """Static per-output-channel FP8 weights: row n of W [N, K] (bf16 values)
    gets scale s_w[n] = max_k |W[n, k]| / 448 and codes e4m3(W / s_w[n])."""
    return fp8_row_scale_and_codes(_f64(W).astype(np.float32))


def fp8_linear(a32, Wq, w_scale, bias=None):
    """Dynamic per-token FP8 activations against per-channel FP8 weights
    (W8A8): a [M, K] (fp32) is quantised row by row (fp8_activation_codes),
    then y = s_a[m] s_w[n] sum_k code_a[m, k] code_w[n, k] (+ bias[n]) in fp64."""
    qa, sa = fp8_activation_codes(a32)
    y = (qa @ _f64(Wq).T) * _f64(sa)[:, None] * _f64(w_scale)[None, :]
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return y


def fp8_h32(x, residual, bias_in=None) -> np.ndarray:
    """h = x + residual (+ bias_in) as the FP8 path forms it for its code
    decisions (R11): fp32 sums, the bias added to the rounded x + residual."""
    h = (_f32(x) + _f32(residual)).astype(np.float32)
    if bias_in is not None:
        h = (h + _f32(bias_in)[None, :]).astype(np.float32)
    return h


def fp8_normalised32(h32, mean, rstd, gamma, beta):
    """The normalised activation in fp32, as the FP8 path forms it before the
    code decision (R11): the statistics rounded to fp32,
    t = fp32(fp32(h - mean) * rstd), a = fp32(t * gamma + beta) with one
    rounding (mean 0 and beta 0 for RMSNorm)."""
    h32 = _f32(h32)
    m32 = _f32(np.zeros(h32.shape[0]) if mean is None else mean)
    r32 = _f32(rstd)
    t = ((h32 - m32[:, None]).astype(np.float32) * r32[:, None]).astype(np.float32)
    b = np.zeros(h32.shape[1]) if beta is None else _f64(beta)
    return (_f64(t) * _f64(gamma)[None, :] + b[None, :]).astype(np.float32)


def fp8_projection(x, residual, bias_in, gamma, beta, norm, eps, Wq, w_scale, bias):
    """Residual add -> norm statistics -> per-token FP8 codes -> W8A8 projection
    (+ bias), shared by the three FP8 ops. RMSNorm's 1/rms is a positive
    per-token factor, so its codes are decided on h * gamma (the same codes as
    on the normalised row, but for fp32 rounding) and rstd multiplies the
    token's scale (reading R11). Returns (y, h, mean, rstd)."""
    h = residual_add(x, residual, bias_in)
    _, mean, rstd = normalize(h, gamma, beta, norm, eps)
    h32 = fp8_h32(x, residual, bias_in)
    if norm == "rmsnorm":
        a32 = (h32 * _f32(gamma)[None, :]).astype(np.float32)
        qa, sa = fp8_activation_codes(a32)
        y = (qa @ _f64(Wq).T) * (_f64(sa) * rstd)[:, None] * _f64(w_scale)[None, :]
        if bias is not None:
            y = y + _f64(bias)[None, :]
    else:
        y = fp8_linear(fp8_normalised32(h32, mean, rstd, gamma, beta), Wq, w_scale, bias)
    return y, h, mean, rstd


def add_norm_qkv_fp8(x, residual, gamma, beta, norm, eps, Wq, w_scale, bias, Hq, Hkv, D) -> dict:
    """The fused QKV op on FP8 tensor cores, then the head-major Q/K/V split."""
    y, h, mean, rstd = fp8_projection(x, residual, None, gamma, beta, norm, eps, Wq, w_scale, bias)
    q, k, v = split_qkv_head_major(y, Hq, Hkv, D)
    return _stats({"residual_out": bf16_round(h), "q": q, "k": k, "v": v}, mean, rstd)


def add_norm_swiglu_fp8(x, residual, gamma, beta, norm, eps, Wq, w_scale, bias, I) -> dict:
    """The fused gate/up op on FP8 tensor cores (W = [gate; up] rows, one
    scale per row), then SiLU(gate) * up."""
    y, h, mean, rstd = fp8_projection(x, residual, None, gamma, beta, norm, eps, Wq, w_scale, bias)
    return _stats({"residual_out": bf16_round(h), "out": swiglu(y, I)}, mean, rstd)


def add_bias_norm_gelu_fp8(x, residual, bias_in, gamma, beta, norm, eps, Wq, w_scale, bias_out) -> dict:
    """The fused Add + Bias + norm -> Linear + GELU op on FP8 tensor cores."""
    y, h, mean, rstd = fp8_projection(x, residual, bias_in, gamma, beta, norm, eps, Wq, w_scale, bias_out)
    return _stats({"residual_out": bf16_round(h), "out": gelu_tanh(y)}, mean, rstd)


def run(w, inputs: dict, rows=None) -> dict:
    """Evaluate workload ``w`` (a synthetic.Workload) on ``inputs`` (tensors or
    arrays, bf16 values), optionally on a subset of rows (the op is row-wise).
    For the residual-stream projection, "x" holds the activation a and
    "residual" the [M, N] residual stream."""
    def g(name):
        t = inputs.get(name)
        if t is None:
            return None
        if hasattr(t, "detach"):
            t = t.detach().cpu().double().numpy()
        return _f64(t)

    x, r = g("x"), g("residual")
    if rows is not None:
        x, r = x[rows], r[rows]
    if w.op == "residual":
        return linear_add_residual(x, g("W"), g("bias_out"), r)
    if w.op == "qkv_fp8":   # "W_fp8" / "w_scale": the FP8 weights (codes as values) and their scales
        return add_norm_qkv_fp8(x, r, g("gamma"), g("beta"), w.norm, w.eps, g("W_fp8"), g("w_scale"),
                                g("bias_out"), w.Hq, w.Hkv, w.D)
    if w.op == "swiglu_fp8":
        return add_norm_swiglu_fp8(x, r, g("gamma"), g("beta"), w.norm, w.eps, g("W_fp8"), g("w_scale"),
                                   g("bias_out"), w.I)
    if w.op == "gelu_fp8":
        return add_bias_norm_gelu_fp8(x, r, g("bias_in"), g("gamma"), g("beta"), w.norm, w.eps, g("W_fp8"),
                                      g("w_scale"), g("bias_out"))
    if w.op == "qkv":
        return add_norm_qkv(x, r, g("gamma"), g("beta"), w.norm, w.eps, g("W"),
                            g("bias_out"), w.Hq, w.Hkv, w.D)
    if w.op == "swiglu":
        return add_norm_swiglu(x, r, g("gamma"), g("beta"), w.norm, w.eps, g("W"),
                               g("bias_out"), w.I)
    return add_bias_norm_gelu(x, r, g("bias_in"), g("gamma"), g("beta"), w.norm, w.eps,
                              g("W"), g("bias_out"))
