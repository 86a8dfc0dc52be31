"""Comparison of the CUDA path against the fp64 oracle (shared by the GPU tests,
the smoke check and the benchmark's verification step).

Tolerances:
  outputs       |gpu - ref| <= 1e-2 + 1e-2 |ref| per bf16 element
  residual_out  within 1 bf16 ulp of bf16_rne(x + r (+ bias_in)) (the fp32
                sum of three bf16 values can round once more than the exact sum)
  mean          |d| <= 1e-5 max(|mean|, sigma)   (mean ~ 0 makes a pure relative
                bound ill-posed; sigma = sqrt(var) is the row's scale)
  rstd          |d| <= 1e-5 rstd
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

OUT_ABS, OUT_REL, STAT_REL = 1e-2, 1e-2, 1e-5


def sample_rows(M: int, seq_lens=None, n_random: int = 256, seed: int = 0) -> np.ndarray:
    """First/last rows, rows around every 128-row tile boundary up to 1024,
    packed-sequence boundaries, and seeded random rows."""
    rows = {0, M - 1}
    for b in range(128, min(M, 1025), 128):
        rows.update((b - 1, b))
    if seq_lens is not None:
        s = 0
        for L in seq_lens:
            rows.update((s, s + L - 1))
            s += L
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, M, size=min(n_random, M)).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < M), dtype=np.int64)


FP8_TIE_RADIUS = 2.0 ** -20   # relative: about eight fp32 rounding steps
GELU_SLOPE_MAX = 1.13         # max |d/dz GELU_tanh(z)| (1.129 near z = 1.5)
SILU_SLOPE_MAX = 1.1          # max |d/dz SiLU(z)| (1.0998 near z = 2.4)


def fp8_layernorm_flip_bound(w, inputs: dict, rows) -> np.ndarray:
    """Per output element [rows, N]: the largest change that flipping FP8
    activation codes can make, over the codes whose fp32 decision value
    v = a * 448 / amax lies within FP8_TIE_RADIUS |v| of a rounding midpoint.
    With LayerNorm the code decision depends on the token's mean and rstd,
    which the GPU reduces in fp32 in its own order (they differ from the
    oracle's in the last bits, well inside the statistics tolerance), so such
    codes may round either way; every other code must match. RMSNorm decides
    its codes on h * gamma alone and gets no allowance."""
    f = lambda k: None if inputs.get(k) is None else inputs[k].double().numpy()  # noqa: E731
    h = oracle.residual_add(f("x")[rows], f("residual")[rows], f("bias_in"))
    _, mean, rstd = oracle.normalize(h, f("gamma"), f("beta"), w.norm, w.eps)
    h32 = oracle.fp8_h32(f("x")[rows], f("residual")[rows], f("bias_in"))
    a32 = oracle.fp8_normalised32(h32, mean, rstd, f("gamma"), f("beta"))
    amax = np.max(np.abs(a32), axis=1)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    inv = np.where(amax > 0, np.float32(448.0) / safe, np.float32(1.0)).astype(np.float32)
    sa = np.where(amax > 0, safe / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    v = (a32 * inv[:, None]).astype(np.float32).astype(np.float64)
    c = oracle.e4m3_round(v)
    dq = np.maximum(np.abs(oracle.e4m3_round(v * (1 - FP8_TIE_RADIUS)) - c),
                    np.abs(oracle.e4m3_round(v * (1 + FP8_TIE_RADIUS)) - c))
    Wq = f("W_fp8")
    return (dq @ np.abs(Wq).T) * sa.astype(np.float64)[:, None] * f("w_scale")[None, :], int(np.count_nonzero(dq))


def _f64(t) -> np.ndarray:
    return t.detach().float().cpu().double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)


def out_ratio(got, ref, extra=0.0) -> float:
    """max |got - ref| / (abs + rel |ref| + extra); <= 1 passes. `extra` is an
    exact per-element allowance (FP8 LayerNorm codes at rounding ties)."""
    g, r = _f64(got), np.asarray(ref, dtype=np.float64)
    if g.size == 0:
        return 0.0
    return float(np.max(np.abs(g - r) / (OUT_ABS + OUT_REL * np.abs(r) + extra)))


def _ordered_bits(t: torch.Tensor) -> np.ndarray:
    b = t.detach().contiguous().view(torch.int16).cpu().numpy().astype(np.int32) & 0xFFFF
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def residual_ulps(got: torch.Tensor, ref_f64: np.ndarray) -> int:
    ref = torch.from_numpy(np.ascontiguousarray(ref_f64)).to(torch.bfloat16)
    return int(np.max(np.abs(_ordered_bits(got) - _ordered_bits(ref)))) if ref.numel() else 0


def check(w, inputs: dict, got: dict, rows=None, chunk: int = 4096) -> dict:
    """Compare GPU results `got` (binding output dict, device tensors) with the
    oracle on `inputs` (CPU bf16 tensors). Outputs are compared on `rows` (all
    rows if None); residual_out and the statistics on all rows. Returns the
    error figures and raises AssertionError on a violation."""
    M = inputs["x"].shape[0]
    rows_idx = np.arange(M) if rows is None else np.asarray(rows)
    res = {"rows_checked": int(len(rows_idx))}

    ref = oracle.run(w, inputs, rows=rows_idx)
    rt = torch.from_numpy(rows_idx)
    if w.op == "residual":   # residual-stream projection: one output, no statistics
        g = got["out"].index_select(0, rt.to(got["out"].device))
        res["out_ratio"] = out_ratio(g, ref["out"])
        assert res["out_ratio"] <= 1.0, f"{w.name}: outputs off by {res['out_ratio']:.3f} x tolerance"
        return res
    bound = None
    if w.op.endswith("_fp8") and w.norm == "layernorm":
        bound, n_ties = fp8_layernorm_flip_bound(w, inputs, rows_idx)   # on y, before the epilogue
        res["fp8_tie_codes"] = n_ties
    if w.op in ("qkv", "qkv_fp8"):
        extra = {"q": 0.0, "k": 0.0, "v": 0.0}
        if bound is not None:
            extra = dict(zip(("q", "k", "v"), oracle.split_qkv_head_major(bound, w.Hq, w.Hkv, w.D)))
        r = 0.0
        for name in ("q", "k", "v"):
            g = got[name].index_select(1, rt.to(got[name].device))
            r = max(r, out_ratio(g, ref[name], extra[name]))
        res["out_ratio"] = r
    else:
        extra = 0.0
        if bound is not None and w.op == "gelu_fp8":
            extra = GELU_SLOPE_MAX * bound
        elif bound is not None and w.op == "swiglu_fp8":
            f = lambda k: None if inputs.get(k) is None else inputs[k].double().numpy()  # noqa: E731
            y = oracle.fp8_projection(f("x")[rows_idx], f("residual")[rows_idx], None, f("gamma"), f("beta"), w.norm,
                                      w.eps, f("W_fp8"), f("w_scale"), f("bias_out"))[0]
            gate, up, dg, du = y[:, :w.I], y[:, w.I:], bound[:, :w.I], bound[:, w.I:]
            extra = SILU_SLOPE_MAX * np.abs(up) * dg + np.abs(oracle.silu(gate)) * du + SILU_SLOPE_MAX * dg * du
        g = got["out"].index_select(0, rt.to(got["out"].device))
        res["out_ratio"] = out_ratio(g, ref["out"], extra)

    # residual_out and statistics on every row, in chunks
    ulps, mean_err, rstd_err = 0, 0.0, 0.0
    x64 = inputs["x"]
    for s in range(0, M, chunk):
        e = min(M, s + chunk)
        h = oracle.residual_add(inputs["x"][s:e].double().numpy(), inputs["residual"][s:e].double().numpy(),
                                None if inputs.get("bias_in") is None else inputs["bias_in"].double().numpy())
        ulps = max(ulps, residual_ulps(got["residual_out"][s:e], oracle.bf16_round(h)))
        _, mean, rstd = oracle.normalize(h, inputs["gamma"].double().numpy(),
                                         None if inputs.get("beta") is None else inputs["beta"].double().numpy(),
                                         w.norm, w.eps)
        if got.get("rstd") is not None:
            rg = _f64(got["rstd"][s:e])
            rstd_err = max(rstd_err, float(np.max(np.abs(rg - rstd) / rstd)))
        if got.get("mean") is not None and mean is not None:
            sigma = np.sqrt(np.maximum(rstd ** -2 - w.eps, 0.0))
            mg = _f64(got["mean"][s:e])
            mean_err = max(mean_err, float(np.max(np.abs(mg - mean) / np.maximum(np.abs(mean), sigma))))
    del x64
    res.update(residual_ulps=ulps, rstd_rel=rstd_err, mean_rel=mean_err)
    assert res["out_ratio"] <= 1.0, f"{w.name}: outputs off by {res['out_ratio']:.3f} x tolerance"
    assert ulps <= 1, f"{w.name}: residual_out off by {ulps} ulp"
    assert rstd_err <= STAT_REL, f"{w.name}: rstd relative error {rstd_err:.2e}"
    assert mean_err <= STAT_REL, f"{w.name}: mean error {mean_err:.2e}"
    return res


def fp8_inputs(w, inputs: dict) -> dict:
    """The workload's inputs plus its FP8 weights, quantised by the oracle:
    "W_fp8" (float8_e4m3fn codes) and "w_scale" (fp32 [N])."""
    codes, scale = oracle.quantize_weight_fp8(inputs["W"].double().numpy())
    out = dict(inputs)
    out["W_fp8"] = torch.from_numpy(codes).to(torch.float8_e4m3fn)
    out["w_scale"] = torch.from_numpy(np.asarray(scale, dtype=np.float32))
    return out
