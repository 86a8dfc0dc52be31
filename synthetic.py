"""Seeded synthetic inputs for the fused pre-norm linear layer.

This module holds the workloads (shapes) and the input distributions, nothing of
the method's arithmetic: it draws tensors and hands them out. The oracle and the
CUDA path both receive exactly these tensors; neither imports the other.

Distributions (per workload description of the fused LayerNorm+QKV / SwiGLU /
Add+Bias+LayerNorm->Linear+GELU layer):
  x, residual, bias_in ~ N(0, 1)
  gamma = 1 + 0.1 * N(0, 1);  beta = 0.1 * N(0, 1)
  W ~ N(0, 1/K)  (std 1/sqrt(K), so each output is O(1))
  bias_out ~ 0.02 * N(0, 1)
Every draw is fp32 from a CPU torch.Generator seeded once per workload, rounded
to bf16 (round to nearest even). Draw order: ragged lengths (packed workload
only), x, residual, bias_in, gamma, beta, W, bias_out; draws a workload does not
use are skipped. The residual-stream projection draws its activation a (kept
under the key "x") ~ N(0, 1) [M, K], the residual stream ~ N(0, 1) [M, N], W and
bias_out, in that order.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

LAYERNORM = "layernorm"
RMSNORM = "rmsnorm"

QKV = "qkv"
SWIGLU = "swiglu"
GELU = "gelu"
RESIDUAL = "residual"   # residual-stream projection: out = residual + a W^T (+ bias)
QKV_FP8 = "qkv_fp8"     # the QKV op with FP8 (e4m3) weights and activations; W is drawn in bf16
SWIGLU_FP8 = "swiglu_fp8"
GELU_FP8 = "gelu_fp8"
FP8_OPS = (QKV_FP8, SWIGLU_FP8, GELU_FP8)
NONORM = "none"


@dataclasses.dataclass(frozen=True)
class Workload:
    """One shape of the fused op."""

    name: str
    op: str               # QKV | SWIGLU | GELU
    norm: str             # LAYERNORM | RMSNORM
    M: int                # tokens (rows)
    K: int                # hidden size
    N: int                # rows of W (total output columns before the epilogue)
    Hq: int = 0           # QKV only
    Hkv: int = 0
    D: int = 0
    I: int = 0            # SwiGLU only: intermediate size, N = 2*I
    eps: float = 1e-5
    has_bias_in: bool = False
    has_bias_out: bool = False
    seq_lens: Optional[tuple] = None   # packed ragged batch, M = sum(seq_lens)
    x_loc: float = 0.0    # mean of x (edge cases with |mean| >> sigma); 0 for the workloads

    @property
    def n_out(self) -> int:
        """Columns of the stored output (I for SwiGLU, N otherwise)."""
        return self.I if self.op in (SWIGLU, SWIGLU_FP8) else self.N

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def algorithmic_bytes(self) -> float:
        """Bytes the fused op must move at least once: read x and residual,
        write residual_out, read W once, write the outputs, read the vectors.
        Residual-stream projection: read a [M, K], the residual [M, N] and W
        once, write out [M, N], read the bias."""
        M, K, N = self.M, self.K, self.N
        if self.op == RESIDUAL:
            return float(M * K * 2 + 2 * M * N * 2 + N * K * 2 + (N * 2 if self.has_bias_out else 0))
        if self.op in FP8_OPS:   # one byte per weight plus a 4-byte scale per row
            b = 2 * M * K * 2 + M * K * 2 + N * K + N * 4 + M * self.n_out * 2
            b += K * 2 * (2 if self.norm == LAYERNORM else 1) + (K * 2 if self.has_bias_in else 0)
            return float(b + (N * 2 if self.has_bias_out else 0))
        b = 2 * M * K * 2 + M * K * 2 + N * K * 2 + M * self.n_out * 2
        b += K * 2 * (2 if self.norm == LAYERNORM else 1)
        if self.has_bias_in:
            b += K * 2
        if self.has_bias_out:
            b += N * 2
        return float(b)


def qkv(name, M, K, Hq, Hkv, D, norm, **kw) -> Workload:
    return Workload(name, QKV, norm, M, K, (Hq + 2 * Hkv) * D, Hq=Hq, Hkv=Hkv, D=D, **kw)


def ragged_lengths(n_seqs: int = 64, max_len: int = 2048, seed: int = 0) -> tuple:
    """Sequence lengths uniform in [1, max_len], the first draw of the seeded
    generator (the packed workload's draw order starts with them)."""
    g = torch.Generator().manual_seed(seed)
    return tuple(int(v) for v in torch.randint(1, max_len + 1, (n_seqs,), generator=g))


def workloads() -> dict:
    """The five workloads, by name."""
    w = {}
    w["c1_tiny_ln_qkv"] = qkv("c1_tiny_ln_qkv", 8, 256, 4, 2, 64, LAYERNORM)
    w["c2_decode_rms_qkv"] = qkv("c2_decode_rms_qkv", 32, 4096, 32, 8, 128, RMSNORM)
    w["c3_prefill_rms_swiglu"] = Workload(
        "c3_prefill_rms_swiglu", SWIGLU, RMSNORM, 16384, 4096, 2 * 14336, I=14336)
    w["c4_gpt_ln_gelu"] = Workload(
        "c4_gpt_ln_gelu", GELU, LAYERNORM, 4096, 4096, 16384,
        has_bias_in=True, has_bias_out=True)
    for m in (1, 8, 32, 256, 2048, 8192):
        nm = f"c5_70b_rms_qkv_m{m}"
        w[nm] = qkv(nm, m, 8192, 64, 8, 128, RMSNORM)
    lens = ragged_lengths()
    w["c5_70b_rms_qkv_ragged"] = qkv(
        "c5_70b_rms_qkv_ragged", sum(lens), 8192, 64, 8, 128, RMSNORM, seq_lens=lens)
    w.update(residual_workloads())
    w.update(fp8_workloads())
    return w


def fp8_workloads() -> dict:
    """Decode shapes (32 tokens) with FP8 (e4m3) weights and activations: the
    QKV projections of Llama-3-8B (K=4096, N=6144) and Llama-2-70B (K=8192,
    N=10240) after RMSNorm, the Llama-3-8B gate/up projection (K=4096,
    I=14336) after RMSNorm, and a GPT-style up-projection (K=4096, N=16384)
    after LayerNorm with both biases. The bf16 W is drawn as for the bf16 op;
    its FP8 codes and scales are derived from it by the quantiser under test
    (or the oracle's)."""
    return {
        "c2_decode_rms_qkv_fp8": Workload("c2_decode_rms_qkv_fp8", QKV_FP8, RMSNORM, 32, 4096, 6144,
                                          Hq=32, Hkv=8, D=128),
        "c5_70b_rms_qkv_m32_fp8": Workload("c5_70b_rms_qkv_m32_fp8", QKV_FP8, RMSNORM, 32, 8192, 10240,
                                           Hq=64, Hkv=8, D=128),
        "llama3_8b_mlp_decode_swiglu_fp8": Workload("llama3_8b_mlp_decode_swiglu_fp8", SWIGLU_FP8, RMSNORM,
                                                    32, 4096, 2 * 14336, I=14336),
        "gpt_mlp_decode_ln_gelu_fp8": Workload("gpt_mlp_decode_ln_gelu_fp8", GELU_FP8, LAYERNORM, 32, 4096,
                                               16384, has_bias_in=True, has_bias_out=True),
    }


def residual_workloads() -> dict:
    """The residual-stream projections that close a Llama-3-8B layer's residual
    loop: the attention output projection at decode (M=32, K=N=4096) and the
    MLP down projection at prefill (M=16384 tokens, K=14336, N=4096)."""
    return {
        "llama3_8b_o_proj_decode": Workload("llama3_8b_o_proj_decode", RESIDUAL, NONORM, 32, 4096, 4096),
        "llama3_8b_down_proj_prefill": Workload("llama3_8b_down_proj_prefill", RESIDUAL, NONORM, 16384,
                                                14336, 4096),
    }


def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


def make_inputs(w: Workload, seed: int = 0, rows: Optional[int] = None) -> dict:
    """Draw the inputs of workload ``w`` (CPU bf16 tensors).

    ``rows`` overrides M (used to build reduced-size cases with the same
    distributions). The packed workload's lengths are drawn first so that the
    rest of its draws follow the documented order.
    """
    g = torch.Generator().manual_seed(seed)
    M = w.M if rows is None else rows
    K, N = w.K, w.N
    if w.seq_lens is not None:
        torch.randint(1, 2049, (len(w.seq_lens),), generator=g)   # keeps draw order
    out = {}
    if w.op == RESIDUAL:   # a [M, K], residual [M, N], W [N, K], bias [N]
        out["x"] = _bf16(torch.randn(M, K, generator=g) + w.x_loc)
        out["residual"] = _bf16(torch.randn(M, N, generator=g))
        out["W"] = _bf16(torch.randn(N, K, generator=g) / (K ** 0.5))
        if w.has_bias_out:
            out["bias_out"] = _bf16(0.02 * torch.randn(N, generator=g))
        return out
    out["x"] = _bf16(torch.randn(M, K, generator=g) + w.x_loc)
    out["residual"] = _bf16(torch.randn(M, K, generator=g))
    if w.has_bias_in:
        out["bias_in"] = _bf16(torch.randn(K, generator=g))
    out["gamma"] = _bf16(1.0 + 0.1 * torch.randn(K, generator=g))
    if w.norm == LAYERNORM:
        out["beta"] = _bf16(0.1 * torch.randn(K, generator=g))
    out["W"] = _bf16(torch.randn(N, K, generator=g) / (K ** 0.5))
    if w.has_bias_out:
        out["bias_out"] = _bf16(0.02 * torch.randn(N, generator=g))
    return out


def make_custom(op: str, norm: str, M: int, K: int, *, Hq=0, Hkv=0, D=0, I=0, N=0,
                bias_in=False, bias_out=False, eps=1e-5, seed=0, x_loc=0.0) -> tuple:
    """A workload of arbitrary shape with the same distributions (tile-tail and
    edge-case tests); x_loc shifts the mean of x (e.g. x ~ N(50, 1))."""
    if op == RESIDUAL:
        w = Workload(f"custom_residual_{M}x{K}x{N}", RESIDUAL, NONORM, M, K, N,
                     has_bias_out=bias_out, x_loc=x_loc)
    elif op == QKV:
        w = qkv(f"custom_qkv_{M}x{K}", M, K, Hq, Hkv, D, norm, eps=eps,
                has_bias_in=bias_in, has_bias_out=bias_out, x_loc=x_loc)
    elif op == QKV_FP8:
        w = Workload(f"custom_qkv_fp8_{M}x{K}", QKV_FP8, norm, M, K, (Hq + 2 * Hkv) * D, Hq=Hq, Hkv=Hkv, D=D,
                     eps=eps, has_bias_in=bias_in, has_bias_out=bias_out, x_loc=x_loc)
    elif op == SWIGLU_FP8:
        w = Workload(f"custom_swiglu_fp8_{M}x{K}", SWIGLU_FP8, norm, M, K, 2 * I, I=I, eps=eps,
                     has_bias_in=bias_in, has_bias_out=bias_out, x_loc=x_loc)
    elif op == GELU_FP8:
        w = Workload(f"custom_gelu_fp8_{M}x{K}", GELU_FP8, norm, M, K, N, eps=eps,
                     has_bias_in=bias_in, has_bias_out=bias_out, x_loc=x_loc)
    elif op == SWIGLU:
        w = Workload(f"custom_swiglu_{M}x{K}", SWIGLU, norm, M, K, 2 * I, I=I, eps=eps,
                     has_bias_in=bias_in, has_bias_out=bias_out, x_loc=x_loc)
    else:
        w = Workload(f"custom_gelu_{M}x{K}", GELU, norm, M, K, N, eps=eps,
                     has_bias_in=bias_in, has_bias_out=bias_out, x_loc=x_loc)
    return w, make_inputs(w, seed=seed)
