"""Fused pre-norm linear layer for B200 (sm_100a): residual add -> LayerNorm /
RMSNorm -> bf16 tcgen05 GEMM (fp32 accumulate) -> QKV head-major split /
SwiGLU / bias + GELU, behind the C-ABI library libfnl.so (include/fnl.h).

The Python layer is a ctypes binding (``fnl``); the library is built in-tree
with ``python -m transformer_layer_residual_b200.build``.
"""
from .fnl import (  # noqa: F401
    FnlError,
    Handle,
    add_bias_norm_gelu,
    add_norm_qkv,
    add_norm_qkv_static,
    add_norm_swiglu,
    lib,
    lib_path,
    run_workload,
)
