"""ctypes binding of libfnl.so (include/fnl.h), same names as the C entry points.

Argument marshalling only: the functions take torch CUDA tensors, check their
dtype/device/contiguity, allocate missing outputs with torch, and pass raw
pointers plus the current CUDA stream to the C library. Every step of the fused
op runs in the library's kernels. There is no fallback: if the library is
missing or the device is not sm_100, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

# FNL_LIBRARY=debug selects the debug build (output stores checked against their buffers)
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libfnl_debug.so" if os.environ.get("FNL_LIBRARY") == "debug" else "libfnl.so")
_lib = None

FNL_OK = 0
STATUS_NAMES = {0: "FNL_OK", 1: "FNL_ERR_INVALID_ARG", 2: "FNL_ERR_ALIGNMENT", 3: "FNL_ERR_ALIAS",
                4: "FNL_ERR_UNSUPPORTED", 5: "FNL_ERR_CUDA", 6: "FNL_ERR_DEVICE_STATUS"}
NORMS = {"layernorm": 0, "rmsnorm": 1}
PATHS = {"auto": 0, "tile": 1, "splitk": 2, "wide": 3, "cluster": 4, "pair": 5, "pair_sk": 6}
PRECISIONS = {"default": 0, "split": 1, "single": 2}

EXPORTED = ("fnl_create", "fnl_destroy", "fnl_status_string", "fnl_last_error", "fnl_last_plan", "fnl_check",
            "fnl_add_norm_qkv", "fnl_add_norm_swiglu", "fnl_add_bias_norm_gelu", "fnl_linear_add_residual",
            "fnl_add_norm_qkv_fp8", "fnl_add_norm_swiglu_fp8", "fnl_add_bias_norm_gelu_fp8",
            "fnl_quantize_weight_fp8", "fnl_tp_allreduce",
            "fnl_add_norm_qkv_static", "fnl_check_static")


class FnlError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class _Options(ctypes.Structure):
    _fields_ = [("max_tokens", ctypes.c_int), ("max_n", ctypes.c_int), ("path", ctypes.c_int),
                ("max_ctas", ctypes.c_int), ("precision", ctypes.c_int), ("wait_ns", ctypes.c_longlong),
                ("debug_stall_calls", ctypes.c_int), ("tune", ctypes.c_int)]


def lib_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libfnl.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m transformer_layer_residual_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.fnl_create.argtypes = [ctypes.POINTER(P), I, ctypes.POINTER(_Options)]
    L.fnl_destroy.argtypes = [P]
    L.fnl_status_string.argtypes = [I]
    L.fnl_status_string.restype = ctypes.c_char_p
    L.fnl_last_error.argtypes = [P]
    L.fnl_last_error.restype = ctypes.c_char_p
    L.fnl_last_plan.argtypes = [P]
    L.fnl_last_plan.restype = ctypes.c_char_p
    L.fnl_check.argtypes = [P, P]
    L.fnl_add_norm_qkv.argtypes = [P, P, P, P, P, P, P, I, F, P, P, I, I, I, I, I, P, P, P, P, P]
    L.fnl_add_norm_swiglu.argtypes = [P, P, P, P, P, P, P, I, F, P, P, I, I, I, P, P, P]
    L.fnl_add_bias_norm_gelu.argtypes = [P, P, P, P, P, P, P, P, I, F, P, P, I, I, I, P, P, P]
    L.fnl_linear_add_residual.argtypes = [P, P, P, P, P, P, P, I, I, I]
    L.fnl_add_norm_qkv_fp8.argtypes = [P, P, P, P, P, P, P, I, F, P, P, P, I, I, I, I, I, P, P, P, P, P]
    L.fnl_quantize_weight_fp8.argtypes = [P, P, P, I, I, P, P]
    L.fnl_tp_allreduce.argtypes = [P, P, ctypes.POINTER(P), I, P, ctypes.c_longlong]
    L.fnl_add_norm_swiglu_fp8.argtypes = [P, P, P, P, P, P, P, I, F, P, P, P, I, I, I, P, P, P]
    L.fnl_add_bias_norm_gelu_fp8.argtypes = [P, P, P, P, P, P, P, P, I, F, P, P, P, I, I, I, P, P, P]
    L.fnl_add_norm_qkv_static.argtypes = [P, P, P, P, P, P, I, F, P, P, I, I, I, I, I, P, P, P, P, P]
    L.fnl_check_static.argtypes = [P]
    for name in EXPORTED:
        if getattr(L, name).restype is None and name not in ("fnl_status_string", "fnl_last_error", "fnl_last_plan"):
            getattr(L, name).restype = I
    _lib = L
    return L


class Handle:
    """Owns an fnl_handle (device workspace). One stream / thread at a time.

    max_tokens / max_n reserve the workspace up front (no reallocation, and so
    no stream synchronisation, on later calls up to that size). path forces a
    kernel: "auto" (by M), "splitk" (small-M kernel, stream-K form), "cluster"
    (small-M kernel, cluster form), "tile" (128x256 tiles), "wide" (128x512
    tiles), "pair" (256x512 tiles on CTA pairs), "pair_sk" (the pair kernel's
    stream-K form, its split tiles finished by the fix-up kernel). max_ctas
    caps the grid (0 = all SMs). precision: "default" (split
    hi + lo operand for SwiGLU only), "split", "single". wait_ns: limit of the
    kernels' main-loop waits (0 = 4 s). debug_stall_calls: fault injection for
    tests of the status path (the next that-many calls withhold one weight copy,
    so a wait runs out and check() raises). tune: shape auto-tuning (the first
    call of each shape times the candidate plans and keeps the fastest)."""

    def __init__(self, device: int = 0, max_tokens: int = 0, max_n: int = 0, path: str = "auto",
                 max_ctas: int = 0, precision: str = "default", wait_ns: int = 0, debug_stall_calls: int = 0,
                 tune: bool = False):
        L = lib()
        self._h = ctypes.c_void_p()
        opt = _Options(max_tokens, max_n, PATHS[path], max_ctas, PRECISIONS[precision], wait_ns,
                       debug_stall_calls, int(bool(tune)))
        st = L.fnl_create(ctypes.byref(self._h), device, ctypes.byref(opt))
        if st != FNL_OK:
            raise FnlError(st, f"fnl_create(device={device}) failed")
        self.device = device

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            lib().fnl_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def ptr(self):
        return self._h

    def _raise(self, st: int, what: str):
        msg = lib().fnl_last_error(self._h)
        raise FnlError(st, f"{what}: {msg.decode() if msg else ''}")

    def last_plan(self) -> str:
        """fnl_last_plan: the kernel, form and grid of the last call."""
        t = lib().fnl_last_plan(self._h)
        return t.decode() if t else ""

    def check(self, stream: Optional[torch.cuda.Stream] = None):
        """Synchronise the stream and raise if a kernel gave up a bounded wait."""
        st = lib().fnl_check(self._h, _stream_ptr(stream))
        if st != FNL_OK:
            self._raise(st, "fnl_check")


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _need(t, name, shape=None, dtype=torch.bfloat16):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _common(x, residual, gamma, beta, norm, residual_out, mean_out, rstd_out, W, bias):
    M, K = x.shape
    _need(x, "x", (M, K))
    _need(residual, "residual", (M, K))
    _need(gamma, "gamma", (K,))
    _need(beta, "beta", (K,))
    _need(W, "W")
    if W.dim() != 2 or W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    _need(bias, "bias", (W.shape[0],))
    if residual_out is None:
        residual_out = torch.empty_like(x)
    _need(residual_out, "residual_out", (M, K))
    if norm not in NORMS:
        raise ValueError(f"norm must be one of {list(NORMS)}")
    if rstd_out is not None:
        _need(rstd_out, "rstd_out", (M,), torch.float32)
    if mean_out is not None:
        _need(mean_out, "mean_out", (M,), torch.float32)
    return M, K, residual_out


def add_norm_qkv(h: Handle, x, residual, gamma, beta, W, Hq, Hkv, D, norm="rmsnorm", eps=1e-5, bias=None,
                 residual_out=None, q=None, k=None, v=None, mean_out=None, rstd_out=None, stream=None):
    """fnl_add_norm_qkv. Returns dict(residual_out, q [Hq,M,D], k, v, mean, rstd)."""
    M, K, residual_out = _common(x, residual, gamma, beta, norm, residual_out, mean_out, rstd_out, W, bias)
    q = torch.empty(Hq, M, D, dtype=torch.bfloat16, device=x.device) if q is None else q
    k = torch.empty(Hkv, M, D, dtype=torch.bfloat16, device=x.device) if k is None else k
    v = torch.empty(Hkv, M, D, dtype=torch.bfloat16, device=x.device) if v is None else v
    _need(q, "q", (Hq, M, D)); _need(k, "k", (Hkv, M, D)); _need(v, "v", (Hkv, M, D))
    st = lib().fnl_add_norm_qkv(h.ptr, _stream_ptr(stream), _p(x), _p(residual), _p(residual_out), _p(gamma),
                                _p(beta), NORMS[norm], float(eps), _p(W), _p(bias), M, K, Hq, Hkv, D,
                                _p(q), _p(k), _p(v), _p(mean_out), _p(rstd_out))
    if st != FNL_OK:
        h._raise(st, "fnl_add_norm_qkv")
    return {"residual_out": residual_out, "q": q, "k": k, "v": v, "mean": mean_out, "rstd": rstd_out}


def add_norm_swiglu(h: Handle, x, residual, gamma, beta, W, I, norm="rmsnorm", eps=1e-5, bias=None,
                    residual_out=None, out=None, mean_out=None, rstd_out=None, stream=None):
    """fnl_add_norm_swiglu. W is [2I, K] (gate rows then up rows). Returns dict."""
    M, K, residual_out = _common(x, residual, gamma, beta, norm, residual_out, mean_out, rstd_out, W, bias)
    out = torch.empty(M, I, dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, "out", (M, I))
    st = lib().fnl_add_norm_swiglu(h.ptr, _stream_ptr(stream), _p(x), _p(residual), _p(residual_out),
                                   _p(gamma), _p(beta), NORMS[norm], float(eps), _p(W), _p(bias), M, K, I,
                                   _p(out), _p(mean_out), _p(rstd_out))
    if st != FNL_OK:
        h._raise(st, "fnl_add_norm_swiglu")
    return {"residual_out": residual_out, "out": out, "mean": mean_out, "rstd": rstd_out}


def add_bias_norm_gelu(h: Handle, x, residual, gamma, beta, W, bias_in=None, bias_out=None, norm="layernorm",
                       eps=1e-5, residual_out=None, out=None, mean_out=None, rstd_out=None, stream=None):
    """fnl_add_bias_norm_gelu. Returns dict(residual_out, out [M,N], mean, rstd)."""
    M, K, residual_out = _common(x, residual, gamma, beta, norm, residual_out, mean_out, rstd_out, W,
                                 bias_out)
    _need(bias_in, "bias_in", (K,))
    N = W.shape[0]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, "out", (M, N))
    st = lib().fnl_add_bias_norm_gelu(h.ptr, _stream_ptr(stream), _p(x), _p(residual), _p(bias_in),
                                      _p(residual_out), _p(gamma), _p(beta), NORMS[norm], float(eps), _p(W),
                                      _p(bias_out), M, K, N, _p(out), _p(mean_out), _p(rstd_out))
    if st != FNL_OK:
        h._raise(st, "fnl_add_bias_norm_gelu")
    return {"residual_out": residual_out, "out": out, "mean": mean_out, "rstd": rstd_out}


def tp_allreduce(h: Handle, parts, out=None, stream=None):
    """fnl_tp_allreduce: out = bf16(sum of the P same-shape bf16 tensors in
    `parts`, in list order). On a node the parts are the ranks' partial outputs
    (the peers' as tensors over their mapped memory); here any device tensors.
    Returns out."""
    parts = list(parts)
    if not parts:
        raise ValueError("tp_allreduce needs at least one part")
    shape = tuple(parts[0].shape)
    for t in parts:
        _need(t, "part", shape)
    out = torch.empty(shape, dtype=torch.bfloat16, device=parts[0].device) if out is None else out
    _need(out, "out", shape)
    arr = (ctypes.c_void_p * len(parts))(*[t.data_ptr() for t in parts])
    st = lib().fnl_tp_allreduce(h.ptr, _stream_ptr(stream), arr, len(parts), _p(out), out.numel())
    if st != FNL_OK:
        h._raise(st, "fnl_tp_allreduce")
    return out


def add_norm_qkv_tp(h: Handle, parts, residual, gamma, beta, W, Hq, Hkv, D, norm="rmsnorm", eps=1e-5, bias=None,
                    x_buf=None, stream=None, **outs):
    """The QKV op fed by the tensor-parallel all-reduce: x = tp_allreduce(parts)
    (into x_buf if given), then add_norm_qkv(x, residual, ...). Two launches on
    the stream; the fused op is a programmatic dependent of the all-reduce."""
    x = tp_allreduce(h, parts, out=x_buf, stream=stream)
    return add_norm_qkv(h, x, residual, gamma, beta, W, Hq, Hkv, D, norm=norm, eps=eps, bias=bias, stream=stream,
                        **outs)


def linear_add_residual(h: Handle, a, W, residual, bias=None, out=None, stream=None):
    """fnl_linear_add_residual: out = residual + a W^T (+ bias), bf16. a [M, K],
    W [N, K], residual [M, N]; out may be `residual` itself (in-place update of
    the residual stream). Returns dict(out)."""
    M, K = a.shape
    _need(a, "a", (M, K))
    _need(W, "W")
    if W.dim() != 2 or W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    N = W.shape[0]
    _need(bias, "bias", (N,))
    _need(residual, "residual", (M, N))
    out = torch.empty(M, N, dtype=torch.bfloat16, device=a.device) if out is None else out
    _need(out, "out", (M, N))
    st = lib().fnl_linear_add_residual(h.ptr, _stream_ptr(stream), _p(a), _p(W), _p(bias), _p(residual), _p(out),
                                       M, K, N)
    if st != FNL_OK:
        h._raise(st, "fnl_linear_add_residual")
    return {"out": out}


def quantize_weight_fp8(h: Handle, W, stream=None):
    """fnl_quantize_weight_fp8: (Wq uint8 [N, K] e4m3 codes, w_scale fp32 [N])."""
    _need(W, "W")
    if W.dim() != 2:
        raise ValueError("W must be [N, K]")
    N, K = W.shape
    Wq = torch.empty(N, K, dtype=torch.uint8, device=W.device)
    w_scale = torch.empty(N, dtype=torch.float32, device=W.device)
    st = lib().fnl_quantize_weight_fp8(h.ptr, _stream_ptr(stream), _p(W), N, K, _p(Wq), _p(w_scale))
    if st != FNL_OK:
        h._raise(st, "fnl_quantize_weight_fp8")
    return Wq, w_scale


def add_norm_qkv_fp8(h: Handle, x, residual, gamma, beta, Wq, w_scale, Hq, Hkv, D, norm="rmsnorm", eps=1e-5,
                     bias=None, residual_out=None, q=None, k=None, v=None, mean_out=None, rstd_out=None,
                     stream=None):
    """fnl_add_norm_qkv_fp8: Wq uint8 [N, K] e4m3 codes, w_scale fp32 [N].
    Returns dict(residual_out, q, k, v, mean, rstd)."""
    M, K = x.shape
    _need(x, "x", (M, K))
    _need(residual, "residual", (M, K))
    _need(gamma, "gamma", (K,))
    _need(beta, "beta", (K,))
    N = (Hq + 2 * Hkv) * D
    _need(Wq, "Wq", (N, K), torch.uint8)
    _need(w_scale, "w_scale", (N,), torch.float32)
    _need(bias, "bias", (N,))
    if norm not in NORMS:
        raise ValueError(f"norm must be one of {list(NORMS)}")
    residual_out = torch.empty_like(x) if residual_out is None else residual_out
    q = torch.empty(Hq, M, D, dtype=torch.bfloat16, device=x.device) if q is None else q
    k = torch.empty(Hkv, M, D, dtype=torch.bfloat16, device=x.device) if k is None else k
    v = torch.empty(Hkv, M, D, dtype=torch.bfloat16, device=x.device) if v is None else v
    _need(residual_out, "residual_out", (M, K))
    _need(q, "q", (Hq, M, D)); _need(k, "k", (Hkv, M, D)); _need(v, "v", (Hkv, M, D))
    if rstd_out is not None:
        _need(rstd_out, "rstd_out", (M,), torch.float32)
    if mean_out is not None:
        _need(mean_out, "mean_out", (M,), torch.float32)
    st = lib().fnl_add_norm_qkv_fp8(h.ptr, _stream_ptr(stream), _p(x), _p(residual), _p(residual_out), _p(gamma),
                                    _p(beta), NORMS[norm], float(eps), _p(Wq), _p(w_scale), _p(bias), M, K, Hq,
                                    Hkv, D, _p(q), _p(k), _p(v), _p(mean_out), _p(rstd_out))
    if st != FNL_OK:
        h._raise(st, "fnl_add_norm_qkv_fp8")
    return {"residual_out": residual_out, "q": q, "k": k, "v": v, "mean": mean_out, "rstd": rstd_out}


def _fp8_common(x, residual, gamma, beta, Wq, w_scale, n_rows, norm, residual_out, mean_out, rstd_out):
    M, K = x.shape
    _need(x, "x", (M, K))
    _need(residual, "residual", (M, K))
    _need(gamma, "gamma", (K,))
    _need(beta, "beta", (K,))
    _need(Wq, "Wq", (n_rows, K), torch.uint8)
    _need(w_scale, "w_scale", (n_rows,), torch.float32)
    if norm not in NORMS:
        raise ValueError(f"norm must be one of {list(NORMS)}")
    residual_out = torch.empty_like(x) if residual_out is None else residual_out
    _need(residual_out, "residual_out", (M, K))
    if rstd_out is not None:
        _need(rstd_out, "rstd_out", (M,), torch.float32)
    if mean_out is not None:
        _need(mean_out, "mean_out", (M,), torch.float32)
    return M, K, residual_out


def add_norm_swiglu_fp8(h: Handle, x, residual, gamma, beta, Wq, w_scale, I, norm="rmsnorm", eps=1e-5, bias=None,
                        residual_out=None, out=None, mean_out=None, rstd_out=None, stream=None):
    """fnl_add_norm_swiglu_fp8: Wq uint8 [2I, K] e4m3 codes (gate rows, then up
    rows), w_scale fp32 [2I]. Returns dict(residual_out, out [M, I], mean, rstd)."""
    M, K, residual_out = _fp8_common(x, residual, gamma, beta, Wq, w_scale, 2 * I, norm, residual_out, mean_out,
                                     rstd_out)
    _need(bias, "bias", (2 * I,))
    out = torch.empty(M, I, dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, "out", (M, I))
    st = lib().fnl_add_norm_swiglu_fp8(h.ptr, _stream_ptr(stream), _p(x), _p(residual), _p(residual_out),
                                       _p(gamma), _p(beta), NORMS[norm], float(eps), _p(Wq), _p(w_scale), _p(bias),
                                       M, K, I, _p(out), _p(mean_out), _p(rstd_out))
    if st != FNL_OK:
        h._raise(st, "fnl_add_norm_swiglu_fp8")
    return {"residual_out": residual_out, "out": out, "mean": mean_out, "rstd": rstd_out}


def add_bias_norm_gelu_fp8(h: Handle, x, residual, gamma, beta, Wq, w_scale, bias_in=None, bias_out=None,
                           norm="layernorm", eps=1e-5, residual_out=None, out=None, mean_out=None, rstd_out=None,
                           stream=None):
    """fnl_add_bias_norm_gelu_fp8: Wq uint8 [N, K] e4m3 codes, w_scale fp32 [N].
    Returns dict(residual_out, out [M, N], mean, rstd)."""
    N = Wq.shape[0]
    M, K, residual_out = _fp8_common(x, residual, gamma, beta, Wq, w_scale, N, norm, residual_out, mean_out,
                                     rstd_out)
    _need(bias_in, "bias_in", (K,))
    _need(bias_out, "bias_out", (N,))
    out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, "out", (M, N))
    st = lib().fnl_add_bias_norm_gelu_fp8(h.ptr, _stream_ptr(stream), _p(x), _p(residual), _p(bias_in),
                                          _p(residual_out), _p(gamma), _p(beta), NORMS[norm], float(eps), _p(Wq),
                                          _p(w_scale), _p(bias_out), M, K, N, _p(out), _p(mean_out), _p(rstd_out))
    if st != FNL_OK:
        h._raise(st, "fnl_add_bias_norm_gelu_fp8")
    return {"residual_out": residual_out, "out": out, "mean": mean_out, "rstd": rstd_out}


def run_workload(h: Handle, w, dev: dict, stats: bool = True, stream=None) -> dict:
    """Run a synthetic.Workload on device tensors `dev` (same keys as
    synthetic.make_inputs). Allocates the outputs and statistics buffers."""
    if w.op == "residual":
        return linear_add_residual(h, dev["x"], dev["W"], dev["residual"], bias=dev.get("bias_out"), stream=stream)
    M = dev["x"].shape[0]
    if w.op.endswith("_fp8"):   # dev["W_fp8"]: e4m3 codes (float8_e4m3fn or uint8), dev["w_scale"]: fp32 [N]
        rstd = torch.empty(M, dtype=torch.float32, device=dev["x"].device) if stats else None
        mean = (torch.empty(M, dtype=torch.float32, device=dev["x"].device)
                if stats and w.norm == "layernorm" else None)
        Wq = dev["W_fp8"]
        Wq = Wq.view(torch.uint8) if Wq.dtype != torch.uint8 else Wq
        if w.op == "swiglu_fp8":
            return add_norm_swiglu_fp8(h, dev["x"], dev["residual"], dev["gamma"], dev.get("beta"), Wq,
                                       dev["w_scale"], w.I, norm=w.norm, eps=w.eps, bias=dev.get("bias_out"),
                                       mean_out=mean, rstd_out=rstd, stream=stream)
        if w.op == "gelu_fp8":
            return add_bias_norm_gelu_fp8(h, dev["x"], dev["residual"], dev["gamma"], dev.get("beta"), Wq,
                                          dev["w_scale"], bias_in=dev.get("bias_in"), bias_out=dev.get("bias_out"),
                                          norm=w.norm, eps=w.eps, mean_out=mean, rstd_out=rstd, stream=stream)
        return add_norm_qkv_fp8(h, dev["x"], dev["residual"], dev["gamma"], dev.get("beta"), Wq, dev["w_scale"],
                                w.Hq, w.Hkv, w.D, norm=w.norm, eps=w.eps, bias=dev.get("bias_out"), mean_out=mean,
                                rstd_out=rstd, stream=stream)
    rstd = torch.empty(M, dtype=torch.float32, device=dev["x"].device) if stats else None
    mean = (torch.empty(M, dtype=torch.float32, device=dev["x"].device)
            if stats and w.norm == "layernorm" else None)
    if w.op == "qkv":
        return add_norm_qkv(h, dev["x"], dev["residual"], dev["gamma"], dev.get("beta"), dev["W"], w.Hq, w.Hkv,
                            w.D, norm=w.norm, eps=w.eps, bias=dev.get("bias_out"), mean_out=mean,
                            rstd_out=rstd, stream=stream)
    if w.op == "swiglu":
        return add_norm_swiglu(h, dev["x"], dev["residual"], dev["gamma"], dev.get("beta"), dev["W"], w.I,
                               norm=w.norm, eps=w.eps, bias=dev.get("bias_out"), mean_out=mean, rstd_out=rstd,
                               stream=stream)
    return add_bias_norm_gelu(h, dev["x"], dev["residual"], dev["gamma"], dev.get("beta"), dev["W"],
                              bias_in=dev.get("bias_in"), bias_out=dev.get("bias_out"), norm=w.norm, eps=w.eps,
                              mean_out=mean, rstd_out=rstd, stream=stream)


def add_norm_qkv_static(x, residual, gamma, beta, W, Hq, Hkv, D, norm="rmsnorm", eps=1e-5, bias=None,
                        residual_out=None, q=None, k=None, v=None, mean_out=None, rstd_out=None, stream=None):
    """fnl_add_norm_qkv_static: fnl_add_norm_qkv without a handle and without
    any device allocation inside the library (its scratch is a static device
    array of the library; M <= 128). Output tensors not given are allocated
    here by torch, before the call. Returns the same dict as add_norm_qkv."""
    M, K, residual_out = _common(x, residual, gamma, beta, norm, residual_out, mean_out, rstd_out, W, bias)
    q = torch.empty(Hq, M, D, dtype=torch.bfloat16, device=x.device) if q is None else q
    k = torch.empty(Hkv, M, D, dtype=torch.bfloat16, device=x.device) if k is None else k
    v = torch.empty(Hkv, M, D, dtype=torch.bfloat16, device=x.device) if v is None else v
    _need(q, "q", (Hq, M, D)); _need(k, "k", (Hkv, M, D)); _need(v, "v", (Hkv, M, D))
    st = lib().fnl_add_norm_qkv_static(_stream_ptr(stream), _p(x), _p(residual), _p(residual_out), _p(gamma),
                                       _p(beta), NORMS[norm], float(eps), _p(W), _p(bias), M, K, Hq, Hkv, D,
                                       _p(q), _p(k), _p(v), _p(mean_out), _p(rstd_out))
    if st != FNL_OK:
        raise FnlError(st, "fnl_add_norm_qkv_static")
    return {"residual_out": residual_out, "q": q, "k": k, "v": v, "mean": mean_out, "rstd": rstd_out}


def check_static(stream=None):
    """fnl_check_static: synchronise the stream and raise if a call of the
    allocation-free entry point gave up a bounded wait since the last check."""
    st = lib().fnl_check_static(_stream_ptr(stream))
    if st != FNL_OK:
        raise FnlError(st, "fnl_check_static")
