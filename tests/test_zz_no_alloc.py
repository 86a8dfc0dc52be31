"""fnl_add_norm_qkv_static: the allocation-free entry point for callers that
cannot allocate device memory on the call path (graph capture, sync-free decode
loops, engines with their own static memory plan). Called through the C-ABI
with ctypes, it must give what fnl_add_norm_qkv gives, on two calls in a row
(the second call reuses the static scratch the first one left behind).

Named to be collected last, so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

import synthetic
from parity import OUT_ABS, OUT_REL
from transformer_layer_residual_b200 import fnl

pytestmark = pytest.mark.gpu

NORM = {"layernorm": 0, "rmsnorm": 1}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_call(w, d, outs):
    L = fnl.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.fnl_add_norm_qkv_static(
        stream, _ptr(d["x"]), _ptr(d["residual"]), _ptr(outs["residual_out"]), _ptr(d["gamma"]),
        _ptr(d.get("beta")), NORM[w.norm], ctypes.c_float(w.eps), _ptr(d["W"]), _ptr(d.get("bias_out")),
        w.M, w.K, w.Hq, w.Hkv, w.D, _ptr(outs["q"]), _ptr(outs["k"]), _ptr(outs["v"]), _ptr(outs.get("mean")),
        _ptr(outs["rstd"]))


def _empty_outputs(w, dev):
    bf = dict(dtype=torch.bfloat16, device=dev)
    return {"residual_out": torch.empty(w.M, w.K, **bf), "q": torch.empty(w.Hq, w.M, w.D, **bf),
            "k": torch.empty(w.Hkv, w.M, w.D, **bf), "v": torch.empty(w.Hkv, w.M, w.D, **bf),
            "rstd": torch.empty(w.M, dtype=torch.float32, device=dev),
            "mean": torch.empty(w.M, dtype=torch.float32, device=dev) if w.norm == "layernorm" else None}


def _within_tolerance(got, ref):
    g, r = got.float(), ref.float()
    return bool(torch.all((g - r).abs() <= OUT_ABS + OUT_REL * r.abs()))


CASES = [synthetic.workloads()["c2_decode_rms_qkv"],
         synthetic.make_custom("qkv", "layernorm", 7, 520, Hq=6, Hkv=2, D=40, bias_out=True, seed=11)[0],
         synthetic.workloads()["c5_70b_rms_qkv_m8"]]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_static_matches_handle_entry_point_twice(cuda_device, w):
    torch.cuda.set_device(0)
    d = {k: t.cuda() for k, t in synthetic.make_inputs(w).items()}
    h = fnl.Handle(0)
    ref = fnl.run_workload(h, w, d)
    h.check()
    for call in range(2):
        outs = _empty_outputs(w, d["x"].device)
        for t in outs.values():
            if t is not None:
                t.fill_(float("nan"))
        st = _static_call(w, d, outs)
        assert st == 0, f"call {call}: {fnl.STATUS_NAMES.get(st, st)}"
        torch.cuda.synchronize()
        for key in ("q", "k", "v", "residual_out"):
            assert _within_tolerance(outs[key], ref[key]), (call, key)
        assert torch.allclose(outs["rstd"], ref["rstd"], rtol=1e-6, atol=0)
        if w.norm == "layernorm":
            assert torch.allclose(outs["mean"], ref["mean"], rtol=1e-6, atol=1e-7)
    h.close()


def test_static_rejects_what_does_not_fit(cuda_device):
    torch.cuda.set_device(0)
    # M beyond the decode kernel, and a split-K scratch larger than the array
    for M, Hq, Hkv in ((129, 4, 2), (128, 256, 128)):
        w = synthetic.qkv("too_big", M, 64, Hq, Hkv, 128, "rmsnorm")
        bf = dict(dtype=torch.bfloat16, device="cuda")
        d = {"x": torch.zeros(M, 64, **bf), "residual": torch.zeros(M, 64, **bf),
             "gamma": torch.ones(64, **bf), "W": torch.zeros(w.N, 64, **bf)}
        outs = _empty_outputs(w, "cuda")
        assert _static_call(w, d, outs) == 4   # FNL_ERR_UNSUPPORTED
