"""fnl_add_norm_qkv_static: the allocation-free entry point for callers that
cannot call cudaMalloc on the call path (plugins in an engine that owns all
device memory through its own static memory plan, decode loops that must not
pay cudaMalloc's implicit synchronisation). Called through the C-ABI with
ctypes, on two calls in a row (the second call reuses the static scratch the
first one left behind), it must match the fp64 oracle within the tolerance of
every other parity test, give bitwise what fnl_add_norm_qkv gives on a handle
forced to the same kernel (FNL_PATH_SPLITK), leave the device's free memory
unchanged, and leave fnl_check_static reporting no failed wait.

Named to be collected last, so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

import synthetic
from parity import check
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


CASES = [synthetic.workloads()["c2_decode_rms_qkv"],
         synthetic.make_custom("qkv", "layernorm", 7, 520, Hq=6, Hkv=2, D=40, bias_out=True, seed=11)[0],
         synthetic.workloads()["c5_70b_rms_qkv_m8"]]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_static_matches_oracle_and_handle_entry_point_twice(cuda_device, w):
    torch.cuda.set_device(0)
    inputs = synthetic.make_inputs(w)
    d = {k: t.cuda() for k, t in inputs.items()}
    h = fnl.Handle(0, path="splitk")
    ref = fnl.run_workload(h, w, d)
    h.check()
    free = []
    for call in range(2):
        outs = _empty_outputs(w, d["x"].device)
        for t in outs.values():
            if t is not None:
                t.fill_(float("nan"))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        st = _static_call(w, d, outs)
        assert st == 0, f"call {call}: {fnl.STATUS_NAMES.get(st, st)}"
        fnl.check_static()   # synchronises the stream; no failed wait
        free.append(free0 - torch.cuda.mem_get_info()[0])
        res = check(w, inputs, outs)   # against the fp64 oracle
        print(w.name, call, res)
        for key in ("q", "k", "v", "residual_out", "rstd"):
            assert torch.equal(outs[key], ref[key]), (call, key)
        if w.norm == "layernorm":
            assert torch.equal(outs["mean"], ref["mean"])
    # the second call allocates nothing on the device (the first one may load the
    # library's module, which holds the static array)
    assert free[1] == 0, free
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
