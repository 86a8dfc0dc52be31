"""The debug build of the library (libfnl_debug.so, compiled with
FNL_DEBUG_CHECKS): every epilogue store is checked against the output buffer
it targets before it is issued; a store that would leave its buffer is skipped
and records device code 8, which fnl_check reports as FNL_ERR_DEVICE_STATUS, so
a wrong index shows up as an error instead of a write into a neighbour's
memory.

Each case runs in a child process that selects the debug build through
FNL_LIBRARY=debug (the library is loaded once per process), forces one kernel
form, and must give oracle parity with no bounds status: every kernel form,
every epilogue, row tails that cut a tile, ragged K, the stream-K forms and the
FP8 form.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FORMS = {
    "tile": [("qkv", "rmsnorm", 130, 520), ("swiglu", "layernorm", 200, 328), ("gelu", "layernorm", 5, 200),
             ("residual", "none", 129, 200)],
    "wide": [("qkv", "layernorm", 300, 520), ("swiglu", "rmsnorm", 64, 200), ("residual", "none", 7, 328)],
    "pair": [("qkv", "rmsnorm", 600, 328), ("swiglu", "layernorm", 257, 520), ("gelu", "layernorm", 129, 200),
             ("residual", "none", 255, 328)],
    # stream-K needs at least one (tile, k-block) unit per pair: 74 pairs
    "pair_sk": [("qkv", "rmsnorm", 300, 2048), ("swiglu", "layernorm", 260, 4096), ("gelu", "layernorm", 260, 2000),
                ("residual", "none", 384, 2048)],
    "splitk": [("qkv", "layernorm", 33, 1024), ("swiglu", "rmsnorm", 1, 200), ("gelu", "rmsnorm", 128, 520),
               ("residual", "none", 16, 520), ("qkv_fp8", "rmsnorm", 16, 528), ("swiglu_fp8", "layernorm", 33, 208)],
    "cluster": [("qkv", "rmsnorm", 8, 4096), ("swiglu", "layernorm", 64, 520), ("gelu", "layernorm", 5, 520),
                ("residual", "none", 128, 328), ("gelu_fp8", "rmsnorm", 7, 528), ("qkv_fp8", "layernorm", 128, 528)],
}


def _workload(synthetic, op, norm, M, K, seed):
    base = op[:-4] if op.endswith("_fp8") else op
    if base == "residual":
        return synthetic.make_custom(op, "none", M, K, N=328, bias_out=True, seed=seed)
    if base == "qkv":
        return synthetic.make_custom(op, norm, M, K, Hq=6, Hkv=2, D=40, bias_out=True, seed=seed)
    if base == "swiglu":
        return synthetic.make_custom(op, norm, M, K, I=200, bias_out=True, seed=seed)
    return synthetic.make_custom(op, norm, M, K, N=328, bias_in=True, bias_out=True, seed=seed)


def _child(path):
    """Runs in the child process: FNL_LIBRARY=debug is already set."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import synthetic
    from parity import check, fp8_inputs
    from transformer_layer_residual_b200 import fnl

    assert fnl.lib_path().endswith("libfnl_debug.so"), fnl.lib_path()
    h = fnl.Handle(0, path=path)
    with open("/proc/self/maps") as f:
        assert "libfnl_debug.so" in f.read(), "the debug build is not the loaded library"
    for i, (op, norm, M, K) in enumerate(FORMS[path]):
        w, inputs = _workload(synthetic, op, norm, M, K, seed=M + K + i)
        if op.endswith("_fp8"):
            inputs = fp8_inputs(w, inputs)
        got = fnl.run_workload(h, w, {k: v.cuda() for k, v in inputs.items() if v is not None})
        h.check()   # raises FnlError if a store was refused (device code 8)
        res = check(w, inputs, got)
        print(path, w.name, h.last_plan(), res, flush=True)
    h.close()


@pytest.mark.parametrize("path", sorted(FORMS))
def test_debug_build_parity_no_bounds_status(cuda_device, path):
    lib = os.path.join(ROOT, "transformer_layer_residual_b200", "libfnl_debug.so")
    if not os.path.exists(lib):
        pytest.fail(f"{lib} is missing: build it with python -m transformer_layer_residual_b200.build --debug")
    env = dict(os.environ, FNL_LIBRARY="debug")
    r = subprocess.run([sys.executable, os.path.abspath(__file__), path], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    print(r.stdout[-4000:])
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]


if __name__ == "__main__":
    _child(sys.argv[1])
