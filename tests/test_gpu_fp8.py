"""GPU parity of the FP8 (W8A8) form: the weight quantiser bit for bit against
the oracle's, and the fused FP8 QKV op (decode shapes, tails, both small-M
forms) against the fp64 oracle's FP8 arithmetic, on weights the oracle
quantised."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity import check, fp8_inputs
from transformer_layer_residual_b200 import fnl

pytestmark = pytest.mark.gpu

WL = synthetic.workloads()


@pytest.fixture(scope="module")
def handle(cuda_device):
    h = fnl.Handle(0)
    yield h
    h.check()
    h.close()


@pytest.mark.parametrize("N,K,seed", [(64, 4096, 1), (130, 520, 2), (8, 8, 3)])
def test_weight_quantizer_matches_oracle(handle, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=g) * 0.03).to(torch.bfloat16)
    W[min(3, N - 1)] = 0.0                       # an all-zero row: scale 1, codes 0
    W[0, 0] = 0.5                                # a row whose amax is one clear element
    Wq, ws = fnl.quantize_weight_fp8(handle, W.cuda())
    handle.check()
    codes, scale = oracle.quantize_weight_fp8(W.double().numpy())
    ref = torch.from_numpy(codes).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(Wq.cpu(), ref)
    assert np.array_equal(ws.cpu().numpy(), scale)


def run_fp8(h, w, inputs):
    full = fp8_inputs(w, inputs)
    dev = {k: v.cuda() for k, v in full.items()}
    got = fnl.run_workload(h, w, dev)
    h.check()
    return check(w, full, got)


@pytest.mark.parametrize("name", sorted(synthetic.fp8_workloads()))
def test_fp8_full_compare(handle, name):
    w = WL[name]
    res = run_fp8(handle, w, synthetic.make_inputs(w))
    print(name, res)


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
@pytest.mark.parametrize("M", [1, 7, 16, 33, 128])
def test_fp8_tails(handle, norm, M):
    # K = 208: three full 64-wide k-blocks and a ragged one; N not a tile multiple
    w, inputs = synthetic.make_custom("qkv_fp8", norm, M, 208, Hq=6, Hkv=2, D=40, bias_out=True, seed=M)
    run_fp8(handle, w, inputs)


@pytest.mark.parametrize("path", ["splitk", "cluster"])
def test_fp8_forced_forms(cuda_device, path):
    h = fnl.Handle(0, path=path)
    for M in (5, 64, 128):
        w, inputs = synthetic.make_custom("qkv_fp8", "layernorm", M, 528, Hq=6, Hkv=2, D=40, bias_out=True,
                                          seed=M)
        run_fp8(h, w, inputs)
    h.close()


def test_fp8_large_mean(handle):
    w, inputs = synthetic.make_custom("qkv_fp8", "layernorm", 16, 4096, Hq=6, Hkv=2, D=64, seed=5, x_loc=50.0)
    run_fp8(handle, w, inputs)


def test_fp8_errors(cuda_device):
    bf = dict(dtype=torch.bfloat16, device="cuda")
    Hq, Hkv, D = 2, 1, 16
    N = (Hq + 2 * Hkv) * D
    h = fnl.Handle(0)
    for M, K, status in ((129, 64, 4), (4, 200, 2)):   # M past the small-M kernel; K not a multiple of 16
        x = torch.randn(M, K, **bf)
        Wq = torch.zeros(N, K, dtype=torch.uint8, device="cuda")
        with pytest.raises(fnl.FnlError) as e:
            fnl.add_norm_qkv_fp8(h, x, x.clone(), torch.ones(K, **bf), None, Wq,
                                 torch.ones(N, dtype=torch.float32, device="cuda"), Hq, Hkv, D)
        assert e.value.status == status
    h.close()
    h = fnl.Handle(0, path="tile")
    x = torch.randn(4, 64, **bf)
    with pytest.raises(fnl.FnlError) as e:
        fnl.add_norm_qkv_fp8(h, x, x.clone(), torch.ones(64, **bf), None,
                             torch.zeros(N, 64, dtype=torch.uint8, device="cuda"),
                             torch.ones(N, dtype=torch.float32, device="cuda"), Hq, Hkv, D)
    assert e.value.status == 4
    h.close()


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
@pytest.mark.parametrize("M", [1, 16, 33, 128])
def test_fp8_swiglu_tails(handle, norm, M):
    w, inputs = synthetic.make_custom("swiglu_fp8", norm, M, 208, I=200, bias_out=True, seed=M + 1)
    run_fp8(handle, w, inputs)


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
@pytest.mark.parametrize("M", [1, 16, 33, 128])
def test_fp8_gelu_tails(handle, norm, M):
    w, inputs = synthetic.make_custom("gelu_fp8", norm, M, 208, N=328, bias_in=True, bias_out=True, seed=M + 2)
    run_fp8(handle, w, inputs)


@pytest.mark.parametrize("op", ["swiglu_fp8", "gelu_fp8"])
@pytest.mark.parametrize("path", ["splitk", "cluster"])
def test_fp8_epilogues_forced_forms(cuda_device, op, path):
    h = fnl.Handle(0, path=path)
    for M in (5, 64):
        if op == "swiglu_fp8":
            w, inputs = synthetic.make_custom(op, "rmsnorm", M, 528, I=200, bias_out=True, seed=M)
        else:
            w, inputs = synthetic.make_custom(op, "layernorm", M, 528, N=328, bias_in=True, bias_out=True, seed=M)
        run_fp8(h, w, inputs)
    h.close()
