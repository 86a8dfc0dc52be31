"""The tensor-parallel all-reduce (fnl_tp_allreduce) against the oracle, on one
GPU: the P ranks' partial outputs are P local buffers (on a node they would be
the peers' buffers mapped into this device's address space; the kernel reads
them the same way)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity import check
from transformer_layer_residual_b200 import fnl

pytestmark = pytest.mark.gpu


def _parts(P, shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return [(scale * torch.randn(shape, generator=g)).to(torch.bfloat16) for _ in range(P)]


def _within_one_ulp(got, ref):
    """|got - ref| <= one bf16 spacing at |ref| (the fp32 sum in rank order may
    round a value that lies next to a midpoint the other way)."""
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126)))
    return np.abs(got - ref) <= np.ldexp(1.0, (e - 7).astype(int))


@pytest.fixture(scope="module")
def handle(cuda_device):
    h = fnl.Handle(0)
    yield h
    h.close()


@pytest.mark.parametrize("P", [1, 2, 3, 8, 16])
@pytest.mark.parametrize("n", [8, 1003, 32 * 4096 + 5])
def test_tp_allreduce_matches_oracle(handle, P, n):
    parts = _parts(P, (n,), seed=P * 7919 + n)
    out = fnl.tp_allreduce(handle, [p.cuda() for p in parts])
    handle.check()
    ref = oracle.tp_allreduce([p.double().numpy() for p in parts])
    got = out.double().cpu().numpy()
    assert np.all(_within_one_ulp(got, ref))
    if P == 1:
        assert torch.equal(out.cpu(), parts[0])


def test_tp_allreduce_exact_sums(handle):
    """Partials that sum exactly in fp32: the result is the oracle's bit for bit."""
    g = torch.Generator().manual_seed(5)
    parts = [torch.randint(-64, 65, (4096,), generator=g).to(torch.bfloat16) for _ in range(4)]
    out = fnl.tp_allreduce(handle, [p.cuda() for p in parts]).cpu()
    ref = oracle.tp_allreduce([p.double().numpy() for p in parts])
    assert np.array_equal(out.double().numpy(), ref)


@pytest.mark.parametrize("norm", ["rmsnorm", "layernorm"])
def test_add_norm_qkv_tp(handle, norm):
    """Decode-sized QKV (Llama-3-8B, M = 32) fed by four ranks' o_proj partials."""
    w, inputs = synthetic.make_custom("qkv", norm, 32, 4096, Hq=32, Hkv=8, D=128, seed=77)
    parts = _parts(4, (32, 4096), seed=78, scale=0.5)
    dev = {k: v.cuda() for k, v in inputs.items()}
    got = fnl.add_norm_qkv_tp(handle, [p.cuda() for p in parts], dev["residual"], dev["gamma"], dev.get("beta"),
                              dev["W"], w.Hq, w.Hkv, w.D, norm=norm, eps=w.eps, mean_out=None)
    handle.check()
    x = torch.from_numpy(oracle.tp_allreduce([p.double().numpy() for p in parts])).to(torch.bfloat16)
    check(w, {**inputs, "x": x}, got)


def test_tp_allreduce_errors(handle):
    a = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fnl.FnlError) as e:
        fnl.tp_allreduce(handle, [a, b], out=a)
    assert e.value.status == 3   # FNL_ERR_ALIAS
    big = torch.zeros(72, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fnl.FnlError) as e:
        fnl.tp_allreduce(handle, [big[1:65], b])
    assert e.value.status == 2   # FNL_ERR_ALIGNMENT
    with pytest.raises(fnl.FnlError) as e:
        fnl.tp_allreduce(handle, [b] * 17)
    assert e.value.status == 1   # FNL_ERR_INVALID_ARG
