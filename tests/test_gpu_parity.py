"""GPU parity: the CUDA path (through the C-ABI) against the fp64 oracle.

Every workload runs at its full size in the launch configuration the benchmark
times; small workloads are compared on every element, large ones on a seeded
row sample (tile boundaries, packed-sequence boundaries, random rows), with
residual_out and the statistics compared on every row.
"""
import numpy as np
import pytest
import torch

import synthetic
from parity import check, sample_rows
from transformer_layer_residual_b200 import fnl

pytestmark = pytest.mark.gpu

WL = synthetic.workloads()


@pytest.fixture(scope="module")
def handle(cuda_device):
    h = fnl.Handle(0)
    yield h
    h.check()
    h.close()


def run_and_check(h, w, inputs, rows=None, **hkw):
    dev = {k: v.cuda() for k, v in inputs.items()}
    got = fnl.run_workload(h, w, dev)
    h.check()
    res = check(w, inputs, got, rows=rows)
    return res, got


@pytest.mark.parametrize("name", ["c1_tiny_ln_qkv", "c2_decode_rms_qkv", "c5_70b_rms_qkv_m1",
                                  "c5_70b_rms_qkv_m8", "c5_70b_rms_qkv_m32", "c5_70b_rms_qkv_m256",
                                  "llama3_8b_o_proj_decode"])
def test_full_compare(handle, name):
    w = WL[name]
    res, _ = run_and_check(handle, w, synthetic.make_inputs(w))
    print(name, res)


@pytest.mark.parametrize("name", ["c3_prefill_rms_swiglu", "c4_gpt_ln_gelu", "c5_70b_rms_qkv_m2048",
                                  "c5_70b_rms_qkv_m8192", "c5_70b_rms_qkv_ragged", "llama3_8b_down_proj_prefill"])
def test_sampled_compare(handle, name):
    w = WL[name]
    inputs = synthetic.make_inputs(w)
    rows = sample_rows(w.M, w.seq_lens)
    res, _ = run_and_check(handle, w, inputs, rows=rows)
    print(name, res)


TAIL_CASES = []
for op in ("qkv", "swiglu", "gelu"):
    for norm in ("layernorm", "rmsnorm"):
        for M in (1, 7, 16, 129, 200):
            TAIL_CASES.append((op, norm, M))
for M in (1, 7, 16, 129, 200):
    TAIL_CASES.append(("residual", "none", M))


def _tail_workload(op, norm, M, K=200, seed=3):
    # K = 200: three full 64-wide k-blocks and a ragged one; N not a tile multiple
    if op == "residual":
        return synthetic.make_custom(op, "none", M, K, N=328, bias_out=True, seed=seed)
    if op == "qkv":
        return synthetic.make_custom(op, norm, M, K, Hq=6, Hkv=2, D=40, bias_out=True, seed=seed)
    if op == "swiglu":
        return synthetic.make_custom(op, norm, M, K, I=200, bias_out=True, seed=seed)
    return synthetic.make_custom(op, norm, M, K, N=328, bias_in=True, bias_out=True, seed=seed)


@pytest.mark.parametrize("op,norm,M", TAIL_CASES)
def test_tile_tails(handle, op, norm, M):
    w, inputs = _tail_workload(op, norm, M)
    run_and_check(handle, w, inputs)


FORCED = [(op, norm) for op in ("qkv", "swiglu", "gelu") for norm in ("layernorm", "rmsnorm")]
FORCED.append(("residual", "none"))


@pytest.mark.parametrize("path", ["tile", "wide", "pair", "splitk", "cluster"])
@pytest.mark.parametrize("op,norm", FORCED)
def test_forced_paths(cuda_device, path, op, norm):
    """Both kernels on the same small-M problems (the dispatch threshold is a
    performance choice, not a correctness one)."""
    h = fnl.Handle(0, path=path)
    for M in (5, 64, 128):
        w, inputs = _tail_workload(op, norm, M, K=520, seed=M)
        run_and_check(h, w, inputs)
    h.close()


@pytest.mark.parametrize("path", ["splitk", "cluster"])
@pytest.mark.parametrize("name", ["c2_decode_rms_qkv", "c1_tiny_ln_qkv"])
def test_small_m_forms(cuda_device, path, name):
    """The small-M kernel's stream-K and cluster forms, each at full size (the
    automatic choice takes the cluster form for these shapes when it fits)."""
    w = WL[name]
    h = fnl.Handle(0, path=path)
    run_and_check(h, w, synthetic.make_inputs(w))
    h.close()


def test_few_ctas_many_segments(cuda_device):
    """Capping the grid forces several split-K segments and tiles per CTA."""
    for ctas in (1, 3, 7):
        h = fnl.Handle(0, max_ctas=ctas)
        w, inputs = _tail_workload("qkv", "rmsnorm", 33, K=1024)
        run_and_check(h, w, inputs)
        w, inputs = _tail_workload("swiglu", "layernorm", 300, K=320)
        run_and_check(h, w, inputs)
        h.close()


def test_deterministic(handle):
    w = WL["c2_decode_rms_qkv"]
    dev = {k: v.cuda() for k, v in synthetic.make_inputs(w).items()}
    a = fnl.run_workload(handle, w, dev)
    b = fnl.run_workload(handle, w, dev)
    handle.check()
    for k in ("q", "k", "v", "residual_out", "rstd"):
        assert torch.equal(a[k], b[k]), k


def test_m_zero_is_a_noop(handle):
    K, Hq, Hkv, D = 64, 2, 1, 8
    x = torch.zeros(0, K, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((Hq + 2 * Hkv) * D, K, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(K, dtype=torch.bfloat16, device="cuda")
    out = fnl.add_norm_qkv(handle, x, x.clone(), g, None, W, Hq, Hkv, D, norm="rmsnorm")
    handle.check()
    assert out["q"].shape == (Hq, 0, D)


def test_output_guard_bands(handle):
    """Outputs written into the middle of larger buffers leave the sentinels alone."""
    w, inputs = _tail_workload("qkv", "layernorm", 129)
    dev = {k: v.cuda() for k, v in inputs.items()}
    M, K = w.M, w.K
    pad = 64
    sent = torch.tensor(-12345.0, dtype=torch.bfloat16)

    def guarded(n):
        buf = torch.full((n + 2 * pad,), float(sent), dtype=torch.bfloat16, device="cuda")
        return buf, buf[pad:pad + n]

    rb, ro = guarded(M * K)
    qb, qo = guarded(w.Hq * M * w.D)
    kbuf, ko = guarded(w.Hkv * M * w.D)
    vb, vo = guarded(w.Hkv * M * w.D)
    fnl.add_norm_qkv(handle, dev["x"], dev["residual"], dev["gamma"], dev["beta"], dev["W"], w.Hq, w.Hkv, w.D,
                     norm=w.norm, bias=dev["bias_out"], residual_out=ro.view(M, K),
                     q=qo.view(w.Hq, M, w.D), k=ko.view(w.Hkv, M, w.D), v=vo.view(w.Hkv, M, w.D))
    handle.check()
    for buf in (rb, qb, kbuf, vb):
        assert torch.all(buf[:pad] == sent) and torch.all(buf[-pad:] == sent)


def test_argument_errors(handle):
    K, Hq, Hkv, D, M = 64, 2, 1, 8, 4
    bf = dict(dtype=torch.bfloat16, device="cuda")
    x = torch.randn(M, K, **bf)
    r = torch.randn(M, K, **bf)
    g = torch.ones(K, **bf)
    W = torch.randn((Hq + 2 * Hkv) * D, K, **bf)
    with pytest.raises(fnl.FnlError) as e:   # residual_out aliases x
        fnl.add_norm_qkv(handle, x, r, g, None, W, Hq, Hkv, D, residual_out=x)
    assert e.value.status == 3
    with pytest.raises(fnl.FnlError) as e:   # beta with RMSNorm
        fnl.add_norm_qkv(handle, x, r, g, g, W, Hq, Hkv, D, norm="rmsnorm")
    assert e.value.status == 1
    with pytest.raises(fnl.FnlError) as e:   # Hq not a multiple of Hkv
        fnl.add_norm_qkv(handle, x, r, g, None, torch.randn(5 * 8 + 2 * 2 * 8, K, **bf), 5, 2, 8)
    assert e.value.status == 1
    big = torch.randn(M * K + 8, **bf)
    with pytest.raises(fnl.FnlError) as e:   # misaligned x (2-byte offset)
        fnl.add_norm_qkv(handle, big[1:1 + M * K].view(M, K), r, g, None, W, Hq, Hkv, D)
    assert e.value.status == 2
    xs = torch.randn(M, 12, **bf)
    with pytest.raises(fnl.FnlError) as e:   # K not a multiple of 8
        fnl.add_norm_qkv(handle, xs, xs.clone(), torch.ones(12, **bf), None, torch.randn(32, 12, **bf), 2, 1, 8)
    assert e.value.status == 2
    handle.check()


@pytest.mark.parametrize("path", ["splitk", "cluster", "tile", "wide", "pair"])
def test_device_status_path(cuda_device, path):
    """A wait that runs out: the call's first CTA withholds one weight copy
    (fault injection), its wait gives up after 2 ms, fnl_check reports
    FNL_ERR_DEVICE_STATUS and resets the split-K arrival counters, and the next
    normal call on the same handle matches the oracle."""
    h = fnl.Handle(0, path=path, wait_ns=2_000_000, debug_stall_calls=1)
    M = 64 if path in ("splitk", "cluster") else 300
    w, inputs = _tail_workload("qkv", "rmsnorm", M, K=1024, seed=9)
    dev = {k: v.cuda() for k, v in inputs.items()}
    fnl.run_workload(h, w, dev)
    with pytest.raises(fnl.FnlError) as e:
        h.check()
    assert e.value.status == 6
    for _ in range(2):
        got = fnl.run_workload(h, w, dev)
        h.check()
        check(w, inputs, got)
    h.close()


@pytest.mark.parametrize("path", ["auto", "splitk", "tile", "wide", "pair"])
@pytest.mark.parametrize("op", ["qkv", "gelu"])
@pytest.mark.parametrize("M", [16, 200])
def test_layernorm_large_mean(cuda_device, path, op, M):
    """x ~ N(50, 1): |mean| >> sigma, where a one-pass variance would cancel;
    the statistics kernel's two-pass fp32 reduction must still meet 1e-5."""
    if path == "splitk" and M > 128:
        pytest.skip("the small-M kernel takes M <= 128")
    h = fnl.Handle(0, path=path)
    if op == "qkv":
        w, inputs = synthetic.make_custom(op, "layernorm", M, 4096, Hq=6, Hkv=2, D=64, bias_out=True,
                                          seed=5, x_loc=50.0)
    else:
        w, inputs = synthetic.make_custom(op, "layernorm", M, 4096, N=520, bias_in=True, bias_out=True,
                                          seed=6, x_loc=50.0)
    res, _ = run_and_check(h, w, inputs)
    print(path, op, M, res)
    h.close()


def test_eps_must_be_positive(handle):
    K, Hq, Hkv, D, M = 64, 2, 1, 8, 4
    bf = dict(dtype=torch.bfloat16, device="cuda")
    x, r = torch.randn(M, K, **bf), torch.randn(M, K, **bf)
    g = torch.ones(K, **bf)
    W = torch.randn((Hq + 2 * Hkv) * D, K, **bf)
    for eps in (0.0, -1e-5, float("nan"), float("inf")):
        with pytest.raises(fnl.FnlError) as e:
            fnl.add_norm_qkv(handle, x, r, g, None, W, Hq, Hkv, D, norm="layernorm", eps=eps)
        assert e.value.status == 1, eps


@pytest.mark.parametrize("M", [32, 300])
def test_residual_projection_in_place(handle, M):
    """out may be the residual buffer itself (the residual stream updated in
    place); the result matches the oracle on the original residual."""
    w, inputs = synthetic.make_custom("residual", "none", M, 4096, N=4096, bias_out=True, seed=21)
    dev = {k: v.cuda() for k, v in inputs.items()}
    stream_buf = dev["residual"].clone()
    got = fnl.linear_add_residual(handle, dev["x"], dev["W"], stream_buf, bias=dev["bias_out"], out=stream_buf)
    handle.check()
    assert got["out"].data_ptr() == stream_buf.data_ptr()
    print(check(w, inputs, got))


def test_residual_projection_alias_errors(handle):
    bf = dict(dtype=torch.bfloat16, device="cuda")
    M, K, N = 8, 64, 64
    a, W = torch.randn(M, K, **bf), torch.randn(N, K, **bf)
    buf = torch.randn(2 * M * N, **bf)
    res = buf[: M * N].view(M, N)
    with pytest.raises(fnl.FnlError) as e:   # out partly overlaps residual
        fnl.linear_add_residual(handle, a, W, res, out=buf[8: 8 + M * N].view(M, N))
    assert e.value.status == 3
    with pytest.raises(fnl.FnlError) as e:   # out overlaps a
        fnl.linear_add_residual(handle, a, W, torch.randn(M, N, **bf), out=a)
    assert e.value.status == 3
    handle.check()


@pytest.mark.parametrize("name", ["c1_tiny_ln_qkv", "c2_decode_rms_qkv", "c5_70b_rms_qkv_m256",
                                  "llama3_8b_o_proj_decode"])
def test_tuner(cuda_device, name):
    """Shape auto-tuning: the first call times the candidate plans and keeps the
    fastest (its result matches the oracle), the second call of the same shape
    takes the cached plan without re-timing, and matches the oracle too."""
    w = WL[name]
    inputs = synthetic.make_inputs(w)
    dev = {k: v.cuda() for k, v in inputs.items()}
    h = fnl.Handle(0, tune=True)
    got = fnl.run_workload(h, w, dev)
    h.check()
    first = h.last_plan()
    assert "tuned:" in first, first
    check(w, inputs, got)
    got = fnl.run_workload(h, w, dev)
    h.check()
    second = h.last_plan()
    assert "from the cache" in second, second
    assert first.split(" (")[0] == second.split(" (")[0]
    check(w, inputs, got)
    print(name, first)
    h.close()


@pytest.mark.parametrize("name", ["c3_prefill_rms_swiglu", "c4_gpt_ln_gelu", "c5_70b_rms_qkv_m2048",
                                  "llama3_8b_down_proj_prefill"])
def test_pair_kernel_full_size(cuda_device, name):
    """The CTA-pair kernel forced on the large workloads (sampled rows, every
    row's residual_out and statistics)."""
    w = WL[name]
    h = fnl.Handle(0, path="pair")
    inputs = synthetic.make_inputs(w)
    res, _ = run_and_check(h, w, inputs, rows=sample_rows(w.M, w.seq_lens))
    print(name, h.last_plan(), res)
    h.close()


@pytest.mark.parametrize("M", [129, 255, 256, 257, 600])
@pytest.mark.parametrize("op,norm", [("qkv", "rmsnorm"), ("swiglu", "layernorm"), ("gelu", "layernorm"),
                                     ("residual", "none")])
def test_pair_kernel_row_tails(cuda_device, M, op, norm):
    """Pair tiles cut by M: the odd CTA's rows partly or wholly past M."""
    h = fnl.Handle(0, path="pair")
    w, inputs = _tail_workload(op, norm, M, K=328, seed=M)
    run_and_check(h, w, inputs)
    h.close()


# Pair kernel, stream-K form (forced): few tiles for the 74 pairs, so the (tile,
# k-block) units are dealt over all pairs and the fix-up kernel sums each tile
# from several pairs' partial sums (K not a multiple of the 32-wide k-block in
# two cases); every epilogue with each norm.
STREAM_K_CASES = [
    ("qkv", "rmsnorm", 300, 2048, dict(Hq=6, Hkv=2, D=128, bias_out=True)),
    ("qkv", "layernorm", 513, 2000, dict(Hq=4, Hkv=2, D=128)),
    ("swiglu", "rmsnorm", 260, 1536, dict(I=600, bias_out=True)),
    ("swiglu", "layernorm", 256, 4096, dict(I=256)),   # one tile over every pair
    ("gelu", "layernorm", 256, 2600, dict(N=1000, bias_in=True, bias_out=True)),
    ("gelu", "rmsnorm", 300, 1024, dict(N=1000, bias_out=True)),
    ("residual", "none", 384, 2048, dict(N=704, bias_out=True)),
]


@pytest.mark.parametrize("op,norm,M,K,kw", STREAM_K_CASES)
def test_pair_kernel_stream_k(cuda_device, op, norm, M, K, kw):
    h = fnl.Handle(0, path="pair_sk")
    w, inputs = synthetic.make_custom(op, norm, M, K, seed=M + K, **kw)
    _, got = run_and_check(h, w, inputs)
    assert "stream-K" in h.last_plan(), h.last_plan()
    # the slot-order sum makes the result independent of which pair finishes first
    _, again = run_and_check(h, w, inputs)
    for k, v in got.items():
        if v is not None:
            assert torch.equal(v, again[k]), k
    h.close()


def test_pair_kernel_stream_k_without_split_tiles(cuda_device):
    """The stream-K form forced on 74 tiles (37 row pairs x 2 column tiles):
    whole waves only on a B200's 74 resident pairs, so nothing is split and the
    plan is the plain form (no fix-up launch); every element against the oracle."""
    h = fnl.Handle(0, path="pair_sk")
    w, inputs = synthetic.make_custom("qkv", "rmsnorm", 37 * 256, 256, Hq=6, Hkv=1, D=128, bias_out=True, seed=9)
    run_and_check(h, w, inputs)
    h.close()


@pytest.mark.parametrize("kind", ["whole tiles", "stream-K", "whole waves + stream-K"])
def test_pair_kernel_repeat_full_compare(cuda_device, kind):
    """Every row against the oracle, and bitwise-equal repeats, with the
    activation tiles resident in L2 (copies land fast, so a ring slot released
    too early would be overwritten before its reads): 72 pair tiles for 74
    pairs (whole tiles), the 70B QKV at M = 256 (20 tiles, all split), and 80
    tiles (one whole wave of 74, the other 6 split)."""
    if kind == "whole tiles":
        w, inputs = synthetic.make_custom("qkv", "rmsnorm", 2304, 1024, Hq=24, Hkv=4, D=128, seed=11)
    elif kind == "stream-K":
        w = WL["c5_70b_rms_qkv_m256"]
        inputs = synthetic.make_inputs(w)
    else:
        w, inputs = synthetic.make_custom("qkv", "rmsnorm", 2560, 1024, Hq=24, Hkv=4, D=128, seed=12)
    h = fnl.Handle(0, path="pair" if kind == "whole tiles" else "pair_sk")
    _, first = run_and_check(h, w, inputs)
    assert ("stream-K" in h.last_plan()) == (kind != "whole tiles"), h.last_plan()
    dev = {k: v.cuda() for k, v in inputs.items()}
    for _ in range(3):
        again = fnl.run_workload(h, w, dev)
        h.check()
        for k in ("q", "k", "v"):
            assert torch.equal(first[k], again[k]), k
    h.close()
