"""Pins of the fp64 CPU oracle to things other than itself.

Each pin checks the oracle against an invariant, a closed form, a library
routine on a special case, or a brute-force loop on tiny inputs. The mutation
tests at the bottom plant plausible mistakes in the oracle (on the CPU, by
monkeypatching one function at a time) and require that at least one pin
fails for every planted mistake.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import core


def _rand(shape, seed, scale=1.0, loc=0.0):
    return np.random.default_rng(seed).normal(loc, scale, size=shape)


def _t(a):
    return torch.tensor(np.asarray(a, dtype=np.float64))


# --------------------------------------------------------------------------
# pins: each takes the oracle module so that the mutation tests can reuse them
# --------------------------------------------------------------------------

def pin_layernorm_invariants(ora):
    """gamma=1, beta=0: every row of a has mean 0 and population variance
    var/(var+eps); the returned statistics match numpy's mean and variance."""
    K = 96
    h = _rand((16, K), 1, scale=1.7, loc=0.3)
    eps = 0.05
    a, mean, rstd = ora.layernorm(h, np.ones(K), np.zeros(K), eps)
    var = np.var(h, axis=1)
    assert np.max(np.abs(a.mean(axis=1))) <= 1e-12
    np.testing.assert_allclose(np.var(a, axis=1), var / (var + eps), rtol=1e-12, atol=0)
    np.testing.assert_allclose(mean, np.mean(h, axis=1), rtol=0, atol=1e-13)
    np.testing.assert_allclose(rstd ** -2 - eps, var, rtol=1e-12)


def pin_rmsnorm_invariant(ora):
    """gamma=1: mean(a^2) = ms/(ms+eps) with ms = mean(h^2) (rows with a
    non-zero mean, so a centred variant fails)."""
    K = 96
    h = _rand((16, K), 2, scale=1.3, loc=0.4)
    eps = 0.05
    a, rstd = ora.rmsnorm(h, np.ones(K), eps)
    ms = np.mean(h * h, axis=1)
    np.testing.assert_allclose(np.mean(a * a, axis=1), ms / (ms + eps), rtol=1e-12)
    np.testing.assert_allclose(rstd ** -2 - eps, ms, rtol=1e-12)


def pin_norms_match_torch(ora):
    """Special case = library routine: torch's float64 layer_norm / rms_norm."""
    K = 64
    h = _rand((8, K), 3, scale=2.0, loc=-0.5)
    g = _rand(K, 4, 0.1, 1.0)
    b = _rand(K, 5, 0.1)
    for eps in (1e-5, 0.3):
        a, _, _ = ora.layernorm(h, g, b, eps)
        ref = F.layer_norm(_t(h), (K,), _t(g), _t(b), eps).numpy()
        assert np.max(np.abs(a - ref)) <= 1e-12
        a2, _ = ora.rmsnorm(h, g, eps)
        ref2 = F.rms_norm(_t(h), (K,), _t(g), eps).numpy()
        assert np.max(np.abs(a2 - ref2)) <= 1e-12


def pin_identity_weight(ora):
    """W = identity (N = K): QKV is a re-indexing of the normalised rows,
    SwiGLU with W = [I; 2I] is SiLU(a) * 2a, GELU with W = I is GELU(a + b)."""
    Hq, Hkv, D = 2, 1, 8
    K = (Hq + 2 * Hkv) * D
    M = 5
    x, r = _rand((M, K), 6), _rand((M, K), 7)
    g, b = _rand(K, 8, 0.1, 1.0), _rand(K, 9, 0.1)
    eps = 1e-5
    a = F.layer_norm(_t(x) + _t(r), (K,), _t(g), _t(b), eps).numpy()
    out = ora.add_norm_qkv(x, r, g, b, "layernorm", eps, np.eye(K), None, Hq, Hkv, D)
    assert out["q"].shape == (Hq, M, D) and out["k"].shape == (Hkv, M, D)
    assert out["v"].shape == (Hkv, M, D)
    for m in range(M):
        for d in range(D):
            for hh in range(Hq):
                assert abs(out["q"][hh, m, d] - a[m, hh * D + d]) <= 1e-12
            for hh in range(Hkv):
                assert abs(out["k"][hh, m, d] - a[m, (Hq + hh) * D + d]) <= 1e-12
                assert abs(out["v"][hh, m, d] - a[m, (Hq + Hkv + hh) * D + d]) <= 1e-12

    W2 = np.concatenate([np.eye(K), 2.0 * np.eye(K)], axis=0)
    ar = F.rms_norm(_t(x) + _t(r), (K,), _t(g), eps)
    sw = ora.add_norm_swiglu(x, r, g, None, "rmsnorm", eps, W2, None, K)["out"]
    ref = (F.silu(ar) * 2.0 * ar).numpy()
    assert np.max(np.abs(sw - ref)) <= 1e-12

    bi, bo = _rand(K, 10), _rand(K, 11, 0.02)
    al = F.layer_norm(_t(x) + _t(r) + _t(bi), (K,), _t(g), _t(b), eps)
    ge = ora.add_bias_norm_gelu(x, r, bi, g, b, "layernorm", eps, np.eye(K), bo)["out"]
    ref = F.gelu(al + _t(bo), approximate="tanh").numpy()
    assert np.max(np.abs(ge - ref)) <= 1e-12


def pin_one_hot(ora):
    """h = s * e_j (x = s e_j - t e_i, residual = t e_i): closed forms.
    LayerNorm: a_k = gamma_k (delta_kj - 1/K) s rstd + beta_k with
    rstd = (s^2 (K-1)/K^2 + eps)^(-1/2). RMSNorm: y_n = W[n, j] gamma_j s /
    sqrt(s^2/K + eps), which exposes the index order of the projection."""
    K, N = 48, 24
    j, i, s, t = 7, 30, 3.0, 1.25
    x = np.zeros((1, K))
    r = np.zeros((1, K))
    x[0, j], x[0, i], r[0, i] = s, -t, t
    g, b = _rand(K, 12, 0.1, 1.0), _rand(K, 13, 0.1)
    W = _rand((N, K), 14)
    eps = 1e-3
    a, mean, rstd = ora.layernorm(ora.residual_add(x, r), g, b, eps)
    rs = (s * s * (K - 1) / K ** 2 + eps) ** -0.5
    ak = g * ((np.arange(K) == j) - 1.0 / K) * s * rs + b
    assert abs(mean[0] - s / K) <= 1e-15
    assert abs(rstd[0] - rs) <= 1e-12 * rs
    assert np.max(np.abs(a[0] - ak)) <= 1e-12
    # RMS through the whole QKV path: N = (Hq + 2 Hkv) D with Hq=2, Hkv=1, D=6
    out = ora.add_norm_qkv(x, r, g, None, "rmsnorm", eps, W, None, 2, 1, 6)
    yn = W[:, j] * g[j] * s / math.sqrt(s * s / K + eps)
    y = np.concatenate([out["q"][:, 0, :].reshape(-1), out["k"][:, 0, :].reshape(-1),
                        out["v"][:, 0, :].reshape(-1)])
    assert np.max(np.abs(y - yn)) <= 1e-12


def _brute(op, x, r, bias_in, g, b, norm, eps, W, bias_out, Hq=0, Hkv=0, D=0, I=0):
    """Per-element loops, independent of the vectorised oracle."""
    M, K = len(x), len(x[0])
    N = len(W)
    res = {"rows": []}
    for m in range(M):
        h = [x[m][k] + r[m][k] + (bias_in[k] if bias_in is not None else 0.0) for k in range(K)]
        if norm == "layernorm":
            mu = 0.0
            for k in range(K):
                mu += h[k]
            mu /= K
            var = 0.0
            for k in range(K):
                var += (h[k] - mu) * (h[k] - mu)
            var /= K
            rs = 1.0 / math.sqrt(var + eps)
            a = [g[k] * (h[k] - mu) * rs + (b[k] if b is not None else 0.0) for k in range(K)]
        else:
            ss = 0.0
            for k in range(K):
                ss += h[k] * h[k]
            rs = 1.0 / math.sqrt(ss / K + eps)
            a = [h[k] * rs * g[k] for k in range(K)]
        y = []
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += a[k] * W[n][k]
            if bias_out is not None:
                acc += bias_out[n]
            y.append(acc)
        res["rows"].append(y)
    return res


def pin_brute_force(ora):
    """Tiny shapes against per-element loops, all three epilogues."""
    M, K = 3, 16
    x, r = _rand((M, K), 20), _rand((M, K), 21)
    g, b, bi = _rand(K, 22, 0.1, 1.0), _rand(K, 23, 0.1), _rand(K, 24)
    eps = 1e-5
    # QKV, LayerNorm, with bias
    Hq, Hkv, D = 2, 1, 4
    N = (Hq + 2 * Hkv) * D
    W, bo = _rand((N, K), 25, 0.25), _rand(N, 26, 0.02)
    out = ora.add_norm_qkv(x, r, g, b, "layernorm", eps, W, bo, Hq, Hkv, D)
    y = _brute("qkv", x.tolist(), r.tolist(), None, g, b, "layernorm", eps, W.tolist(), bo)["rows"]
    for m in range(M):
        for n in range(N):
            if n < Hq * D:
                got = out["q"][n // D, m, n % D]
            elif n < (Hq + Hkv) * D:
                got = out["k"][(n - Hq * D) // D, m, n % D]
            else:
                got = out["v"][(n - (Hq + Hkv) * D) // D, m, n % D]
            assert abs(got - y[m][n]) <= 1e-12
    # SwiGLU, RMSNorm
    I = 5
    W = _rand((2 * I, K), 27, 0.25)
    out = ora.add_norm_swiglu(x, r, g, None, "rmsnorm", eps, W, None, I)["out"]
    y = _brute("swiglu", x.tolist(), r.tolist(), None, g, None, "rmsnorm", eps, W.tolist(), None)["rows"]
    for m in range(M):
        for j in range(I):
            gate, up = y[m][j], y[m][I + j]
            assert abs(out[m, j] - gate / (1.0 + math.exp(-gate)) * up) <= 1e-12
    # Bias + LayerNorm + GELU
    N = 6
    W, bo = _rand((N, K), 28, 0.25), _rand(N, 29, 0.02)
    out = ora.add_bias_norm_gelu(x, r, bi, g, b, "layernorm", eps, W, bo)
    y = _brute("gelu", x.tolist(), r.tolist(), bi, g, b, "layernorm", eps, W.tolist(), bo)["rows"]
    c = math.sqrt(2.0 / math.pi)
    for m in range(M):
        for n in range(N):
            z = y[m][n]
            ref = 0.5 * z * (1.0 + math.tanh(c * (z + 0.044715 * z ** 3)))
            assert abs(out["out"][m, n] - ref) <= 1e-12
    for m in range(M):
        h = x[m] + r[m] + bi
        assert np.all(out["residual_out"][m] == ora.bf16_round(h))


def pin_epilogue_values(ora):
    """SiLU / GELU_tanh: hand values, limits, torch float64, erf-GELU within 1e-3."""
    assert float(ora.silu(0.0)) == 0.0 and float(ora.gelu_tanh(0.0)) == 0.0
    assert abs(float(ora.silu(40.0)) - 40.0) <= 1e-12
    assert abs(float(ora.silu(-40.0)) - (-40.0 * math.exp(-40.0))) <= 1e-25
    assert abs(float(ora.gelu_tanh(10.0)) - 10.0) <= 1e-12
    # gelu_tanh(1) = 0.5 (1 + tanh(sqrt(2/pi) * 1.044715))
    assert abs(float(ora.gelu_tanh(1.0)) - 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * 1.044715))) <= 1e-15
    z = np.linspace(-8.0, 8.0, 321)
    assert np.max(np.abs(ora.silu(z) - F.silu(_t(z)).numpy())) <= 1e-14
    assert np.max(np.abs(ora.gelu_tanh(z) - F.gelu(_t(z), approximate="tanh").numpy())) <= 1e-14
    erf_gelu = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in z])
    assert np.max(np.abs(ora.gelu_tanh(z) - erf_gelu)) <= 1e-3
    y = np.stack([z, -z[::-1] * 0.5], axis=1)
    sw = ora.swiglu(np.concatenate([y[:, :1], y[:, 1:]], axis=1), 1)[:, 0]
    assert np.max(np.abs(sw - F.silu(_t(z)).numpy() * (-z[::-1] * 0.5))) <= 1e-14


def pin_qkv_bijection(ora):
    """Unique ids through the split: each lands exactly once, at Q[h,m,d] =
    y[m, h*D + d] and likewise for K and V after the Q block."""
    M, Hq, Hkv, D = 3, 4, 2, 5
    N = (Hq + 2 * Hkv) * D
    y = np.arange(M * N, dtype=np.float64).reshape(M, N)
    q, k, v = ora.split_qkv_head_major(y, Hq, Hkv, D)
    assert q.shape == (Hq, M, D) and k.shape == (Hkv, M, D) and v.shape == (Hkv, M, D)
    ids = np.sort(np.concatenate([q.ravel(), k.ravel(), v.ravel()]))
    assert np.array_equal(ids, np.arange(M * N, dtype=np.float64))
    for m in range(M):
        for d in range(D):
            for h in range(Hq):
                assert q[h, m, d] == m * N + h * D + d
            for h in range(Hkv):
                assert k[h, m, d] == m * N + (Hq + h) * D + d
                assert v[h, m, d] == m * N + (Hq + Hkv + h) * D + d


def pin_bf16_round(ora):
    """Ties go to even; values representable in fp32 round as torch's
    single-rounding fp32 -> bf16 conversion does."""
    e = 2.0 ** -8
    cases = {1 + e: 1.0, 1 + 3 * e: 1 + 2 ** -6, 1 + e + 2 ** -30: 1 + 2 ** -7,
             -(1 + e): -1.0, 2 * (1 + 3 * e): 2 * (1 + 2 ** -6), 0.0: 0.0}
    for v, want in cases.items():
        assert float(ora.bf16_round(np.array([v]))[0]) == want, v
    v = torch.randn(4096, generator=torch.Generator().manual_seed(3), dtype=torch.float32) * 7
    ref = v.to(torch.bfloat16).double().numpy()
    assert np.array_equal(ora.bf16_round(v.double().numpy()), ref)


def pin_residual_out(ora):
    """residual_out: x when residual = 0, 2x when residual = x (exact in bf16),
    and torch's fp32 -> bf16 rounding of x + r wherever the fp32 sum is exact."""
    g = torch.Generator().manual_seed(5)
    xb = torch.randn(4, 64, generator=g).to(torch.bfloat16)
    rb = torch.randn(4, 64, generator=g).to(torch.bfloat16)
    x, r = xb.double().numpy(), rb.double().numpy()
    K = 64
    gam = np.ones(K)
    o = ora.add_norm_swiglu(x, np.zeros_like(x), gam, None, "rmsnorm", 1e-5, np.ones((2, K)), None, 1)
    assert np.array_equal(o["residual_out"], x)
    o = ora.add_norm_swiglu(x, x, gam, None, "rmsnorm", 1e-5, np.ones((2, K)), None, 1)
    assert np.array_equal(o["residual_out"], 2 * x)
    o = ora.add_norm_swiglu(x, r, gam, None, "rmsnorm", 1e-5, np.ones((2, K)), None, 1)
    s32 = (xb.float() + rb.float())
    exact = s32.double().numpy() == x + r
    assert exact.mean() > 0.9
    assert np.array_equal(o["residual_out"][exact], s32.to(torch.bfloat16).double().numpy()[exact])


def pin_run_maps_workload_inputs(ora):
    """run(): the workload's tensors reach the right arguments. Every optional
    vector present (beta, bias_in, bias_out), an unsorted non-contiguous row
    subset, and the expected values from the per-element loops on the rows
    picked by hand, for all three epilogues and both norms."""
    import synthetic
    rows = np.array([5, 0, 3, 6], dtype=np.int64)
    cases = [synthetic.make_custom("qkv", "layernorm", 7, 16, Hq=2, Hkv=1, D=4, bias_out=True, seed=40),
             synthetic.make_custom("qkv", "rmsnorm", 7, 16, Hq=2, Hkv=1, D=4, bias_out=True, seed=41),
             synthetic.make_custom("swiglu", "layernorm", 7, 16, I=5, bias_out=True, seed=42),
             synthetic.make_custom("gelu", "layernorm", 7, 16, N=6, bias_in=True, bias_out=True, seed=43),
             synthetic.make_custom("gelu", "rmsnorm", 7, 16, N=6, bias_in=True, bias_out=True, seed=44)]
    for w, inputs in cases:
        f = {k: v.double().numpy() for k, v in inputs.items()}
        beta = f.get("beta")
        got = ora.run(w, inputs, rows=rows)
        ref = _brute(w.op, f["x"][rows].tolist(), f["residual"][rows].tolist(), f.get("bias_in"), f["gamma"],
                     beta, w.norm, w.eps, f["W"].tolist(), f.get("bias_out"))["rows"]
        for i, m in enumerate(rows):
            h = f["x"][m] + f["residual"][m] + (f["bias_in"] if "bias_in" in f else 0.0)
            assert np.array_equal(got["residual_out"][i], ora.bf16_round(h))
            if w.norm == "layernorm":
                assert abs(got["mean"][i] - h.mean()) <= 1e-13
                assert abs(got["rstd"][i] - 1.0 / math.sqrt(np.var(h) + w.eps)) <= 1e-12 * got["rstd"][i]
            else:
                assert abs(got["rstd"][i] - 1.0 / math.sqrt(np.mean(h * h) + w.eps)) <= 1e-12 * got["rstd"][i]
            y = ref[i]
            if w.op == "qkv":
                D = w.D
                for n in range(w.N):
                    if n < w.Hq * D:
                        g = got["q"][n // D, i, n % D]
                    elif n < (w.Hq + w.Hkv) * D:
                        g = got["k"][(n - w.Hq * D) // D, i, n % D]
                    else:
                        g = got["v"][(n - (w.Hq + w.Hkv) * D) // D, i, n % D]
                    assert abs(g - y[n]) <= 1e-12
            elif w.op == "swiglu":
                for j in range(w.I):
                    gate, up = y[j], y[w.I + j]
                    assert abs(got["out"][i, j] - gate / (1.0 + math.exp(-gate)) * up) <= 1e-12
            else:
                c = math.sqrt(2.0 / math.pi)
                for n in range(w.N):
                    z = y[n]
                    assert abs(got["out"][i, n] - 0.5 * z * (1.0 + math.tanh(c * (z + 0.044715 * z ** 3)))) <= 1e-12


def pin_residual_projection(ora):
    """out = residual + a W^T + bias: identity W gives residual + a + bias;
    a one-hot row a = s e_j gives residual[n] + s W[n, j] + bias[n] (exposes
    W's index order); per-element loops on a tiny non-square shape; run() maps
    the workload's tensors (a under "x", the [M, N] residual) on a row subset."""
    M, K = 4, 12
    a, res, bias = _rand((M, K), 60), _rand((M, K), 61), _rand(K, 62, 0.02)
    out = ora.linear_add_residual(a, np.eye(K), bias, res)["out"]
    assert np.max(np.abs(out - (res + a + bias[None, :]))) <= 1e-15
    N, j, sc = 7, 5, 2.5
    W = _rand((N, K), 63)
    oh = np.zeros((1, K))
    oh[0, j] = sc
    Wsq = _rand((K, K), 69)   # square: a transposed W would still have the right shape
    out = ora.linear_add_residual(oh, Wsq, None, np.zeros((1, K)))["out"]
    assert np.max(np.abs(out[0] - sc * Wsq[:, j])) <= 1e-14
    r1 = _rand((1, N), 64)
    out = ora.linear_add_residual(oh, W, None, r1)["out"]
    assert np.max(np.abs(out[0] - (r1[0] + sc * W[:, j]))) <= 1e-14
    a, res, b = _rand((3, K), 65), _rand((3, N), 66), _rand(N, 67, 0.02)
    out = ora.linear_add_residual(a, W, b, res)["out"]
    for m in range(3):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += a[m, k] * W[n, k]
            assert abs(out[m, n] - (res[m, n] + acc + b[n])) <= 1e-12
    import synthetic
    w, inputs = synthetic.make_custom("residual", "none", 6, 16, N=24, bias_out=True, seed=68)
    rows = np.array([4, 1, 2], dtype=np.int64)
    f = {k: v.double().numpy() for k, v in inputs.items()}
    got = ora.run(w, inputs, rows=rows)["out"]
    for i, m in enumerate(rows):
        for n in range(24):
            acc = sum(f["x"][m, k] * f["W"][n, k] for k in range(16))
            assert abs(got[i, n] - (f["residual"][m, n] + acc + f["bias_out"][n])) <= 1e-12


def _e4m3_values():
    """All finite e4m3 values, from the format's definition: sign, 4 exponent
    bits (bias 7), 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6);
    exponent 15 with mantissa 7 is NaN."""
    vals = set()
    for sign in (1.0, -1.0):
        for e in range(16):
            for m in range(8):
                if e == 15 and m == 7:
                    continue
                v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
                vals.add(sign * v)
    return np.array(sorted(vals))


def pin_e4m3_format(ora):
    """e4m3 rounding: every finite value of the format rounds to itself, the
    largest is 448, midpoints go to the even mantissa, values past 448
    saturate, and torch's float8_e4m3fn conversion agrees on +-448."""
    vals = _e4m3_values()
    assert len(vals) == 253 and vals.max() == 448.0   # +0 and -0 are one value
    assert np.array_equal(ora.e4m3_round(vals), vals)
    pos = vals[vals > 0]
    mids = (pos[:-1] + pos[1:]) / 2
    got = ora.e4m3_round(mids)
    # the even neighbour: mantissa field even (bit pattern of the value's code)
    def mant(v):
        if v < 2.0 ** -6:
            return int(round(v / 2.0 ** -9))
        e = math.floor(math.log2(v))
        return int(round((v / 2.0 ** e - 1.0) * 8))
    for g, lo, hi in zip(got, pos[:-1], pos[1:]):
        assert g in (lo, hi)
        assert mant(g) % 2 == 0, (lo, hi, g)
    assert np.array_equal(ora.e4m3_round(np.array([460.0, 1e6, -1e9])), np.array([448.0, 448.0, -448.0]))
    rng = np.random.default_rng(70)
    v = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 0.02, 20000), mids, -mids])
    ref = torch.tensor(v).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(ora.e4m3_round(v), ref)


def pin_fp8_quantisers(ora):
    """Per-row FP8 quantisation: the row's largest magnitude maps to exactly
    +-448, scale = amax / 448 in fp32, the error is within half a step
    (2^-4 relative for normals, 2^-10 s below 2^-6 s), signs are symmetric,
    a power-of-two row scaling moves only the scale, a zero row has scale 1."""
    rng = np.random.default_rng(71)
    W = rng.normal(0, 0.02, (6, 64))
    W[3] = 0.0
    q, s_ = ora.quantize_weight_fp8(W)
    assert s_.dtype == np.float32 and s_[3] == 1.0 and np.all(q[3] == 0)
    for n in (0, 1, 2, 4, 5):
        j = int(np.argmax(np.abs(W[n])))
        assert abs(q[n, j]) == 448.0 and np.sign(q[n, j]) == np.sign(W[n, j])
        assert s_[n] == np.float32(np.float32(abs(W[n, j])) / np.float32(448.0))
        err = np.abs(W[n] - q[n] * np.float64(s_[n]))
        assert np.all(err <= 2.0 ** -4 * np.abs(W[n]) + 2.0 ** -10 * np.float64(s_[n]) + 1e-12)
    q2, s2 = ora.quantize_weight_fp8(-W)
    assert np.array_equal(q2, -q) and np.array_equal(s2, s_)
    q3, s3 = ora.quantize_weight_fp8(W * 8.0)
    assert np.array_equal(q3, q) and np.array_equal(s3[[0, 1, 2, 4, 5]], 8 * s_[[0, 1, 2, 4, 5]])


def pin_fp8_linear(ora):
    """W8A8 projection: a one-hot activation row gives y_n = c W~[n, j]
    (W~ = codes * s_w), per-element loops over the codes on a tiny case, and
    the result stays within the quantisation error bound of the exact
    product."""
    rng = np.random.default_rng(72)
    K, N = 32, 12
    W = rng.normal(0, 0.2, (N, K))
    Wq, sw = ora.quantize_weight_fp8(W)
    Wd = Wq * sw.astype(np.float64)[:, None]
    a = np.zeros((1, K))
    a[0, 5] = -2.5
    y = ora.fp8_linear(a, Wq, sw)
    # exact but for the fp32 rounding of s_a = 2.5 / 448 (relative 2^-24)
    assert np.max(np.abs(y[0] - (-2.5) * Wd[:, 5])) <= 2.0 ** -23 * np.max(np.abs(2.5 * Wd[:, 5]))
    a = rng.normal(0, 1, (3, K)).astype(np.float32)
    b = rng.normal(0, 0.02, N)
    y = ora.fp8_linear(a, Wq, sw, b)
    qa, sa = ora.fp8_activation_codes(a)
    for m in range(3):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += qa[m, k] * Wq[n, k]
            assert abs(y[m, n] - (acc * float(sa[m]) * float(sw[n]) + b[n])) <= 1e-12 * (1 + abs(y[m, n]))
    exact = a.astype(np.float64) @ Wd.T + b
    bound = (2.0 ** -4 * np.abs(a) + 2.0 ** -10 * sa.astype(np.float64)[:, None]) @ np.abs(Wd).T + 1e-6
    assert np.all(np.abs(y - exact) <= bound)


def pin_fp8_activation_codes(ora):
    """Per-token activation codes: the row's amax element maps to +-448, every
    code is within half a step of a * 448 / amax, s_a * 448 recovers amax,
    a zero row gives zero codes and scale 1; the fp32 normalisation used for the
    decision is the fp64 normalisation within two fp32 rounding steps."""
    rng = np.random.default_rng(74)
    a = rng.normal(0, 1.5, (5, 96)).astype(np.float32)
    a[2] = 0.0
    q, s_ = ora.fp8_activation_codes(a)
    assert s_[2] == 1.0 and np.all(q[2] == 0)
    for m in (0, 1, 3, 4):
        j = int(np.argmax(np.abs(a[m])))
        assert abs(q[m, j]) == 448.0
        amax = float(np.abs(a[m]).max())
        assert abs(float(s_[m]) * 448.0 - amax) <= 2.0 ** -23 * amax
        v = a[m].astype(np.float64) * 448.0 / amax
        step = np.where(np.abs(v) < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(v), 1e-30))) - 3))
        assert np.all(np.abs(q[m] - v) <= 0.5 * step * (1 + 1e-6))
    h = rng.normal(0, 1, (4, 64))
    g, be = 1 + 0.1 * rng.normal(size=64), 0.1 * rng.normal(size=64)
    a64, mean, rstd = ora.layernorm(h, g, be, 1e-5)
    a32 = ora.fp8_normalised32(h.astype(np.float32), mean, rstd, g, be)
    assert a32.dtype == np.float32
    # h rounded to fp32 first (as the kernel holds it), then the fp32 steps
    assert np.all(np.abs(a32 - a64) <= 2.0 ** -20 * (np.abs(a64) + np.abs(be)[None, :] + 1))
    r64, rs = ora.rmsnorm(h, g, 1e-5)
    r32 = ora.fp8_normalised32(h.astype(np.float32), None, rs, g, None)
    assert np.all(np.abs(r32 - r64) <= 2.0 ** -20 * (np.abs(r64) + 1))


def pin_fp8_fused_qkv(ora):
    """The FP8 fused QKV op: one-hot x (RMSNorm) gives y_n = W~[n, j] gamma_j s /
    sqrt(s^2/K + eps); residual_out and the statistics are those of the bf16 op."""
    Hq, Hkv, D = 2, 1, 4
    N, K = (Hq + 2 * Hkv) * D, 24
    j, sc, eps = 9, 3.0, 1e-3
    rng = np.random.default_rng(73)
    g = 1.0 + 0.1 * rng.normal(size=K)
    Wq, sw = ora.quantize_weight_fp8(rng.normal(0, 0.2, (N, K)))
    Wd = Wq * sw.astype(np.float64)[:, None]
    x = np.zeros((1, K))
    x[0, j] = sc
    out = ora.add_norm_qkv_fp8(x, np.zeros((1, K)), g, None, "rmsnorm", eps, Wq, sw, None, Hq, Hkv, D)
    y = np.concatenate([out["q"][:, 0, :].reshape(-1), out["k"][:, 0, :].reshape(-1), out["v"][:, 0, :].reshape(-1)])
    ref = Wd[:, j] * g[j] * sc / math.sqrt(sc * sc / K + eps)
    assert np.max(np.abs(y - ref)) <= 1e-6 * np.max(np.abs(ref))
    xr, rr = rng.normal(size=(3, K)), rng.normal(size=(3, K))
    o8 = ora.add_norm_qkv_fp8(xr, rr, g, None, "layernorm", 1e-5, Wq, sw, None, Hq, Hkv, D)
    o16 = ora.add_norm_qkv(xr, rr, g, None, "layernorm", 1e-5, Wd, None, Hq, Hkv, D)
    for key in ("residual_out", "mean", "rstd"):
        assert np.array_equal(o8[key], o16[key])
    # SwiGLU: one-hot x, W = [gate; up] quantised per row: out = SiLU(y_g) y_u with
    # y = W~[:, j] gamma_j s rstd
    I = 5
    Wsw = rng.normal(0, 0.2, (2 * I, K))
    Wq2, sw2 = ora.quantize_weight_fp8(Wsw)
    Wd2 = Wq2 * sw2.astype(np.float64)[:, None]
    o = ora.add_norm_swiglu_fp8(x, np.zeros((1, K)), g, None, "rmsnorm", eps, Wq2, sw2, None, I)["out"][0]
    yv = Wd2[:, j] * g[j] * sc / math.sqrt(sc * sc / K + eps)
    ref = yv[:I] / (1 + np.exp(-yv[:I])) * yv[I:]
    assert np.max(np.abs(o - ref)) <= 1e-6 * (1 + np.max(np.abs(ref)))
    # Bias + GELU: bias_in enters h (and the codes), bias_out is added before GELU
    bi, bo = rng.normal(size=K), 0.02 * rng.normal(size=N)
    og = ora.add_bias_norm_gelu_fp8(xr, rr, bi, g, None, "layernorm", 1e-5, Wq, sw, bo)
    y_ln = ora.fp8_linear(ora.fp8_normalised32(ora.fp8_h32(xr, rr, bi), og["mean"], og["rstd"], g, None), Wq, sw, bo)
    assert np.max(np.abs(og["out"] - ora.gelu_tanh(y_ln))) <= 1e-12
    assert np.array_equal(og["residual_out"], ora.bf16_round(xr + rr + bi[None, :]))


def pin_tp_allreduce(ora):
    """Tensor-parallel all-reduce (reading R13): integer partials sum exactly;
    one rank is the identity; the sum is rounded once (ties to even) after an
    exact sum, not after each addition; a row-parallel projection split over
    ranks all-reduces to the unsplit one; the composed QKV op on a one-hot row
    split over two ranks has the RMSNorm closed form."""
    rng = np.random.default_rng(91)
    parts = [rng.integers(-20, 21, size=(3, 8)).astype(np.float64) for _ in range(4)]
    assert np.array_equal(ora.tp_allreduce(parts), np.sum(parts, axis=0))
    one = ora.bf16_round(rng.normal(size=(2, 5)))
    assert np.array_equal(ora.tp_allreduce([one]), one)
    t = 2.0 ** -8
    assert ora.tp_allreduce([np.array([1.0]), np.array([t])])[0] == 1.0                    # tie -> even
    assert ora.tp_allreduce([np.array([1.0]), np.array([3 * t])])[0] == 1.0 + 2 * 2.0 ** -7   # tie -> even
    assert ora.tp_allreduce([np.array([1.0]), np.array([t]), np.array([t])])[0] == 1.0 + 2.0 ** -7
    assert ora.tp_allreduce([np.array([2.0 ** 30]), np.array([1.0]), np.array([-2.0 ** 30])])[0] == 1.0
    # row-parallel projection: K split over 2 ranks, small integers (exact)
    a = rng.integers(-3, 4, size=(4, 12)).astype(np.float64)
    W = rng.integers(-3, 4, size=(6, 12)).astype(np.float64)
    ranks = [ora.projection(a[:, :5], W[:, :5]), ora.projection(a[:, 5:], W[:, 5:])]
    assert np.array_equal(ora.tp_allreduce(ranks), a @ W.T)
    # the composed QKV op: x = e_j s arrives as two ranks' parts (1 and 2)
    Hq, Hkv, D, K, j, eps = 2, 1, 4, 16, 5, 1e-3
    g = 1.0 + 0.1 * rng.normal(size=K)
    Wq = rng.normal(0, 0.2, ((Hq + 2 * Hkv) * D, K))
    p0, p1 = np.zeros((1, K)), np.zeros((1, K))
    p0[0, j], p1[0, j] = 1.0, 2.0
    out = ora.add_norm_qkv_tp([p0, p1], np.zeros((1, K)), g, None, "rmsnorm", eps, Wq, None, Hq, Hkv, D)
    y = np.concatenate([out["q"][:, 0, :].reshape(-1), out["k"][:, 0, :].reshape(-1), out["v"][:, 0, :].reshape(-1)])
    ref = Wq[:, j] * g[j] * 3.0 / math.sqrt(9.0 / K + eps)
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    assert np.array_equal(out["residual_out"][0], np.where(np.arange(K) == j, 3.0, 0.0))


PINS = [pin_layernorm_invariants, pin_rmsnorm_invariant, pin_norms_match_torch,
        pin_identity_weight, pin_one_hot, pin_brute_force, pin_epilogue_values,
        pin_qkv_bijection, pin_bf16_round, pin_residual_out,
        pin_run_maps_workload_inputs, pin_residual_projection, pin_e4m3_format, pin_fp8_quantisers,
        pin_fp8_linear, pin_fp8_activation_codes, pin_fp8_fused_qkv, pin_tp_allreduce]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin_holds(pin):
    pin(core)


# --------------------------------------------------------------------------
# planted mistakes: every one must break at least one pin
# --------------------------------------------------------------------------

ORIG = {name: getattr(core, name) for name in ("layernorm", "rmsnorm", "split_qkv_head_major", "run",
                                               "e4m3_round", "fp8_row_scale_and_codes", "fp8_activation_codes",
                                               "fp8_linear", "fp8_normalised32", "tp_allreduce")}


def _ln_unbiased(h, gamma, beta, eps):
    h = np.asarray(h, np.float64)
    K = h.shape[1]
    mean = h.sum(1) / K
    var = ((h - mean[:, None]) ** 2).sum(1) / (K - 1)
    rstd = 1 / np.sqrt(var + eps)
    bb = 0 if beta is None else np.asarray(beta)[None]
    return np.asarray(gamma)[None] * (h - mean[:, None]) * rstd[:, None] + bb, mean, rstd


def _ln_eps_outside(h, gamma, beta, eps):
    h = np.asarray(h, np.float64)
    K = h.shape[1]
    mean = h.sum(1) / K
    var = ((h - mean[:, None]) ** 2).sum(1) / K
    rstd = 1 / (np.sqrt(var) + eps)
    bb = 0 if beta is None else np.asarray(beta)[None]
    return np.asarray(gamma)[None] * (h - mean[:, None]) * rstd[:, None] + bb, mean, rstd


def _ln_no_beta(h, gamma, beta, eps):
    return ORIG["layernorm"](h, gamma, None, eps)


def _ln_gamma_before_centering(h, gamma, beta, eps):
    h = np.asarray(h, np.float64)
    K = h.shape[1]
    mean = h.sum(1) / K
    var = ((h - mean[:, None]) ** 2).sum(1) / K
    rstd = 1 / np.sqrt(var + eps)
    bb = 0 if beta is None else np.asarray(beta)[None]
    return (np.asarray(gamma)[None] * h - mean[:, None]) * rstd[:, None] + bb, mean, rstd


def _rms_centred(h, gamma, eps):
    a, _, rstd = ORIG["layernorm"](h, gamma, None, eps)
    return a, rstd


def _rms_no_eps(h, gamma, eps):
    return ORIG["rmsnorm"](h, gamma, 0.0)


def _proj_transposed(a, W, bias=None):
    y = np.asarray(a) @ np.asarray(W)
    return y if bias is None else y + np.asarray(bias)[None]


def _proj_no_bias(a, W, bias=None):
    return np.asarray(a) @ np.asarray(W).T


def _split_kv_swapped(y, Hq, Hkv, D):
    q, k, v = ORIG["split_qkv_head_major"](y, Hq, Hkv, D)
    return q, v, k


def _split_token_major(y, Hq, Hkv, D):
    q, k, v = ORIG["split_qkv_head_major"](y, Hq, Hkv, D)
    return (np.ascontiguousarray(q.transpose(1, 0, 2)), np.ascontiguousarray(k.transpose(1, 0, 2)),
            np.ascontiguousarray(v.transpose(1, 0, 2)))


def _swiglu_swapped(y, I):
    y = np.asarray(y, np.float64)
    return core.silu(y[:, I:2 * I]) * y[:, :I]


def _gelu_wrong_cubic(z):
    z = np.asarray(z, np.float64)
    return 0.5 * z * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (z + 0.0447 * z ** 3)))


def _silu_sigmoid_only(z):
    z = np.asarray(z, np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def _gelu_bias_after(x, residual, bias_in, gamma, beta, norm, eps, W, bias_out):
    h = core.residual_add(x, residual, bias_in)
    a, mean, rstd = core.normalize(h, gamma, beta, norm, eps)
    out = core.gelu_tanh(core.projection(a, W)) + (0 if bias_out is None else np.asarray(bias_out)[None])
    return {"residual_out": core.bf16_round(h), "out": out, "rstd": rstd, "mean": mean}


def _residual_drops_bias_in(x, residual, bias_in=None):
    return np.asarray(x, np.float64) + np.asarray(residual, np.float64)


def _residual_ignores_residual(x, residual, bias_in=None):
    h = np.asarray(x, np.float64)
    return h if bias_in is None else h + np.asarray(bias_in)[None]


def _bf16_truncate(v):
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.trunc(m * 256.0) / 256.0, e)


def _run_subsets_x_only(w, inputs, rows=None):
    """x is taken in the rows' order, the residual in sorted row order."""
    if rows is None:
        return ORIG["run"](w, inputs, rows)
    rows = np.asarray(rows)
    sub = {**inputs, "x": inputs["x"][rows], "residual": inputs["residual"][np.sort(rows)]}
    return ORIG["run"](w, sub, None)


def _run_drops(name):
    def run(w, inputs, rows=None):
        return ORIG["run"](w, {k: v for k, v in inputs.items() if k != name}, rows)
    return run


def _run_qkv_bias_dropped(w, inputs, rows=None):
    if w.op != "qkv":
        return ORIG["run"](w, inputs, rows)
    return _run_drops("bias_out")(w, inputs, rows)


def _resid_dropped(a, W, bias, residual):
    return {"out": core.projection(a, W, bias)}


def _resid_bias_dropped(a, W, bias, residual):
    return {"out": np.asarray(residual, np.float64) + np.asarray(a) @ np.asarray(W).T}


def _resid_w_untransposed(a, W, bias, residual):
    y = np.asarray(a) @ np.asarray(W)
    return {"out": np.asarray(residual, np.float64) + y + (0 if bias is None else np.asarray(bias)[None])}


def _resid_subtracted(a, W, bias, residual):
    return {"out": core.projection(a, W, bias) - np.asarray(residual, np.float64)}


def _e4m3_truncates(v):
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -6.0)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.minimum(np.floor(a / quantum) * quantum, 448.0)
    return np.where(a > 0, np.sign(v) * q, 0.0)


def _e4m3_no_subnormals(v):
    q = ORIG["e4m3_round"](v)
    return np.where(np.abs(q) < 2.0 ** -6, 0.0, q)


def _e4m3_e5m2_max(v):
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -6.0)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.minimum(np.rint(a / quantum) * quantum, 480.0)
    return np.where(a > 0, np.sign(v) * q, 0.0)


def _fp8_per_tensor(v32):
    v32 = np.asarray(v32, np.float32)
    amax = np.float32(np.max(np.abs(v32)))
    s_ = np.full(v32.shape[0], amax / np.float32(448.0) if amax > 0 else np.float32(1.0), np.float32)
    return core.e4m3_round((v32 / s_[:, None]).astype(np.float32)), s_


def _fp8_scale_inverted(v32):
    q, s_ = ORIG["fp8_row_scale_and_codes"](v32)
    return q, (np.float32(1.0) / s_).astype(np.float32)


def _fp8_linear_no_weight_scale(a, Wq, w_scale, bias=None):
    return ORIG["fp8_linear"](a, Wq, np.ones_like(np.asarray(w_scale)), bias)


def _fp8_act_per_tensor(a32):
    a32 = np.asarray(a32, np.float32)
    q, s_ = ORIG["fp8_activation_codes"](a32.reshape(1, -1))
    return q.reshape(a32.shape), np.full(a32.shape[0], s_[0], np.float32)


def _fp8_act_no_dequant(a32):
    q, s_ = ORIG["fp8_activation_codes"](a32)
    return q, np.ones_like(s_)


def _fp8_norm32_drops_beta(h, mean, rstd, gamma, beta):
    return ORIG["fp8_normalised32"](h, mean, rstd, gamma, None)


def _tp_rounds_each_addition(parts):
    acc = core.bf16_round(np.asarray(parts[0], dtype=np.float64))
    for v in parts[1:]:
        acc = core.bf16_round(acc + np.asarray(v, dtype=np.float64))
    return acc


def _tp_drops_last_rank(parts):
    return ORIG["tp_allreduce"](list(parts)[:-1]) if len(parts) > 1 else ORIG["tp_allreduce"](parts)


def _tp_mean(parts):
    return ORIG["tp_allreduce"](parts) / len(parts)


MUTANTS = {
    "variance_divides_by_K_minus_1": ("layernorm", _ln_unbiased),
    "eps_outside_sqrt": ("layernorm", _ln_eps_outside),
    "beta_dropped": ("layernorm", _ln_no_beta),
    "gamma_before_centering": ("layernorm", _ln_gamma_before_centering),
    "rmsnorm_subtracts_mean": ("rmsnorm", _rms_centred),
    "rmsnorm_without_eps": ("rmsnorm", _rms_no_eps),
    "projection_transposed": ("projection", _proj_transposed),
    "projection_drops_bias": ("projection", _proj_no_bias),
    "k_and_v_swapped": ("split_qkv_head_major", _split_kv_swapped),
    "token_major_not_head_major": ("split_qkv_head_major", _split_token_major),
    "gate_and_up_swapped": ("swiglu", _swiglu_swapped),
    "gelu_cubic_coefficient": ("gelu_tanh", _gelu_wrong_cubic),
    "silu_is_sigmoid": ("silu", _silu_sigmoid_only),
    "bias_out_after_gelu": ("add_bias_norm_gelu", _gelu_bias_after),
    "bias_in_dropped": ("residual_add", _residual_drops_bias_in),
    "residual_ignored": ("residual_add", _residual_ignores_residual),
    "bf16_truncates": ("bf16_round", _bf16_truncate),
    "run_residual_rows_misordered": ("run", _run_subsets_x_only),
    "run_drops_bias_in": ("run", _run_drops("bias_in")),
    "run_drops_beta": ("run", _run_drops("beta")),
    "run_qkv_bias_dropped": ("run", _run_qkv_bias_dropped),
    "residual_projection_drops_residual": ("linear_add_residual", _resid_dropped),
    "residual_projection_drops_bias": ("linear_add_residual", _resid_bias_dropped),
    "residual_projection_w_untransposed": ("linear_add_residual", _resid_w_untransposed),
    "residual_projection_subtracts_residual": ("linear_add_residual", _resid_subtracted),
    "e4m3_truncates": ("e4m3_round", _e4m3_truncates),
    "e4m3_flushes_subnormals": ("e4m3_round", _e4m3_no_subnormals),
    "e4m3_saturates_at_480": ("e4m3_round", _e4m3_e5m2_max),
    "fp8_scale_per_tensor": ("fp8_row_scale_and_codes", _fp8_per_tensor),
    "fp8_scale_inverted": ("fp8_row_scale_and_codes", _fp8_scale_inverted),
    "fp8_weight_scale_dropped": ("fp8_linear", _fp8_linear_no_weight_scale),
    "fp8_activation_scale_per_tensor": ("fp8_activation_codes", _fp8_act_per_tensor),
    "fp8_activation_scale_dropped": ("fp8_activation_codes", _fp8_act_no_dequant),
    "fp8_normalisation_drops_beta": ("fp8_normalised32", _fp8_norm32_drops_beta),
    "tp_allreduce_rounds_each_addition": ("tp_allreduce", _tp_rounds_each_addition),
    "tp_allreduce_drops_last_rank": ("tp_allreduce", _tp_drops_last_rank),
    "tp_allreduce_averages": ("tp_allreduce", _tp_mean),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_breaks_a_pin(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(core, attr, fn)
    broken = []
    for pin in PINS:
        try:
            pin(core)
        except (AssertionError, ValueError, IndexError):
            broken.append(pin.__name__)
    assert broken, f"planted mistake {mutant!r} passed every pin"
