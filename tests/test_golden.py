"""The oracle still reproduces its frozen tiny cases (regression guard)."""
import json
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _arr(v):
    return np.asarray(v["data"], dtype=np.float64).reshape(v["shape"])


def load_cases():
    with open(os.path.join(HERE, "golden", "tiny_cases.json")) as f:
        doc = json.load(f)
    out = []
    for c in doc["cases"]:
        d = {}
        for k, v in c.items():
            if isinstance(v, dict) and "shape" in v:
                d[k] = _arr(v)
            elif k == "expected":
                d[k] = {kk: _arr(vv) for kk, vv in v.items()}
            else:
                d[k] = v
        out.append(d)
    return out


def test_inputs_are_bf16_values():
    for c in load_cases():
        for k in ("x", "residual", "gamma", "W"):
            assert np.array_equal(oracle.bf16_round(c[k]), c[k])


def test_oracle_reproduces_golden():
    for c in load_cases():
        if c["kind"] == "qkv":
            o = oracle.add_norm_qkv(c["x"], c["residual"], c["gamma"], c["beta"], c["norm"],
                                    c["eps"], c["W"], None, c["Hq"], c["Hkv"], c["D"])
        elif c["kind"] == "swiglu":
            o = oracle.add_norm_swiglu(c["x"], c["residual"], c["gamma"], None, c["norm"],
                                       c["eps"], c["W"], None, c["I"])
        else:
            o = oracle.add_bias_norm_gelu(c["x"], c["residual"], c["bias_in"], c["gamma"],
                                          c["beta"], c["norm"], c["eps"], c["W"], c["bias_out"])
        for k, want in c["expected"].items():
            np.testing.assert_allclose(o[k], want, rtol=1e-13, atol=1e-14)
