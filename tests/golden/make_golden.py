"""Writes tests/golden/tiny_cases.json: three tiny cases (one per epilogue) with
their inputs and the fp64 oracle's outputs.

The pages print no worked numeric example, so these values are not the pages':
they are the oracle's, frozen as a regression fixture (the oracle's own pins
are in tests/test_oracle_pins.py). Inputs are bf16 values drawn with numpy's
seeded generator; this script calls nothing but numpy and oracle/.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402


def bf16(a):
    return oracle.bf16_round(a)


def case(kind, seed):
    rng = np.random.default_rng(seed)
    M, K = 3, 32
    c = {"kind": kind, "M": M, "K": K, "eps": 1e-5}
    c["x"] = bf16(rng.normal(size=(M, K)))
    c["residual"] = bf16(rng.normal(size=(M, K)))
    c["gamma"] = bf16(1 + 0.1 * rng.normal(size=K))
    if kind == "qkv":
        c.update(norm="layernorm", Hq=2, Hkv=1, D=8)
        c["beta"] = bf16(0.1 * rng.normal(size=K))
        N = (2 + 2) * 8
        c["W"] = bf16(rng.normal(size=(N, K)) / np.sqrt(K))
        o = oracle.add_norm_qkv(c["x"], c["residual"], c["gamma"], c["beta"], "layernorm",
                                c["eps"], c["W"], None, 2, 1, 8)
    elif kind == "swiglu":
        c.update(norm="rmsnorm", I=16)
        c["W"] = bf16(rng.normal(size=(32, K)) / np.sqrt(K))
        o = oracle.add_norm_swiglu(c["x"], c["residual"], c["gamma"], None, "rmsnorm",
                                   c["eps"], c["W"], None, 16)
    else:
        c.update(norm="layernorm", N=24)
        c["bias_in"] = bf16(rng.normal(size=K))
        c["beta"] = bf16(0.1 * rng.normal(size=K))
        c["W"] = bf16(rng.normal(size=(24, K)) / np.sqrt(K))
        c["bias_out"] = bf16(0.02 * rng.normal(size=24))
        o = oracle.add_bias_norm_gelu(c["x"], c["residual"], c["bias_in"], c["gamma"],
                                      c["beta"], "layernorm", c["eps"], c["W"], c["bias_out"])
    c["expected"] = o
    return c


def to_json(v):
    if isinstance(v, np.ndarray):
        return {"shape": list(v.shape), "data": [float(t) for t in v.ravel()]}
    if isinstance(v, dict):
        return {k: to_json(t) for k, t in v.items()}
    return v


def main():
    cases = [case("qkv", 101), case("swiglu", 102), case("gelu", 103)]
    doc = {
        "source": "fp64 oracle (oracle/), frozen by tests/golden/make_golden.py; "
                  "the pages print no worked values for this op",
        "cases": [to_json(c) for c in cases],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_cases.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=0)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
