"""The benchmark's bookkeeping (no GPU needed): each workload's shape,
algorithmic FLOPs and bytes, and its roofline bound, against the figures the
workload table of the method's measurement plan states (2MNK FLOPs; bytes =
x and residual read, residual_out written, W read once, outputs written, the
vectors), so that every fraction the bench reports divides the right work by
the right peak."""
import pytest

import bench
import synthetic

WL = synthetic.workloads()

# name: (M, K, N, FLOPs, algorithmic bytes, bound)
TABLE = {
    "c1_tiny_ln_qkv": (8, 256, 512, 2.10e6, 0.284e6, "hbm"),
    "c2_decode_rms_qkv": (32, 4096, 6144, 1.61e9, 51.5e6, "hbm"),
    "c3_prefill_rms_swiglu": (16384, 4096, 28672, 3.848e12, 1.107e9, "tensor"),
    "c4_gpt_ln_gelu": (4096, 4096, 16384, 5.50e11, 369e6, "tensor"),
    "c5_70b_rms_qkv_m1": (1, 8192, 10240, 1.68e8, 167.9e6, "hbm"),
    "c5_70b_rms_qkv_m8": (8, 8192, 10240, 1.68e8 * 8, 168.4e6, "hbm"),
    "c5_70b_rms_qkv_m32": (32, 8192, 10240, 1.68e8 * 32, 170.0e6, "hbm"),
    "c5_70b_rms_qkv_m256": (256, 8192, 10240, 1.68e8 * 256, 185.6e6, "hbm"),
    "c5_70b_rms_qkv_m2048": (2048, 8192, 10240, 3.44e11, 310e6, "tensor"),
    "c5_70b_rms_qkv_m8192": (8192, 8192, 10240, 1.37e12, 738e6, "tensor"),
    "c5_70b_rms_qkv_ragged": (62386, 8192, 10240, 1.047e13, 4.51e9, "tensor"),
}


@pytest.mark.parametrize("name", sorted(TABLE))
def test_workload_matches_the_table(name):
    M, K, N, flops, nbytes, bound = TABLE[name]
    w = WL[name]
    assert (w.M, w.K, w.N) == (M, K, N)
    assert w.flops() == pytest.approx(flops, rel=5e-3)
    assert w.algorithmic_bytes() == pytest.approx(nbytes, rel=5e-3)
    assert bench.units(w)[2] == bound


def test_packed_batch_lengths():
    w = WL["c5_70b_rms_qkv_ragged"]
    assert len(w.seq_lens) == 64 and sum(w.seq_lens) == w.M == 62386
    assert all(1 <= n <= 2048 for n in w.seq_lens)


def test_units_per_step_are_the_bound_quantity():
    for w in WL.values():
        unit, per_step, bound = bench.units(w)
        if bound == "hbm":
            assert unit == "GB/s" and per_step == pytest.approx(w.algorithmic_bytes() / 1e9)
        else:
            assert unit == "TFLOP/s" and per_step == pytest.approx(w.flops() / 1e12)


def test_roofline_denominators_are_the_measured_peaks():
    pk, src = bench.peaks()
    w = WL["c5_70b_rms_qkv_ragged"]
    achieved, peak, unit, _ = bench._roofline(w, 10.0, "tensor")   # 10 ms per launch
    assert peak == pk["bf16_tflops_sustained"] and unit == "TFLOP/s"
    assert achieved == pytest.approx(w.flops() / 1e-2 / 1e12)
    w = WL["c2_decode_rms_qkv"]
    achieved, peak, unit, _ = bench._roofline(w, 0.02, "hbm")      # 20 us per launch
    assert peak == pk["hbm_gbs"] and unit == "GB/s"
    assert achieved == pytest.approx(w.algorithmic_bytes() / 2e-5 / 1e9)
