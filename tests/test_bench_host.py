"""Host logic of bench.py that needs no GPU: clock-record summarising and the byte model."""
import os

import numpy as np

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
from sparse_moe_layer_biased_b200.inputs import WORKLOADS


def test_clock_record_from_smi_lines():
    s = bench.ClockSampler("GPU-fake")
    s.lines = ["1965, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
               "1950, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
               "1800, 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active",
               "garbage"]
    r = s.stop()
    assert r["samples"] == 3 and r["sm_mhz"] == 1950 and r["sm_min_mhz"] == 1800 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_record_flags_thermal_reason():
    s = bench.ClockSampler("GPU-fake")
    s.samples = [(1500.0, 1965.0, {"hw_thermal_slowdown"}), (1965.0, 1965.0, set())]
    r = s.stop()
    assert r["reasons"] == ["hw_thermal_slowdown"] and r["samples"] == 2


def test_no_samples_is_reported():
    r = bench.ClockSampler("GPU-fake").stop()
    assert r["samples"] == 0 and r["sm_mhz"] is None


def test_gate_up_byte_model_counts_touched_experts_only():
    sh = WORKLOADS["step35_prefill"]
    counts = np.zeros(sh.E + 1, np.int64)
    counts[:10] = 5
    b, touched = bench.gate_up_bytes(sh, counts)
    assert touched == 10
    w = 10 * 2 * sh.I * sh.H * 2 + 2 * sh.Is * sh.H * 2
    acts = sh.T * sh.H * 2  # x read once; the permuted copy is not algorithmic
    out = sh.T * sh.k * sh.I * 2 + sh.T * sh.Is * 2
    assert b == w + acts + out
    b8, _ = bench.gate_up_bytes(sh, counts, fp8=True)
    assert b8 == b - 10 * 2 * sh.I * sh.H + 10 * (2 * sh.I // 128) * (sh.H // 128) * 4


PEAKS = {"hbm_gbs": 6541.8, "bf16_tflops": 1662.5, "bf16_tflops_sustained": 1383.5}


def _counts(sh, touched):
    c = np.zeros(sh.E + 1, np.int64)
    c[:touched] = 1
    return c


def test_roofline_bound_follows_arithmetic_intensity():
    # skewed Step-5 shape (248 experts touched): 3.71 TFLOP against 6.85 GB -> tensor-bound
    sh = WORKLOADS["step5_skewed"]
    r = bench.gate_up_roofline(sh, _counts(sh, 248), 3.0, PEAKS, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    flops = 4.0 * sh.H * (sh.I * sh.T * sh.k + sh.Is * sh.T)
    assert r["algorithmic_flops"] == flops
    assert abs(r["achieved"] - flops / 3e-3 / 1e12) < 1e-9 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 1662.5) < 1e-12
    # Step-3.5 prefill (242 touched): 141 flop/B, below the ~254 flop/B ridge -> HBM-bound
    s35 = WORKLOADS["step35_prefill"]
    r = bench.gate_up_roofline(s35, _counts(s35, 242), 1.0, PEAKS, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["intensity_flop_per_byte"] < r["ridge_flop_per_byte"]
    # decode: HBM-bound; FP8 weights are always reported against HBM
    dec = WORKLOADS["step35_decode"]
    assert bench.gate_up_roofline(dec, _counts(dec, 159), 0.5, PEAKS, "measured")["bound"] == "hbm"
    assert bench.gate_up_roofline(sh, _counts(sh, 248), 3.0, PEAKS, "measured", fp8=True)["bound"] == "hbm"


def test_decode_sized_workloads_flush_l2():
    assert bench.decode_sized(WORKLOADS["step35_decode"])
    assert not bench.decode_sized(WORKLOADS["step5_skewed"])


def test_sample_parity_counts_near_tie_tokens_separately():
    import torch

    rng = np.random.default_rng(0)
    y = torch.from_numpy(rng.standard_normal((10, 8)).astype(np.float32))
    idx = torch.from_numpy(np.tile(np.arange(2, dtype=np.int32), (10, 1)))
    ref = {"y": y.double().numpy()[[1, 4, 7]], "idx": np.array([[1, 0], [0, 1], [0, 5]], np.int32),
           "margin": np.array([1.0, 1.0, 1e-8], np.float32)}
    p = bench.sample_parity(y, idx, None, [1, 4, 7], ref)
    assert p["tokens"] == 3 and p["near_ties"] == 1 and p["near_tie_tokens_routed_differently"] == 1
    assert p["ids_equal_outside_near_ties"] and p["rel_fro"] == 0.0 and p["max_abs"] == 0.0


def test_source_digest_ignores_comments_only():
    src = 'asm("mov.u32 %0, 1; // not a comment inside the string" : "=r"(x));\n'
    a = bench._strip_comments("// header\n" + src + "/* block\n comment */ int y = '/';\n")
    b = bench._strip_comments(src + "int y = '/';  // trailing\n\n")
    assert a == b and "not a comment" in a and "header" not in a
    assert bench._strip_comments("int a;") != bench._strip_comments("int b;")


def test_profiled_traffic_is_tied_to_the_current_sources():
    for (shape, weights), e in bench.PROFILED_TRAFFIC.items():
        assert shape in WORKLOADS
        assert 1.0 <= e["ratio"] < 2.0  # traffic at or a little above the algorithmic bytes
        got = bench.profiled_traffic(shape, weights, 1e9)
        assert got is None or abs(got - e["ratio"] * 1e9) < 1.0
        assert os.path.exists(os.path.join(ROOT, e["source"]))


def test_kernels_per_step():
    s35, dec = WORKLOADS["step35_prefill"], WORKLOADS["step35_decode"]
    assert bench.kernels_per_step(s35) == 6
    assert bench.kernels_per_step(s35, deterministic=True) == 7
    assert bench.kernels_per_step(s35, router=False) == 5
    assert bench.kernels_per_step(s35, fp8=True) == 9  # shared expert on the BF16 pair kernels
    assert bench.kernels_per_step(dec, fp8=True) == 6


def test_gate_up_kernel_name_follows_the_library_configuration():
    assert bench.gate_up_kernel_name(WORKLOADS["step5_skewed"]) == "gate_up_pair_kernel"
    assert bench.gate_up_kernel_name(WORKLOADS["step35_decode"]) == "gate_up_kernel"
    assert bench.gate_up_kernel_name(WORKLOADS["step35_decode"], fp8=True) == "gemm_fp8_mma_kernel<GateUpArgs>"
    assert bench.gate_up_kernel_name(WORKLOADS["step35_prefill"], fp8=True) == "gemm_fp8_kernel<GateUpArgs>"
    odd = WORKLOADS["step35_decode"].replace(Is=192)
    assert bench.gate_up_kernel_name(odd, fp8=True) == "gemm_fp8_kernel<GateUpArgs>"


def test_traffic_sources_exist():
    d = os.path.join(ROOT, "sparse_moe_layer_biased_b200", "csrc")
    for name in bench.TRAFFIC_SOURCES:
        assert os.path.exists(os.path.join(d, name)), name
