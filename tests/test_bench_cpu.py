"""The benchmark's accounting (CPU): algorithmic bytes and FLOPs per
token-head, the per-kernel roofline and the step roofline, checked against
counts written out by hand for the workloads' shapes."""
import pytest

import bench
from gated_delta_rule_72_b200 import inputs

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0}


def test_bytes_per_token_head_by_hand():
    w = inputs.WORKLOADS["skewed"]          # bf16 q, k, v; d_k = d_v = 128
    # q, k, v: 2 B x (128 + 128 + 128); alpha, beta: 8 B; o: 4 B (fp32) or 2 B x 128
    assert bench.bytes_per_token_head(w) == 768 + 8 + 512
    assert bench.bytes_per_token_head(w, out_bytes=2) == 768 + 8 + 256
    t = inputs.WORKLOADS["tiny"]            # fp32, d = 64
    assert bench.bytes_per_token_head(t) == 4 * 192 + 8 + 4 * 64


def test_kernel_bytes_split_between_prep_and_chain():
    w = inputs.WORKLOADS["skewed"]
    prep = bench.kernel_algorithmic_bytes("tc_prep", w)
    chain = bench.kernel_algorithmic_bytes("tc_chain", w)
    assert prep == 776 and chain == 512
    assert prep + chain == bench.bytes_per_token_head(w)
    assert bench.kernel_algorithmic_bytes("tc_chain", w, out_bytes=2) == 256


def test_frame_wise_kernel_bytes_by_hand():
    w = inputs.WORKLOADS["vda480"]          # bf16, d = 128, frames of 1,560 tokens
    assert bench.vda_kernel_bytes("vda_gram_tc", w) == 2 * 256 + 4
    # q in (256 B), o out (512 B), the two directions' fp32-sized states per frame
    assert bench.vda_kernel_bytes("vda_readout_tc", w) == pytest.approx(256 + 512 + 2 * 4 * 128 * 128 / 1560)
    f = bench.vda_kernel_flops(w)
    assert f["vda_gram_tc"] == f["vda_gram"] == 2 * 128 * 256
    assert f["vda_readout_tc"] == f["vda_readout"] == 2 * 128 * 128


def test_flops_per_token_head_by_hand():
    w = inputs.WORKLOADS["stream480"]
    C, d = 64, 128
    assert bench.flops_per_token_head(w) == pytest.approx(C * 10 * d + 6 * d * d + C * C / 3)
    b = inputs.WORKLOADS["bidir720"]
    assert bench.flops_per_token_head(b) == pytest.approx(
        C * 10 * d + 6 * d * d + C * C / 3 + C * 6 * d + 6 * d * d + C * C / 3)


def test_roofline_takes_the_dominant_kernel():
    w = inputs.WORKLOADS["skewed"]
    steps = 10
    kt = {"tc_prep": (10.0, 10), "tc_chain": (5.0, 10)}     # total ms, launches
    r = bench.roofline_of(w, kt, steps, w.token_heads, PEAKS, "measured")
    assert r["kernel"] == "tc_prep" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    # one launch per step, 1.0 ms each, over every token-head of the workload
    want = 776 * w.token_heads / 1e-3 / 1e9
    assert r["achieved"] == pytest.approx(want)
    assert r["frac"] == pytest.approx(want / 6000.0)
    assert r["kernel_share"] == pytest.approx(10.0 / 15.0)
    assert r["traffic"] == pytest.approx(bench.MEASURED_TRAFFIC_PER_TOKEN_HEAD[("tc_prep", "skewed")]
                                         * w.token_heads)


def test_frame_wise_roofline_bounds():
    w = inputs.WORKLOADS["vda480"]
    kt = {"vda_gram_tc": (1.0, 10), "vda_factor": (0.5, 10), "vda_chain": (0.8, 10), "vda_readout_tc": (1.2, 10)}
    r = bench.roofline_of(w, kt, 10, w.token_heads, PEAKS, "measured")
    assert r["kernel"] == "vda_readout_tc" and r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(bench.vda_kernel_bytes("vda_readout_tc", w) * w.token_heads / 0.12e-3 / 1e9)
    kt["vda_chain"] = (3.0, 10)
    r = bench.roofline_of(w, kt, 10, w.token_heads, PEAKS, "measured")
    assert r["kernel"] == "vda_chain" and r["bound"] == "alu" and r["unit"] == "TFLOP/s"
    assert r["peak"] == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def test_step_roofline_is_the_slower_bound():
    w = inputs.WORKLOADS["skewed"]
    bytes_fp32 = bench.algorithmic_bytes_per_step(w)
    assert bytes_fp32 == w.token_heads * 1288 + 4 * 32 * 128 * 128 * 4    # + the final state
    t_mem = bytes_fp32 / 6000e9
    t_flop = w.token_heads * bench.flops_per_token_head(w) / 1500e12
    assert t_mem > t_flop
    r = bench.step_roofline(w, 2.0, PEAKS)
    assert r["bound"] == "hbm"
    assert r["t_roofline_ms"] == pytest.approx(t_mem * 1e3)
    assert r["frac"] == pytest.approx(t_mem * 1e3 / 2.0)
    assert r["t_roofline_ms_bf16_out"] < r["t_roofline_ms"]
