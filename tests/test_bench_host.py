"""Host checks of bench.py's measurement arithmetic (no GPU): the algorithmic
FLOP and byte counts the JSON line divides by, the choice of peak and the
roofline fields."""

import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_nf4_quantized_17_b200 import qlora as Q  # noqa: E402
from bit_nf4_quantized_17_b200 import workloads as WL  # noqa: E402

PEAKS = {"hbm": 6559.0, "bf16": 1656.2, "bf16_sustained": 1389.6, "sm_max_mhz": 1965.0,
         "source": "measured"}


def test_flop_counts():
    # fwd 2MNK + 2MKr + 2MNr; fwd + bwd 4MNK + 6Mr(N + K)
    assert bench.fwd_flops(3, 5, 7, 2) == 2 * 3 * 5 * 7 + 2 * 3 * 7 * 2 + 2 * 3 * 5 * 2
    assert bench.fwd_bwd_flops(4096, 4096, 4096, 16) == 4 * 4096 ** 3 + 6 * 4096 * 16 * 8192


def test_stack_65b_flops_and_storage():
    # 80 layers x (4 x 8192^2 + 3 x 22016 x 8192) at M = 2048, r = 64
    shapes = WL.WORKLOADS["stack_65b"].linears
    per_layer = sum(bench.fwd_bwd_flops(2048, s.d_out, s.d_in, s.r) for s in shapes)
    base = 4 * 2048 * (4 * 8192 * 8192 + 3 * 22016 * 8192)
    lora = 6 * 2048 * 64 * (4 * 16384 + 3 * 30208)
    assert per_layer == base + lora
    assert 80 * per_layer == pytest.approx(540.4e12, rel=1e-3)
    nf4 = 80 * sum(bench.nf4_bytes(s.d_out, s.d_in) for s in shapes)
    # 4.127 bits per weight of 64.76 G weights: about 33.4 GB resident
    assert nf4 == pytest.approx(80 * (4 * 8192 ** 2 + 3 * 22016 * 8192) * 4.126953 / 8, rel=1e-6)
    assert 33.3e9 < nf4 < 33.5e9


def test_nf4_bytes_of_the_mlp_linear():
    # codes n/2 + int8 scale codes nb + fp32 group factors 4 ng + fp32 mean 4
    assert bench.nf4_bytes(11008, 4096) == 23_259_908
    n = 11008 * 4096
    nb = n // 64
    assert bench.nf4_bytes(11008, 4096) == n // 2 + nb + 4 * (-(-nb // 256)) + 4


def test_peak_is_the_burst_figure_and_clock_scaling():
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1680.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.bf16_peak(PEAKS, full)[0] == 1656.2
    assert bench.bf16_peak(PEAKS, capped)[0] == 1656.2
    assert "burst" in bench.bf16_peak(PEAKS, capped)[1]
    assert "sw_power_cap" in bench.bf16_peak(PEAKS, capped)[1]
    assert bench.clock_scaled_peak(PEAKS, full) == 1656.2
    assert bench.clock_scaled_peak(PEAKS, capped) == pytest.approx(1656.2 * 1680 / 1965)
    assert bench.clock_scaled_peak(PEAKS, {"sm_mhz": None, "reasons": []}) == 1656.2


def test_kernel_lines_divide_work_by_event_time():
    M = N = K = 4096
    r = 16
    kt = {Q.QLORA_KERNEL_QUANTIZE: (0.048, 2), Q.QLORA_KERNEL_FUSED_FWD: (0.272, 2),
          Q.QLORA_KERNEL_FUSED_DGRAD: (0.0, 0), Q.QLORA_KERNEL_LORA_GEMM: (0.08, 4)}
    work = {
        "quantize_blocks": (Q.QLORA_KERNEL_QUANTIZE, "hbm", 2 * N * K + N * K // 2 + 4 * (N * K // 64), 1),
        "fused_fwd": (Q.QLORA_KERNEL_FUSED_FWD, "tensor", 2 * M * N * K + 2 * M * N * r, 1),
        "fused_dgrad": (Q.QLORA_KERNEL_FUSED_DGRAD, "tensor", 2 * M * N * K + 2 * M * K * r, 1),
        "lora_gemms": (Q.QLORA_KERNEL_LORA_GEMM, "tensor", 4 * M * K * r + 4 * M * N * r, 4),
    }
    out = bench.kernel_lines(kt, work, PEAKS, 1656.2, "burst",
                             {"sm_mhz": 1680.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert "fused_dgrad" not in out  # no launches, no line
    f = out["fused_fwd"]
    w = 2 * M * N * K + 2 * M * N * r
    assert f["algorithmic_per_launch"] == w
    assert f["achieved"] == pytest.approx(w / 136e-6 / 1e12, rel=1e-4)
    assert f["frac"] == pytest.approx(f["achieved"] / 1656.2, abs=1e-4)
    assert f["frac_of_sustained"] == pytest.approx(f["achieved"] / 1389.6, abs=1e-4)
    assert f["frac_of_clock_scaled_burst"] == pytest.approx(
        f["achieved"] / (1656.2 * 1680 / 1965), abs=1e-4)
    q = out["quantize_blocks"]
    assert q["unit"] == "GB/s" and q["bound"] == "hbm"
    assert q["frac"] == pytest.approx(q["achieved"] / 6559.0, abs=1e-4)
    g = out["lora_gemms"]
    assert g["algorithmic_per_launch"] == (4 * M * K * r + 4 * M * N * r) / 4


def test_mixed_shape_kernel_rate_is_total_work_over_total_time():
    # a kind launched on linears of different shapes: average work per launch
    # over average launch time = total work / total time
    kt = {Q.QLORA_KERNEL_FUSED_FWD: (3.0, 6)}
    out = bench.kernel_lines(kt, {"fused_fwd": (Q.QLORA_KERNEL_FUSED_FWD, "tensor", 3.0e12, 6)},
                             PEAKS, 1656.2, "burst")
    assert out["fused_fwd"]["achieved"] == pytest.approx(3.0e12 / 3.0e-3 / 1e12, rel=1e-6)


def test_roofline_takes_the_largest_kernel_and_drops_stale_traffic(monkeypatch):
    kernels = {"fused_fwd": {"bound": "tensor", "achieved": 1000.0, "peak": 1656.2,
                             "unit": "TFLOP/s", "frac": 0.6, "avg_us": 10.0, "total_ms": 5.0,
                             "algorithmic_per_launch": 1.0, "peak_kind": "burst"},
               "fused_dgrad": {"bound": "tensor", "achieved": 900.0, "peak": 1656.2,
                               "unit": "TFLOP/s", "frac": 0.54, "avg_us": 11.0, "total_ms": 6.0,
                               "algorithmic_per_launch": 1.0, "peak_kind": "burst"}}
    monkeypatch.setattr(bench, "TRAFFIC", {("fused_dgrad", "stack_65b"):
                                           {"sha": bench.sources_sha("fused_dgrad"),
                                            "bytes_per_launch": 123}})
    r = bench.roofline_of(kernels, "stack_65b")
    assert r["kernel"] == "fused_dgrad" and r["traffic"] == 123 and r["frac"] == 0.54
    monkeypatch.setattr(bench, "TRAFFIC", {("fused_dgrad", "stack_65b"):
                                           {"sha": "0" * 16, "bytes_per_launch": 123}})
    assert bench.roofline_of(kernels, "stack_65b")["traffic"] is None


def test_stack_config_names_the_workload():
    c = bench.stack_config("stack_65b", 80, 2)
    assert c["global_batch"] == 8 and c["parallelism"] == "dp2" and c["layers"] == 80
    assert "stack_65b" in c["workload"] and "80 layers" in c["workload"]


def test_decode_alu_roofline_constants():
    # 21 lookup operations per 8 weights plus 16 table operations per 64-weight block,
    # against 64 ALU lanes per clock per SM at the maximum clock (148 SMs without a GPU)
    assert bench.EXPAND_OPS_PER_WEIGHT == 21 / 8 + 16 / 64
    if not torch.cuda.is_available():
        assert bench.alu_peak_ops({"sm_max_mhz": 1965.0}) == 148 * 64 * 1965.0e6
