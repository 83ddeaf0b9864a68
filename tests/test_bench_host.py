"""Host checks of bench.py's measurement arithmetic (no GPU): the algorithmic
FLOP and byte counts the JSON line divides by, and the roofline fields."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_nf4_quantized_17_b200 import qlora as Q  # noqa: E402


def test_flop_counts():
    # fwd 2MNK + 2MKr + 2MNr; fwd + bwd 4MNK + 6Mr(N + K)
    assert bench.fwd_flops(3, 5, 7, 2) == 2 * 3 * 5 * 7 + 2 * 3 * 7 * 2 + 2 * 3 * 5 * 2
    assert bench.fwd_bwd_flops(4096, 4096, 4096, 16) == 4 * 4096 ** 3 + 6 * 4096 * 16 * 8192


def test_nf4_bytes_of_the_mlp_linear():
    # codes n/2 + int8 scale codes nb + fp32 group factors 4 ng + fp32 mean 4
    assert bench.nf4_bytes(11008, 4096) == 23_259_908
    n = 11008 * 4096
    nb = n // 64
    assert bench.nf4_bytes(11008, 4096) == n // 2 + nb + 4 * (-(-nb // 256)) + 4


def test_kernel_rooflines_divide_work_by_event_time():
    peaks = {"hbm": 6559.0, "bf16_sustained": 1389.6, "source": "measured"}
    M = N = K = 4096
    r = 16
    kt = {Q.QLORA_KERNEL_QUANTIZE: (0.048, 2), Q.QLORA_KERNEL_FUSED_FWD: (0.272, 2),
          Q.QLORA_KERNEL_FUSED_DGRAD: (0.0, 0), Q.QLORA_KERNEL_LORA_GEMM: (0.08, 4)}
    out = bench.kernel_rooflines(kt, M, N, K, r, peaks)
    assert "fused_dgrad" not in out  # no launches, no line
    f = out["fused_fwd"]
    work = 2 * M * N * K + 2 * M * N * r
    assert f["algorithmic_per_launch"] == work
    assert f["achieved"] == pytest.approx(work / 136e-6 / 1e12, rel=1e-4)
    assert f["frac"] == pytest.approx(f["achieved"] / 1389.6, abs=1e-4)
    q = out["quantize_blocks"]
    assert q["unit"] == "GB/s" and q["bound"] == "hbm"
    assert q["algorithmic_per_launch"] == 2 * N * K + N * K // 2 + 4 * (N * K // 64)
    g = out["lora_gemms"]
    assert g["algorithmic_per_launch"] == (4 * M * K * r + 4 * M * N * r) / 4


def test_config_names_the_workload():
    c = bench.workload_config(2)
    assert c["global_batch"] == 2 * bench.TOKENS and c["parallelism"] == "dp2"
    assert "attn_4096" in c["workload"]
