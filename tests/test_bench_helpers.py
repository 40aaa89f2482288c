"""The algorithmic byte counts behind the benchmark's roofline numbers (CPU):
what the method must move per launch, from the artifact layout."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_gemv_bytes_of_the_headline_layer():
    # packed codes 0.5 B/weight + fp16 scale and zero per 128 weights + bf16 x and y
    N = K = 4096
    assert bench.gemv_bytes(N, K, 1, False) == N * K // 2 + (N * K // 128) * 4 + 2 * (N + K) == 8_929_280
    assert bench.gemv_bytes(N, K, 1, True) == 8_929_280 - (N * K // 128) * 2


def test_quantize_bytes_of_the_headline_layer():
    # bf16 in (2 B) + packed out (0.5 B) + scale/zero (4 B per group)
    assert bench.quant_bytes(4096, 4096, False) == 42_467_328
    assert bench.quant_bytes(4096, 4096, False) / (4096 * 4096) == 2.53125


def test_traffic_record_names_its_sources():
    rec = json.load(open(os.path.join(ROOT, "profiles", "gemv_traffic.json")))
    # the kernel the headline M=1 layer runs on
    assert rec["kernel"].startswith("gemv_ksplit_res_kernel") and rec["kernel_sources"]
    for f in rec["kernel_sources"]:
        assert os.path.exists(os.path.join(ROOT, "w4a16_bit_gemm_b200", "csrc", f))
    # traffic over algorithmic bytes: no re-reads
    assert 1.0 <= rec["dram_bytes_per_launch"] / bench.gemv_bytes(4096, 4096, 1, False) < 1.01
