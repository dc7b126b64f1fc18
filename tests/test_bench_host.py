"""Host-side pieces of bench.py that need no GPU: the roofline denominators it reads, and the
committed DRAM-traffic summary of the headline step's GEMM launches, which the bench only
reports while it describes the GEMM sources as they stand."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _profile_fields(key):
    fields = {}
    with open(os.path.join(ROOT, "profiles", f"w8a8_gemm_traffic_{key}.md")) as f:
        for line in f:
            if ":" in line and line.split(":")[0].strip().isidentifier():
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    return fields


def test_headline_traffic_summary_describes_the_current_gemm():
    """The summary's source hash matches sq_gemm.cu + sq_ptx.cuh, so the bench line carries its
    figure; its algorithmic bytes are one read of xq and Wq and one bf16 write of y, averaged
    over the step's four linears."""
    key = bench.HEADLINE.key
    traffic = bench.gemm_traffic(key)
    assert traffic is not None, "the GEMM changed since the traffic summary was captured"
    fields = _profile_fields(key)
    M = bench.HEADLINE.tokens
    algorithmic = sum(M * K + N * K + 2 * M * N for _, K, N, _ in bench.HEADLINE.layers) // 4
    assert int(fields["algorithmic_bytes_per_launch"]) == algorithmic
    assert traffic == int(fields["traffic_bytes_per_launch"])
    # DRAM moves at least the operands once (reads) and most of the output (writes)
    assert algorithmic <= traffic < 2 * algorithmic


def test_traffic_is_absent_without_a_summary():
    assert bench.gemm_traffic("no_such_workload") is None


def test_peaks_come_from_the_measured_file():
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        measured = json.load(f)
    p = bench.load_peaks()
    assert p["source"] == "measured"
    assert p["hbm_gbs"] == measured["hbm_gbs"] and p["bf16_tflops"] == measured["bf16_tflops"]
    # the INT8 denominator the bench starts from: twice the dense bf16 rate
    assert bench.INT8_PER_BF16 == 2


def test_workload_ops_count_two_per_multiply_add():
    """2048 tokens through 12288->36864, 12288->12288, 12288->49152 and 49152->12288."""
    macs = 2048 * (12288 * 36864 + 12288 * 12288 + 12288 * 49152 + 49152 * 12288)
    assert bench.HEADLINE.ops() == 2.0 * macs
