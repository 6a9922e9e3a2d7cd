"""Host-side accounting of bench.py (no GPU): the stored bytes per expert that
the HBM roofline divides by, the hot-set rule of the layer-stack workload, and
the gate that drops the recorded DRAM traffic once the kernel sources change."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixed_precision_moe_b200 import synth  # noqa: E402


def test_expert_bytes_follow_the_storage_formula():
    # P = 3 H I weights; BF16 2 P bytes, INT8 P + P/64 (one fp16 scale per 128), INT4 P/2 + P/64
    assert bench.expert_bytes(synth.BF16, 2048, 768) == 9_437_184
    assert bench.expert_bytes(synth.INT8, 2048, 768) == 4_792_320
    assert bench.expert_bytes(synth.INT4, 2048, 768) == 2_433_024
    assert bench.expert_bytes(synth.INT4, 4096, 14336) == 90_832_896
    assert bench.expert_bytes(synth.BF16, 2048, 512) == 6_291_456
    assert bench.expert_bytes(synth.INT4, 2048, 512) == 1_622_016
    # the scales are exactly what the quantised layout stores: 2 bytes per 128 weights
    for H, I in ((256, 512), (2048, 768)):
        P = 3 * H * I
        assert bench.expert_bytes(synth.INT4, H, I) == P // 2 + 2 * (P // 128)
        assert bench.expert_bytes(synth.INT8, H, I) == P + 2 * (P // 128)


def test_traffic_record_is_used_only_for_the_recorded_kernel(tmp_path, monkeypatch):
    rec = tmp_path / "profile.md"
    h = bench.ffn_kernel_hash()
    rec.write_text(f"traffic-record: kernel_sha256={h} dram_bytes=1100 algorithmic_bytes=1000\n")
    monkeypatch.setattr(bench, "FFN_PROFILE", str(rec))
    assert bench.ffn_traffic(2000) == 2200          # scaled by the units processed
    rec.write_text("traffic-record: kernel_sha256=0000000000000000 dram_bytes=1100 "
                   "algorithmic_bytes=1000\n")
    assert bench.ffn_traffic(2000) is None          # counters of another kernel
    monkeypatch.setattr(bench, "FFN_PROFILE", str(tmp_path / "missing.md"))
    assert bench.ffn_traffic(2000) is None

