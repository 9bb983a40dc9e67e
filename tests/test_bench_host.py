"""Host-side pieces of bench.py that need no GPU: the DRAM-traffic figures of the fused GEMMs
are reported only while the kernel sources they were captured on are unchanged."""

import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_reported_for_the_captured_sources():
    assert bench.fused_traffic("dx") == bench.FUSED_TRAFFIC["dx"]
    assert bench.fused_traffic("fwd") == bench.FUSED_TRAFFIC["fwd"]
    assert bench.FUSED_TRAFFIC["dx"] > 0 and bench.FUSED_TRAFFIC["fwd"] > 0


def test_traffic_withdrawn_when_a_kernel_source_changes(tmp_path, monkeypatch):
    # a copy of the package with one fused-GEMM source edited
    fake_root = tmp_path / "root"
    shutil.copytree(os.path.join(ROOT, "bit_nf4_quantized_dq_b200", "csrc"),
                    fake_root / "bit_nf4_quantized_dq_b200" / "csrc")
    with open(fake_root / "bit_nf4_quantized_dq_b200" / "csrc" / "gemm.cuh", "a") as f:
        f.write("\n// edited\n")
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.fused_traffic("dx") is None
    assert bench.fused_traffic("fwd") is None


@pytest.mark.parametrize("name", ["gemm.cuh", "gemm.h", "common.cuh", "nf4_device.cuh", "qlora_nf4.cu"])
def test_every_fused_source_exists(name):
    assert name in bench.FUSED_SOURCES
    assert os.path.exists(os.path.join(ROOT, "bit_nf4_quantized_dq_b200", "csrc", name))
