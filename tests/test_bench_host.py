"""Host logic of bench.py that needs no GPU: a DRAM-traffic figure recorded
from an ncu capture is used only while the kernel's source file and the device
headers beside it are unchanged."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_recorded_traffic_goes_stale_with_kernel_or_header(tmp_path, monkeypatch):
    csrc = tmp_path / "test_sequence_layers_layer_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("kernel v1")
    (csrc / "a.cuh").write_text("header v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.source_sha("k.cu")
    (tmp_path / "profiles" / "k_kernel__w.md").write_text(
        f"traffic: kernel=k_kernel workload=w bytes_per_launch=1234 source_sha={sha}\n")

    def current():
        return bench.recorded_traffic("k_kernel", "w", bench.source_sha("k.cu"))

    assert current() == 1234.0
    assert bench.recorded_traffic("k_kernel", "other_workload", sha) is None
    (csrc / "a.cuh").write_text("header v2")  # a device header changed
    assert current() is None
    (csrc / "a.cuh").write_text("header v1")
    assert current() == 1234.0
    (csrc / "k.cu").write_text("kernel v2")  # the kernel itself changed
    assert current() is None
