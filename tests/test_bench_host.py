"""Host-side logic of the benchmark that needs no GPU."""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_profiled_traffic_is_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"__global__ void k() {}\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "k_traffic.md").write_text(
        f"# traffic\n\ndram_bytes_per_launch: 2320549888\nkernel_source_sha256: {digest}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k_traffic.md", "kernel.cu") == 2320549888.0
    src.write_bytes(b"__global__ void k() { /* changed */ }\n")  # counters no longer describe it
    assert bench.profiled_traffic("k_traffic.md", "kernel.cu") is None
    assert bench.profiled_traffic("missing.md", "kernel.cu") is None


def test_algorithmic_byte_and_flop_counts():
    # q, k, v, o bf16 (4 x 256 B) + g fp32 (512 B) + beta (4 B) per token-head
    assert bench.BYTES_PER_TOKEN_HEAD == 1540
    assert bench.GDN_BYTES_PER_TOKEN_HEAD == 1032
    # the pages' per-head training count 6 d^2 + 3 C d + C^2 at d = 128, C = 64
    assert bench.FLOP_PER_TOKEN_HEAD == 126976
