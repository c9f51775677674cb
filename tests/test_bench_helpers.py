"""Host-side helpers of bench.py on the CPU: the component statistic and the
reading of DRAM traffic from a committed ncu summary (reported only while the
summary's source digest matches the kernel source)."""
from __future__ import annotations

import os

import bench


def test_component_time_median_and_mean():
    sec, mean_ms = bench.component_time([3.0, 1.0, 2.0])
    assert sec == 2.0e-3 and mean_ms == 2.0
    sec, mean_ms = bench.component_time([4.0, 1.0, 2.0, 3.0])
    assert sec == 2.5e-3 and mean_ms == 2.5
    # One slow launch moves the mean, not the median.
    sec, mean_ms = bench.component_time([1.0, 1.0, 1.0, 1.0, 9.0])
    assert sec == 1.0e-3 and mean_ms == 2.6


def _tree(tmp_path, src_text: bytes, digest: str, dram: str):
    csrc = tmp_path / "exact_io_aware_101_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_bytes(src_text)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k.md").write_text("# k\n\nsource_sha256_16: %s   (k.cu)\ndram_bytes_per_launch: %s\n"
                               % (digest, dram))


def test_profiled_traffic_follows_the_source_digest(tmp_path, monkeypatch):
    import hashlib
    src = b"__global__ void k() {}\n"
    digest = hashlib.sha256(src).hexdigest()[:16]
    _tree(tmp_path, src, digest, "123456")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.source_digest("k.cu") == digest
    assert bench.profiled_traffic("k.md", "k.cu") == 123456.0
    # The kernel changed since the capture: no traffic figure.
    (tmp_path / "exact_io_aware_101_b200" / "csrc" / "k.cu").write_bytes(src + b"// edit\n")
    assert bench.profiled_traffic("k.md", "k.cu") is None
    # No summary at all.
    assert bench.profiled_traffic("missing.md", "k.cu") is None


def test_committed_summaries_name_a_digest_and_bytes():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for name in ("prefill_bf16_mha_n8192.md", "decode_paged_gqa.md", "decode_q8_gqa.md",
                 "prefill_chunked_gqa.md"):
        text = open(os.path.join(root, "profiles", name)).read()
        assert "source_sha256_16:" in text and "dram_bytes_per_launch:" in text, name
        assert "--clock-control none" in text, name
