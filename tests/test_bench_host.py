"""Host-side checks of the benchmark script (no GPU needed).

The traffic figure the bench reports is tied to a hash over the sources
that fix the fused kernel's memory traffic; the hash must find every one of
them, so that a moved or renamed function fails here rather than on the GPU.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_sources_hash_finds_every_source():
    h = bench._kernel_sources_sha256()
    assert len(h) == 64 and int(h, 16) >= 0
    assert bench.TRAFFIC["frm_nn_bytes_per_launch"] > 0


def test_timing_rules_are_enforced():
    # fewer than three warm-up steps is refused before anything runs
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2", "--steps", "1"])
