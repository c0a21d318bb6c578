"""Host-side helpers of bench.py (CPU): the heads path chosen per row count,
the launch count a step claims, and the rule that a DRAM-traffic capture is
used only while the heads sources match the digest recorded with it."""
import glob
import os

import pytest

import bench
from seeded_inputs.workloads import WORKLOADS


def test_heads_path_by_row_count():
    assert bench.heads_path(1) == "stream"
    assert all(bench.heads_path(m) == "weights-as-m" for m in (2, 10, 32))
    assert all(bench.heads_path(m) == "row-tiles" for m in (33, 128, 520))


@pytest.mark.parametrize("name,launches", [("llama3-70b", 7), ("llama3-8b", 7), ("llama3-70b-chain", 7),
                                           ("llama3-70b-sampled", 7), ("llama3-70b-rejection", 6), ("tiny", 7)])
def test_step_launch_count(name, launches):
    # heads 3 (residual block, projection with the top-k, merge), tree build 1,
    # one tensor-core attention kernel, acceptance 2 (1 for the rejection walk)
    assert bench.step_launches(WORKLOADS[name]) == launches


def test_traffic_profiles_parse_and_are_not_below_the_algorithmic_bytes():
    paths = sorted(glob.glob(os.path.join(bench.PROFILE_DIR, "heads_traffic_*.md")))
    assert paths
    for p in paths:
        rec = bench._traffic_record(p)
        assert rec and len(rec.get("heads_source_digest", "")) == 16, p
        assert float(rec["traffic_per_algorithmic_byte"]) >= 0.99, p


def test_traffic_capture_is_dropped_when_the_sources_change(monkeypatch):
    w = WORKLOADS["llama3-70b"]
    rec = bench._traffic_record(os.path.join(bench.PROFILE_DIR, f"heads_traffic_{w.name}.md"))
    monkeypatch.setattr(bench, "heads_source_digest", lambda path: rec["heads_source_digest"])
    got, src = bench.measured_heads_traffic(w)
    assert got == float(rec["traffic_per_call_bytes"]) and "this workload" in src
    monkeypatch.setattr(bench, "heads_source_digest", lambda path: "0" * 16)
    assert bench.measured_heads_traffic(w) == (None, None)
