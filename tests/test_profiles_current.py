"""The committed ncu traffic record of the forward kernel belongs to the current
kernel sources (bench.py reports the traffic only while their hash matches; a
kernel change without a new capture would silently report null), and every
profile summary names the command that made it."""
import glob
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_record_matches_the_kernel_sources():
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    assert rec["source_hash"] == bench.kernel_source_hash()
    assert rec["workloads"]["hawk_block"]["dram_bytes_per_launch"] > 0


def test_profile_summaries_state_their_command():
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        text = open(path).read()
        assert "ncu " in text or "bench.py" in text, path
        assert "--clock-control none" in text or "ncu" not in text, path
