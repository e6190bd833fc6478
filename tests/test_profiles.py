"""The committed ncu summaries match the kernels they describe.

bench.py reports a decode kernel's DRAM traffic per launch from profiles/decode_<workload>.md
only while the kernel sources named there hash to the recorded value; a summary left behind
by a source change would silently turn `roofline.traffic` into null.  This test fails
instead, so a kernel change comes with a fresh capture."""

import os
import re

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["c5", "c3", "c4"])
def test_decode_profile_matches_current_sources(workload):
    path = os.path.join(ROOT, "profiles", "decode_%s.md" % workload)
    text = open(path).read()
    names = re.search(r"kernel_sources:\s*(.+)", text).group(1).split()
    recorded = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text).group(1)
    assert bench.kernel_source_hash(names) == recorded, (
        "profiles/decode_%s.md was captured on other kernel sources; re-take its counters" % workload)
    traffic = bench.profile_traffic(workload)
    assert traffic is not None and traffic > 0


def test_profiles_hold_text_summaries_only():
    """profiles/ keeps short text summaries (the figures used and the commands that made
    them), never raw reports."""
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        assert name.endswith((".md", ".txt")), name
        assert os.path.getsize(os.path.join(ROOT, "profiles", name)) < 64 * 1024, name
