"""CPU-only: the committed ncu summaries stay tied to the kernel sources they describe.

bench.py reports a kernel's DRAM traffic from profiles/traffic.json only when the entry's
source hash equals the current source's hash (it reports null otherwise), so a stale figure
is never published."""

from __future__ import annotations

import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stored_traffic_is_published_only_for_the_current_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for kernel in ("fwd", "bwd_main"):
        sha = bench.kernel_source_sha(kernel)
        for workload, e in d[kernel].items():
            assert e["dram_bytes_per_launch"] > 0
            assert os.path.exists(os.path.join(ROOT, e["capture"])), e["capture"]
            expect = e["dram_bytes_per_launch"] if e["source_sha"] == sha else None
            assert bench.stored_traffic(kernel, workload) == expect, f"{kernel} on {workload}"


def test_default_workload_traffic_is_published():
    """The dominant kernels of the default bench workload have a DRAM figure taken on the
    current sources, so the bench line's roofline.traffic is not null."""
    for kernel in ("fwd", "bwd_main"):
        assert bench.stored_traffic(kernel, bench.DEFAULT_WORKLOAD) is not None, kernel


def test_profile_summaries_are_text_and_small():
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        p = os.path.join(ROOT, "profiles", name)
        assert name.endswith((".md", ".txt", ".json")), name
        assert os.path.getsize(p) < 64 * 1024, name
