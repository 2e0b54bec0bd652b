"""Consistency of the committed measurement records (no GPU needed).

profiles/traffic.json holds, per (kernel, workload), the DRAM bytes of one
launch from an ncu capture, the command that took it and a hash of the kernel
sources it was taken on; bench.py reports the bytes only while the hash still
matches.  These tests check that every record is well formed, names a kernel
that bench.py knows, was taken with the GPU clocks left alone, and that every
command quoted in profiles/ does the same.
"""
import json
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def _traffic():
    with open(os.path.join(PROFILES, "traffic.json")) as f:
        return json.load(f)


def test_traffic_records_are_well_formed():
    d = _traffic()
    assert d, "no traffic records"
    for key, e in d.items():
        kernel, workload = key.rsplit(":", 1)
        assert kernel.split("<")[0].split(":")[0] in bench.KERNEL_SOURCES, key
        assert workload in bench.DEFAULT_STEPS, key
        assert e["dram_bytes_per_launch"] > 0, key
        assert re.fullmatch(r"[0-9a-f]{16}", e["source_hash"]), key
        assert e["command"].startswith("ncu "), key
        assert "--clock-control none" in e["command"], key
        assert f"--workload {workload}" in e["command"], key


def test_every_quoted_ncu_command_leaves_the_clocks_alone():
    n = 0
    for name in sorted(os.listdir(PROFILES)):
        if not name.endswith(".md"):
            continue
        with open(os.path.join(PROFILES, name)) as f:
            for line in f:
                if line.lstrip().startswith("ncu --"):
                    n += 1
                    assert "--clock-control none" in line, f"{name}: {line.strip()}"
    assert n > 0


def test_profiles_hold_summaries_only():
    # short text summaries; raw captures stay out of the repository
    for name in os.listdir(PROFILES):
        assert name.endswith((".md", ".txt", ".json")), name
        assert os.path.getsize(os.path.join(PROFILES, name)) < 64 * 1024, name


def test_traffic_records_match_the_current_kernel_sources():
    # a record taken on other sources would be dropped by bench.py (traffic:
    # null); every committed record is current
    for key, e in _traffic().items():
        kernel = key.rsplit(":", 1)[0]
        assert e["source_hash"] == bench.kernel_source_hash(kernel), f"{key}: stale capture"
