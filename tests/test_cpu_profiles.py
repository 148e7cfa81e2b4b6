"""The ncu evidence the bench cites stays consistent: every traffic entry
names a kernel bench.py knows, a positive byte count, a 16-hex-digit source
hash and a summary file in profiles/ that records the same hash."""
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_entries_point_at_their_summaries():
    entries = []
    with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                entries.append(line.split())
    assert entries
    for name, nbytes, digest, capture in entries:
        kernel, _, workload = name.partition("@")
        assert kernel in bench.KERNEL_SOURCES, name
        assert workload, name
        assert int(nbytes) > 0, name
        assert re.fullmatch(r"[0-9a-f]{16}", digest), name
        path = os.path.join(ROOT, "profiles", capture)
        assert os.path.isfile(path), capture
        with open(path) as f:
            assert digest in f.read(), f"{capture} does not record hash {digest}"


def test_profile_summaries_give_their_commands():
    for fn in os.listdir(os.path.join(ROOT, "profiles")):
        if fn.endswith(".md"):
            with open(os.path.join(ROOT, "profiles", fn)) as f:
                text = f.read()
            assert "--clock-control none" in text, fn
            assert "bench.py" in text, fn
