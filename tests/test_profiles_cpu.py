"""The committed profiler summaries that bench.py reads.

A recorded DRAM traffic figure belongs to one ncu capture of one kernel source.
bench.py reports null traffic once the source changes, and an entry whose
source changed is removed, not re-stamped: the only way back is a new capture,
which writes the entry and its summary together.  So every entry must match
the current sources, and the summary it names must state the same source hash
(written from the capture), the kernel, and the command that made it."""
import glob
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_for_profiles", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _entries():
    path = os.path.join(ROOT, "profiles", "traffic.json")
    return json.load(open(path)) if os.path.exists(path) else {}


def test_recorded_traffic_belongs_to_a_capture_of_the_current_sources():
    bench = _bench()
    for key, ent in _entries().items():
        kernel, workload = key.split("@", 1)
        assert ent["source_sha"] == bench.source_sha(ent["sources"]), \
            f"{key}: kernel sources changed since the capture: recapture it, or remove the entry"
        assert bench.recorded_traffic(kernel, workload) == ent["bytes_per_launch"]
        md = os.path.join(ROOT, ent["from"])
        assert os.path.exists(md), ent["from"]
        text = open(md).read()
        assert f"source_sha {ent['source_sha']}" in text, f"{ent['from']} does not state the capture's source hash"
        assert kernel in text, f"{ent['from']} does not name {kernel}"
        assert ent["bytes_per_launch"] > 0


def test_every_summary_gives_its_command():
    mds = glob.glob(os.path.join(ROOT, "profiles", "*.md"))
    assert mds
    for md in mds:
        text = open(md).read()
        assert "ncu " in text and "--clock-control none" in text and "bench.py" in text, md
