"""The committed profiler summaries that bench.py reads: every recorded DRAM traffic figure
belongs to the kernel source as it stands (bench.py reports null traffic otherwise), and
every summary names the command that produced it."""
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


def test_recorded_traffic_matches_current_sources():
    bench = _bench()
    doc = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert doc, "no recorded traffic"
    for key, ent in doc.items():
        kernel, workload = key.split("@")
        assert ent["source_sha"] == bench.source_sha(ent["sources"]), \
            f"{key}: kernel sources changed since the capture (recapture, or re-stamp if the device code is unchanged)"
        assert bench.recorded_traffic(kernel, workload) == ent["bytes_per_launch"]
        assert os.path.exists(os.path.join(ROOT, ent["from"])), ent["from"]
        assert ent["bytes_per_launch"] > 0


def test_default_workload_has_traffic():
    bench = _bench()
    assert bench.recorded_traffic("decode_kernel<true>", "mixtral-8x7b-decode") is not None


def test_every_summary_gives_its_command():
    mds = glob.glob(os.path.join(ROOT, "profiles", "*.md"))
    assert mds
    for md in mds:
        text = open(md).read()
        assert "ncu " in text and "--clock-control none" in text and "bench.py" in text, md
