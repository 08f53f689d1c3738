"""Host-side logic of bench.py that needs no GPU: the DRAM-traffic figure of
the roofline object comes from a committed ncu capture and is reported only
while the sources of the prefill call are those it was captured from."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_prefill_sources_exist():
    csrc = os.path.join(ROOT, "kda_linear_attention_fwd_b200", "csrc")
    for name in bench.PREFILL_SOURCES:
        assert os.path.exists(os.path.join(csrc, name)), name
    # every prefill kernel file is covered, and the plan, fold and entry points
    for name in os.listdir(csrc):
        if name.startswith("kda_prefill") or name.endswith(".cuh"):
            assert name in bench.PREFILL_SOURCES, name
    for name in ("kda_api.cu", "kda_args.h", "kda_chain.cu", "kda_plan.cu"):
        assert name in bench.PREFILL_SOURCES, name


def test_traffic_is_null_when_stale(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (tmp_path / "kda_linear_attention_fwd_b200").symlink_to(os.path.join(ROOT, "kda_linear_attention_fwd_b200"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("long_bf16") == (None, None, "no committed capture")
    h = bench.source_hash()
    entry = {"source_hash": h, "bytes_per_launch": 9.0e9, "kernel": "call", "source": "x.md"}
    (prof / "traffic.json").write_text(json.dumps({"long_bf16": entry}))
    assert bench.measured_traffic("long_bf16") == (9.0e9, "call", "x.md")
    assert bench.measured_traffic("prefill_bf16")[0] is None
    entry["source_hash"] = "0" * 16
    (prof / "traffic.json").write_text(json.dumps({"long_bf16": entry}))
    traffic, _, why = bench.measured_traffic("long_bf16")
    assert traffic is None and why.startswith("stale")


def test_committed_traffic_entries_are_complete():
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return
    with open(path) as f:
        d = json.load(f)
    for workload, e in d.items():
        assert {"source_hash", "bytes_per_launch", "kernel", "source"} <= set(e), workload
        assert os.path.exists(os.path.join(ROOT, e["source"])), e["source"]
        assert e["bytes_per_launch"] > 0


def test_clock_samples_are_taken_inside_the_timed_region(tmp_path):
    """Only nvidia-smi samples stamped between mark_start and mark_end count;
    a throttle reason seen there is reported, one outside is not."""
    import time
    from datetime import datetime
    path = tmp_path / "clocks.csv"
    t = time.time()
    with open(path, "w") as f:
        for k in range(10):
            ts = datetime.fromtimestamp(t + 0.02 * k).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            sm = 1965 if 2 <= k <= 6 else 1200
            cap = "Active" if k == 4 else "Not Active"
            slow = "Active" if k == 8 else "Not Active"
            f.write(f"{ts}, 0, {sm}, 1965, 700.0, 0x0, {slow}, Not Active, Not Active, {cap}\n")

    class Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            pass

    c = bench.Clocks(str(path))
    c.proc, c.f = Done(), open(os.devnull, "w")
    c.t0, c.t1 = t + 0.035, t + 0.125
    r = c.stop()
    assert r == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 5}
