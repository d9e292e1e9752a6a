"""Host-side checks of bench.py and the committed profile summaries (no GPU).

* `bench.py --impl reference` (the float64 oracle on host cores) prints one JSON
  line with the contract's keys, for the CE and the linear-CE workloads and for
  the forward-only operations.
* Every summary under profiles/ gives the ncu command it came from; every DRAM
  traffic figure bench.py reports comes from profiles/traffic.json, whose
  entries are backed by a summary with the same figure, digest and workload.
"""
import glob
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def run_reference(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("args", [("--workload", "ce_small"), ("--workload", "ce_small", "--op", "fwd"),
                                  ("--workload", "ce_small", "--op", "select")])
def test_reference_arm_json_contract(args):
    d = run_reference(*args, "--steps", "3", "--warmup", "3")
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("ce_small")


def test_reference_arm_linear_ce_sample():
    d = run_reference("--workload", "linear_ce_gpt2", "--steps", "1", "--warmup", "3")
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["config"]["N"] == 8192


def test_profile_summaries_state_their_command_and_source():
    files = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))
    assert files
    for f in files:
        txt = open(f).read()
        assert "ncu " in txt, f"{f} does not give the ncu command"


def test_traffic_entries_are_backed_by_a_summary_and_read_back():
    """Every DRAM-traffic figure bench.py reports comes from profiles/traffic.json;
    each entry names the summary that holds the same figure, its source digest
    and its workload, and bench.profiled_traffic returns it for exactly that
    (kernel, digest, workload)."""
    import bench
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        entries = json.load(fh)["entries"]
    assert entries
    for e in entries:
        txt = open(os.path.join(ROOT, "profiles", e["summary"])).read()
        assert str(e["traffic_bytes_per_launch"]) in txt, e
        assert e["source_sha"] in txt and e["workload"] in txt, e
        assert bench.profiled_traffic(e["kernel"], e["source_sha"], e["workload"]) == \
            float(e["traffic_bytes_per_launch"])
        assert bench.profiled_traffic(e["kernel"], "0" * 12, e["workload"]) is None
