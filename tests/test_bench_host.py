"""Host-side checks of bench.py and the committed profile summaries (no GPU).

* `bench.py --impl reference` (the float64 oracle on host cores) prints one JSON
  line with the contract's keys, for the CE and the linear-CE workloads and for
  the forward-only operations.
* Every summary under profiles/ gives the ncu command it came from; a summary
  that states DRAM traffic also states the source digest and the workload, and
  bench.py's parser reads it back.
"""
import glob
import json
import os
import re
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
    import bench
    files = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))
    assert files
    for f in files:
        txt = open(f).read()
        assert "ncu " in txt, f"{f} does not give the ncu command"
        if "traffic_bytes_per_launch" in txt:
            assert re.search(r"source_sha:\s*[0-9a-f]{12}", txt), f
            for m in re.finditer(r"workload:\s*(\S+)\s*\ntraffic_bytes_per_launch:\s*([0-9]+)", txt):
                sha = re.search(r"source_sha:\s*([0-9a-f]+)", txt).group(1)
                kernel = os.path.basename(f).split("_gpt2")[0].split("_fwd")[0]
                kernel = kernel if kernel != "ce_ring_kernel" else "ce_ring_kernel_fwd"
                got = bench.profiled_traffic(kernel, sha, m.group(1))
                assert got == float(m.group(2)), (f, kernel, got)
