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


# --------------------------------------------------------------------------
# the roofline arithmetic bench.py reports (no GPU: fake timings)
# --------------------------------------------------------------------------

def test_linear_roofline_is_the_whole_step_over_the_burst_peak():
    """frac = 6 N V D per step / step time / the dense bf16 peak (burst for a
    timed region under two seconds, sustained beyond, and labelled so); each
    GEMM's own rate is its third of the step's FLOPs over its launches; the
    step's DRAM traffic is the profiled bytes of each GEMM launch times its
    launches per step."""
    import types
    import bench
    N, V, D, steps = 8192, 50257, 768, 20
    flops = 6.0 * N * V * D
    case = types.SimpleNamespace(flops_per_step=flops,
                                 p=types.SimpleNamespace(name="linear_ce_gpt2_8192x768x50257"))
    # per step: 4 logits launches of 0.15 ms, 4 dX of 0.12 ms, 2 dW of 0.21 ms, 4 finalizes of 0.01 ms
    kern = {"logits_gemm": (steps * 4 * 0.15, steps * 4), "dx_gemm": (steps * 4 * 0.12, steps * 4),
            "dw_gemm": (steps * 2 * 0.21, steps * 2), "chunk_ce": (steps * 4 * 0.01, steps * 4)}
    pk = dict(bench.FALLBACK_PEAKS)
    step_ms = 1.6
    r = bench.linear_roofline(case, step_ms * steps, kern, steps, pk, "fallback")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(flops / (step_ms * 1e-3) / 1e12)
    assert r["peak"] == pk["bf16_tflops"] and "burst" in r["peak_source"]
    assert r["frac"] == pytest.approx(r["achieved"] / pk["bf16_tflops"])
    lg = r["kernels"]["logits_gemm"]
    assert lg["launches_per_step"] == 4 and lg["ms_per_step"] == pytest.approx(0.6)
    assert lg["tflops"] == pytest.approx(flops / 3 / 4 / (0.15e-3) / 1e12)
    assert r["kernels"]["dw_gemm"]["tflops"] == pytest.approx(flops / 3 / 2 / (0.21e-3) / 1e12)
    assert "tflops" not in r["kernels"]["chunk_ce"]
    per = {k: bench.profiled_traffic(k, r["source_sha"], case.p.name) for k in bench.GEMM_KINDS}
    if all(v is not None for v in per.values()):
        assert r["traffic"] == pytest.approx(4 * per["logits_gemm"] + 4 * per["dx_gemm"] + 2 * per["dw_gemm"])
    else:
        assert r["traffic"] is None
    # a timed region of two seconds or more is compared with the sustained peak
    long = bench.linear_roofline(case, 2500.0, kern, steps, pk, "fallback")
    assert long["peak"] == pk["bf16_tflops_sustained"] and "sustained" in long["peak_source"]


def test_ce_roofline_is_algorithmic_bytes_over_the_kernel_time(monkeypatch):
    """achieved = the step's algorithmic bytes (valid rows read once, every
    gradient row written once, targets) over the CE kernel's mean launch time;
    frac against the copy bandwidth; traffic looked up for the kernel's digest."""
    import types
    import bench
    monkeypatch.setattr(bench, "ce_kernel_of",
                        lambda case, dev: ("ce_ring2_kernel", ["lm_head_cross_gh_b200/csrc/ce_ring.cu",
                                                                "lm_head_cross_gh_b200/csrc/ce_device.cuh",
                                                                "lm_head_cross_gh_b200/csrc/common.cuh"]))
    case = types.SimpleNamespace(bytes_per_step=1_630_503_130, op="fwd_bwd",
                                 p=types.SimpleNamespace(name="ce_gpt2_bf16_8192x50257"))
    pk = dict(bench.FALLBACK_PEAKS)
    r = bench.ce_roofline(case, {"ce_row": (20 * 0.3, 20)}, 20, pk, "fallback", 0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["kernel"] == "ce_ring2_kernel"
    assert r["kernel_ms"] == pytest.approx(0.3)
    assert r["achieved"] == pytest.approx(1_630_503_130 / 0.3e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / pk["hbm_gbs"]) and r["peak_source"] == "fallback (copy)"
    assert r["traffic"] == bench.profiled_traffic("ce_ring2_kernel", r["source_sha"], case.p.name)


def test_peaks_prefer_the_measured_file(monkeypatch, tmp_path):
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk, kind = bench.peaks()
    assert kind == "fallback" and pk == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6543.4, "bf16_tflops": 1637.0}))
    pk, kind = bench.peaks()
    assert kind == "measured" and pk["hbm_gbs"] == 6543.4


def test_source_digest_ignores_comments_and_layout_only(tmp_path, monkeypatch):
    """The digest that keys profiled DRAM traffic to the kernel source: a
    comment or whitespace edit keeps it (a capture stays valid), any code edit
    changes it (the capture no longer describes the kernel), and comment
    markers inside string literals are code."""
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = ('// header comment\n__global__ void k(float* p) {\n  /* block\n comment */ p[0] = 1.0f;  // tail\n'
           '  printf("// not a comment /* either */");\n}\n')
    (tmp_path / "a.cu").write_text(src)
    d0 = bench.source_digest(["a.cu"])
    (tmp_path / "a.cu").write_text(src.replace("// header comment", "// reworded header").replace("  p[0]", "    p[0]"))
    assert bench.source_digest(["a.cu"]) == d0
    (tmp_path / "a.cu").write_text(src.replace("1.0f", "2.0f"))
    assert bench.source_digest(["a.cu"]) != d0
    (tmp_path / "a.cu").write_text(src.replace("/* either */", "/* neither */"))
    assert bench.source_digest(["a.cu"]) != d0
