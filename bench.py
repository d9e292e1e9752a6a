#!/usr/bin/env python
"""Throughput of the next-token cross-entropy hot path on B200.

One JSON line (rank 0).  Default workload: standalone CE forward+backward on
GPT-2-shaped bf16 logits [8192, 50257] (2% ignored, mean, z-loss 1e-4).  The
same line carries, each under its own key with its own roofline and clocks:

* "linear_ce": chunked linear-CE on the GPT-2 small tied head
  ([8192, 768] x [50257, 768], chunk 2048, fp32 accumulation);
* "linear_ce_llama3_8b": the Llama-3-8B head ([16384, 4096] x [128256, 4096],
  5% ignored, chunk 4096, fp32 accumulation, z-loss 1e-4);
* "ce_large_vocab": CE forward+backward on bf16 [4096, 262144] Student-t logits
  with spikes (sum, z-loss 1e-4).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-e2e] [--no-cpu-baseline] [--no-extra]

Timing: CUDA events on the launching stream around exactly K steps, bracketed
by a barrier and a device synchronise, max over ranks.  Inputs are larger than
L2 (126 MB) for the timed workloads, so no flush runs between steps.  Kernel
durations for the roofline come from libgh's own event pairs around each
kernel, recorded over a separate run of the same K steps just before the timed
region (event records between kernels would hide the programmatic launch
overlap, so they stay out of the region that gives `value`).  The CE roofline
is the dominant kernel's algorithmic bytes over its launch time against the
measured copy bandwidth; the linear-CE roofline is the whole step's 6 N V D
FLOPs over the step time against the dense bf16 matmul peak (burst for short
timed regions), with each GEMM's own rate alongside.  With N > 1 each rank
processes its own batch (seed = rank); nothing is exchanged (weak scaling).
``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload (rank 0 only), on all host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CE tokens/s and HBM GB/s; linear-CE tokens/s and TFLOP/s vs bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

CE_WORKLOADS = {"ce_gpt2": "ce_gpt2", "ce_large_vocab": "ce_large_vocab", "ce_small": "ce_small"}
# bench name -> (generator in gh_synth, grad_weight accumulation or None for the generator's own)
LINEAR_WORKLOADS = {"linear_ce_gpt2": ("linear_ce_gpt2", None),
                    "linear_ce_gpt2_weight_accum": ("linear_ce_gpt2", "weight"),
                    "linear_ce_llama3_8b": ("linear_ce_llama3_8b", None)}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_text(src: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace collapsed, so a
    comment-only edit keeps the digest of the code it describes."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"' or c == "'":  # string or char literal, copied whole
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_digest(files):
    """sha1 (12 hex digits) of the code of `files`, comments and layout aside."""
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(code_text(fh.read()).encode())
    return h.hexdigest()[:12]


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


def profiled_traffic(kernel, digest, workload):
    """DRAM bytes per launch of `kernel` on `workload` (dram__bytes_read.sum +
    dram__bytes_write.sum of one ncu capture), from ``profiles/traffic.json``,
    if that capture was taken of the current source (same digest)."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    with open(TRAFFIC_JSON) as f:
        entries = json.load(f).get("entries", [])
    for e in entries:
        if e["kernel"] == kernel and e["source_sha"] == digest and e["workload"] == workload:
            return float(e["traffic_bytes_per_launch"])
    return None


# --------------------------------------------------------------------------
# clocks
# --------------------------------------------------------------------------

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML in a thread."""

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nvml, self._h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self.period = period_s
        self._t = None

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
                try:
                    r = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    r = n.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((sm, int(r)))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = statistics.median(s for s, _ in self.samples)
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(name for b, name in REASONS.items() if bits & b and name != "gpu_idle")
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------

class Dist:
    """One process per GPU (torchrun env vars); NCCL on GPUs, gloo on CPU (tests)."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        self.backend = None

    def init(self, backend="nccl"):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True
            self.backend = backend

    def _device(self):
        return "cuda" if self.backend == "nccl" else "cpu"

    def barrier(self):
        if self.pg:
            import torch
            import torch.distributed as dist
            if self.backend == "nccl":
                dist.barrier(device_ids=[torch.cuda.current_device()])
            else:
                dist.barrier()

    def _reduce(self, v: float, op) -> float:
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=self._device())
        dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, v: float) -> float:
        import torch.distributed as dist
        return self._reduce(v, dist.ReduceOp.MAX) if self.pg else v

    def sum(self, v: float) -> float:
        import torch.distributed as dist
        return self._reduce(v, dist.ReduceOp.SUM) if self.pg else v

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def aggregate(dist, ms_local: float, tokens_local: float):
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    ms = dist.max(ms_local)
    tokens = dist.sum(tokens_local)
    return tokens / (ms * 1e-3), ms


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

ROWS = 0  # --rows: truncate the batch (profiling cases only)


def make_ce(name, seed):
    import gh_synth
    p = getattr(gh_synth, CE_WORKLOADS[name])(seed=seed) if name != "ce_small" else gh_synth.ce_small(1e-4, seed)
    if ROWS:
        p.logits = p.logits[:ROWS].copy()
        p.targets = p.targets[:ROWS].copy()
        p.name += f"_rows{ROWS}"
    return p


def make_linear(name, seed):
    import gh_synth
    gen, accum = LINEAR_WORKLOADS[name]
    p = getattr(gh_synth, gen)(seed=seed)
    if accum is not None and accum != p.accum:
        p.accum = accum
        p.name += f"_{accum}_accum"
    if ROWS:
        p.inputs = p.inputs[:ROWS].copy()
        p.targets = p.targets[:ROWS].copy()
        p.name += f"_rows{ROWS}"
    return p


def pinned(a):
    import numpy as np
    import torch
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    return t.pin_memory()


CE_OPS = ("fwd_bwd", "fwd", "select")


def select_index(targets):
    """selective_log_softmax has no ignore_index: ignored targets select class 0."""
    import numpy as np
    return np.ascontiguousarray(np.maximum(targets, 0))


def ce_config(p, op):
    return {"workload": p.name, "op": op, "B": p.B, "V": p.V, "dtype": p.dtype, "reduction": p.reduction,
            "z_loss": p.z_loss, "ignore_index": p.ignore_index,
            "ignored_rows": int((p.targets == p.ignore_index).sum()),
            "l2": f"inputs larger than L2 ({p.B * p.V * (4 if p.dtype == 'f32' else 2) / 1e6:.0f} MB); no flush"}


ORACLE_BLOCK_ROWS = 16  # rows per task of the threaded CE oracle


def host_threads() -> int:
    """Host cores this process may use."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def ce_oracle_rows(p, op, rows, threads=1):
    """The float64 oracle on a sample of rows, for the operation `op`; blocks of
    rows run on `threads` host threads (numpy releases the GIL in its loops)."""
    import numpy as np
    import oracle
    _, scale = oracle.n_valid_and_scale(p.targets, p.ignore_index, p.reduction, p.V)

    def block(r):
        x = p.values_f32(r).astype(np.float64)
        if op == "select":
            oracle.selective_log_softmax(x, select_index(p.targets[r]))
        else:
            oracle.ce_rows(x, p.targets[r], p.ignore_index, p.z_loss, scale, with_grad=op == "fwd_bwd")

    blocks = [rows[i:i + ORACLE_BLOCK_ROWS] for i in range(0, len(rows), ORACLE_BLOCK_ROWS)]
    if threads <= 1 or len(blocks) <= 1:
        for b in blocks:
            block(b)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(block, blocks))
    return len(rows)


class CeCase:
    """Standalone CE on one batch: forward+backward (gh_ce_fwd_bwd), the loss
    alone (gh_ce_fwd) or the selected log-probabilities (gh_selective_log_softmax)."""
    kind = "ce"

    def __init__(self, name, seed, dev, op="fwd_bwd"):
        import torch
        self.op = op
        self.p = make_ce(name, seed)
        p = self.p
        self.h_x = pinned(p.logits)
        self.h_t = pinned(select_index(p.targets) if op == "select" else p.targets)
        self.x = self.h_x.to(dev, non_blocking=False)
        self.t = self.h_t.to(dev)
        self.grad = torch.empty_like(self.x) if op == "fwd_bwd" else None
        self.loss = torch.empty((), dtype=torch.float32, device=dev)
        self.h_loss = torch.empty((), dtype=torch.float32).pin_memory()
        self.sel = torch.empty(p.B, dtype=torch.float32, device=dev) if op == "select" else None
        self.h_sel = torch.empty(p.B, dtype=torch.float32).pin_memory() if op == "select" else None
        self.tokens = p.B
        es = 4 if p.dtype == "f32" else 2
        n_ign = int((p.targets == p.ignore_index).sum())
        # algorithmic bytes: every row the operation reads once (ignored rows are
        # not read by the losses), every gradient row written once, the targets,
        # and the selected values written
        if op == "fwd_bwd":
            self.bytes_per_step = ((p.B - n_ign) * p.V + p.B * p.V) * es + 8 * p.B
        elif op == "fwd":
            self.bytes_per_step = (p.B - n_ign) * p.V * es + 8 * p.B
        else:
            self.bytes_per_step = p.B * p.V * es + 12 * p.B
        self.h2d = self.h_x.numel() * self.h_x.element_size() + self.h_t.numel() * 8
        self.d2h = 4 * p.B if op == "select" else 4
        self.dtype = "bf16" if p.dtype == "bf16" else "f32"

    def _call(self):
        import lm_head_cross_gh_b200 as gh
        p = self.p
        if self.op == "fwd_bwd":
            gh.gh_ce_fwd_bwd(self.x, self.t, p.ignore_index, p.reduction, p.z_loss, grad=self.grad, loss=self.loss)
        elif self.op == "fwd":
            gh.gh_ce_fwd(self.x, self.t, p.ignore_index, p.reduction, p.z_loss, loss=self.loss)
        else:
            gh.gh_selective_log_softmax(self.x, self.t, out=self.sel)

    def step(self):
        self._call()

    def e2e_step(self):
        self.x.copy_(self.h_x, non_blocking=True)
        self.t.copy_(self.h_t, non_blocking=True)
        self._call()
        if self.op == "select":
            self.h_sel.copy_(self.sel, non_blocking=True)
        else:
            self.h_loss.copy_(self.loss, non_blocking=True)

    def config(self):
        return ce_config(self.p, self.op)

    def cpu_sample(self, budget_rows):
        import numpy as np
        return np.arange(min(self.p.B, budget_rows))

    def run_oracle(self, rows, threads=1):
        return ce_oracle_rows(self.p, self.op, rows, threads)


def linear_config(p):
    return {"workload": p.name, "N": p.N, "D": p.D, "V": p.V, "chunk": p.chunk, "accum": p.accum,
            "reduction": p.reduction, "z_loss": p.z_loss,
            "ignored_rows": int((p.targets == p.ignore_index).sum()),
            "l2": "weight and chunk logits larger than L2; no flush"}


class LinearCase:
    kind = "linear"

    def __init__(self, name, seed, dev):
        import torch
        self.p = make_linear(name, seed)
        self.h_X = pinned(self.p.inputs)
        self.h_W = pinned(self.p.weight)
        self.h_t = pinned(self.p.targets)
        self.X = self.h_X.to(dev)
        self.W = self.h_W.to(dev)
        self.t = self.h_t.to(dev)
        self.dX = torch.empty_like(self.X)
        self.dW = torch.empty_like(self.W)
        self.loss = torch.empty((), dtype=torch.float32, device=dev)
        self.h_loss = torch.empty((), dtype=torch.float32).pin_memory()
        p = self.p
        self.tokens = p.N
        self.flops_per_step = 6.0 * p.N * p.V * p.D
        self.h2d = (self.h_X.numel() + self.h_W.numel()) * 2 + self.h_t.numel() * 8
        self.d2h = 4
        self.dtype = "bf16"

    def step(self):
        import lm_head_cross_gh_b200 as gh
        p = self.p
        gh.gh_linear_ce(self.X, self.W, self.t, p.ignore_index, p.reduction, p.z_loss, p.chunk, p.accum,
                        grad_inputs=self.dX, grad_weight=self.dW, loss=self.loss)

    def e2e_step(self):
        import lm_head_cross_gh_b200 as gh
        p = self.p
        self.X.copy_(self.h_X, non_blocking=True)
        self.W.copy_(self.h_W, non_blocking=True)
        self.t.copy_(self.h_t, non_blocking=True)
        gh.gh_linear_ce(self.X, self.W, self.t, p.ignore_index, p.reduction, p.z_loss, p.chunk, p.accum,
                        grad_inputs=self.dX, grad_weight=self.dW, loss=self.loss)
        self.h_loss.copy_(self.loss, non_blocking=True)

    def config(self):
        return linear_config(self.p)

    def cpu_sample(self, budget_rows):
        import numpy as np
        return np.arange(min(self.p.N, budget_rows))

    def run_oracle(self, rows, threads=1):
        """Oracle on a row sample: the chunk's logits, CE and both gradient GEMMs
        (float64; numpy's BLAS threads, whatever `threads` says)."""
        import numpy as np
        import gh_synth
        import oracle
        p = self.p
        X = gh_synth.bf16_to_f32(p.inputs[rows]).astype(np.float64)
        W = self._W64 if hasattr(self, "_W64") else gh_synth.bf16_to_f32(p.weight).astype(np.float64)
        self._W64 = W
        oracle.linear_cross_entropy(X, W, p.targets[rows], p.ignore_index, p.reduction, p.z_loss,
                                    chunk=len(rows), accum=p.accum)
        return len(rows)


CE_RING_MIN_ROWS_PER_SM = 8  # the library's switch from the row kernel to the ring pipelines
GEMM_KINDS = ("logits_gemm", "dx_gemm", "dw_gemm")
LINEAR_KINDS = GEMM_KINDS + ("chunk_ce",)
SUSTAINED_AFTER_S = 2.0  # a timed region at least this long is compared with the sustained matmul peak


def ce_kernel_of(case, device_index):
    """(kernel name, its sources) of the CE kernel the
    library picks for this batch: the ring pipelines from 8 rows per SM up,
    the row kernel below (GH_CE_PATH overrides, as in the library)."""
    import torch
    sms = torch.cuda.get_device_properties(device_index).multi_processor_count
    forced = os.environ.get("GH_CE_PATH")
    ring = forced == "ring" or (forced != "rows" and case.p.B >= CE_RING_MIN_ROWS_PER_SM * sms)
    common = ["lm_head_cross_gh_b200/csrc/ce_device.cuh", "lm_head_cross_gh_b200/csrc/common.cuh"]
    if ring:
        name = "ce_ring2_kernel" if case.op == "fwd_bwd" else "ce_ring_kernel"
        return name, ["lm_head_cross_gh_b200/csrc/ce_ring.cu"] + common
    return "ce_row_kernel", ["lm_head_cross_gh_b200/csrc/ce.cu"] + common


LINEAR_SOURCES = ["lm_head_cross_gh_b200/csrc/gemm_sm100.cuh", "lm_head_cross_gh_b200/csrc/linear_ce.cu",
                  "lm_head_cross_gh_b200/csrc/common.cuh"]


def time_steps(case, dist, steps, warmup, clocks=None):
    """Kernel durations for the roofline, then exactly `steps` timed steps.

    The kernel pass runs the same `steps` steps with libgh's per-kernel event
    pairs on (one pass fills the library's event pool, the next is read); it
    comes right after the warm-up so it sees the same clocks as the timed
    region.  The timed region that gives `value` has no per-kernel events
    (event records between kernels would hide the programmatic launch overlap).
    """
    import torch
    import lm_head_cross_gh_b200 as gh
    for _ in range(warmup):
        case.step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    kinds = ["ce_row"] if case.kind == "ce" else list(LINEAR_KINDS)
    for rep in range(2):
        gh.gh_profile_enable(True)
        for _ in range(steps):
            case.step()
        torch.cuda.synchronize()
    gh.gh_profile_enable(False)
    kern = {}
    for k in kinds:
        tot, n = gh.gh_profile_read(k)
        kern[k] = (tot, n)
    n0 = gh.gh_launch_count()
    if clocks:
        clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        case.step()
    e1.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    dist.barrier()
    launches = gh.gh_launch_count() - n0
    # keep the clock record meaningful for short timed regions: the same work
    # continues (untimed) until ~0.5 s of samples exist
    if clocks:
        pad_t = time.perf_counter()
        while time.perf_counter() - pad_t < max(0.0, 0.5 - wall):
            case.step()
            torch.cuda.synchronize()
        clocks.stop()
    ms = e0.elapsed_time(e1)
    return ms, launches, kern


def time_e2e(case, dist, steps):
    import torch
    for _ in range(2):
        case.e2e_step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        case.e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    return e0.elapsed_time(e1)


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        blas = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        return max(blas) if blas else 1
    except Exception:
        return 1


def oracle_threads(case):
    """Threads the oracle runs on: one per host core for the CE row loops, the
    BLAS pool for linear-CE."""
    return host_threads() if case.kind == "ce" else cpu_threads()


def run_oracle_timing(case, budget_rows, reps=1):
    threads = oracle_threads(case)
    rows = case.cpu_sample(budget_rows)
    t0 = time.perf_counter()
    n = 0
    for _ in range(reps):
        n += case.run_oracle(rows, threads)
    dt = time.perf_counter() - t0
    return n / dt, len(rows), dt, threads


# Oracle rows per host thread in one timing sample (linear-CE: per sample, BLAS-threaded).
ORACLE_ROWS = {"ce_gpt2": 1024, "ce_large_vocab": 64, "ce_small": 64, "linear_ce_gpt2": 512,
               "linear_ce_gpt2_weight_accum": 512,
               "linear_ce_llama3_8b": 32}


def ce_roofline(case, kern, steps, pk, pk_kind, device_index):
    """The CE kernel's algorithmic bytes over its event-timed launch duration."""
    k_ms, k_n = kern["ce_row"]
    k_avg = k_ms / max(k_n, 1)
    achieved = case.bytes_per_step / (k_avg * 1e-3) / 1e9
    kname, ksrc = ce_kernel_of(case, device_index)
    digest = source_digest(ksrc)
    prefix = kname if kname != "ce_ring_kernel" else f"ce_ring_kernel_{case.op}"
    return {"bound": "hbm", "kernel": kname, "achieved": achieved,
            "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
            "traffic": profiled_traffic(prefix, digest, case.p.name), "algorithmic_bytes": case.bytes_per_step,
            "kernel_ms": k_avg, "peak_source": f"{pk_kind} (copy)", "source_sha": digest}


def linear_roofline(case, ms_total, kern, steps, pk, pk_kind):
    """The whole step's algorithmic FLOPs (6 N V D: logits, dX and dW GEMMs) over
    the step time, against the dense bf16 matmul peak: the burst figure for a
    timed region shorter than SUSTAINED_AFTER_S, the sustained one beyond.  Each
    GEMM's own rate (2 N V D per step over its event-timed launches) and the
    per-chunk cross-entropy kernels' time are listed alongside."""
    step_ms = ms_total / steps
    sustained = ms_total * 1e-3 >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in pk
    peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    achieved = case.flops_per_step / (step_ms * 1e-3) / 1e12
    digest = source_digest(LINEAR_SOURCES)
    parts = {}
    traffic_step = 0.0
    for k in LINEAR_KINDS:
        tot, n = kern.get(k, (0.0, 0))
        if not n:
            continue
        per_ms = tot / n
        d = {"ms_per_launch": per_ms, "launches_per_step": n / steps, "ms_per_step": tot / steps}
        if k in GEMM_KINDS:
            flops = case.flops_per_step / 3.0 * steps / n
            d["tflops"] = flops / (per_ms * 1e-3) / 1e12
            d["frac"] = d["tflops"] / peak
            tr = profiled_traffic(k, digest, case.p.name)
            d["traffic"] = tr
            traffic_step = None if (tr is None or traffic_step is None) else traffic_step + tr * n / steps
        parts[k] = d
    return {"bound": "tensor", "kernel": "whole step: logits GEMM with its cross-entropy epilogue, "
                                          "per-chunk finalize, dX and dW GEMMs",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic_step if parts else None, "algorithmic_flops": case.flops_per_step,
            "step_ms": step_ms, "kernels": parts,
            "peak_source": f"{pk_kind} bf16 ({'sustained' if sustained else 'burst'})", "source_sha": digest}


def measure(case, dist, steps, warmup, pk, pk_kind):
    """Timed steps of one workload: throughput, roofline, clocks, launches."""
    clocks = ClockSampler(dist.local)
    ms, launches, kern = time_steps(case, dist, steps, warmup, clocks)
    value, ms_max = aggregate(dist, ms, case.tokens * steps)
    out = {"workload": case.p.name, "value": value, "unit": "tokens/s", "ms_per_step": ms_max / steps,
           "steps": steps, "gpu_launches": int(launches)}
    if case.kind == "ce":
        out["roofline"] = ce_roofline(case, kern, steps, pk, pk_kind, dist.local)
        out["hbm_gbs_step"] = case.bytes_per_step * steps / (ms * 1e-3) / 1e9
    else:
        out["roofline"] = linear_roofline(case, ms_max, kern, steps, pk, pk_kind)
        out["tflops"] = out["roofline"]["achieved"]
    out["clocks"] = clocks.summary()
    return out


# Workloads the default CE line also carries (name, steps cap).
EXTRA_WORKLOADS = (("linear_ce", "linear_ce_gpt2", 20), ("linear_ce_weight_accum", "linear_ce_gpt2_weight_accum", 20),
                   ("linear_ce_llama3_8b", "linear_ce_llama3_8b", 3), ("ce_large_vocab", "ce_large_vocab", 20))


def make_case(name, seed, dev, op="fwd_bwd"):
    return CeCase(name, seed, dev, op) if name in CE_WORKLOADS else LinearCase(name, seed, dev)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="ce_gpt2", choices=list(CE_WORKLOADS) + list(LINEAR_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="fwd_bwd", choices=list(CE_OPS),
                    help="standalone CE operation timed on a CE workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", "--no-linear", dest="no_extra", action="store_true",
                    help="omit the other workloads' objects from the default CE line")
    ap.add_argument("--rows", type=int, default=0, help="use only the first ROWS rows/tokens (profiling cases)")
    ap.add_argument("--launches-only", action="store_true",
                    help="run W + K steps and exit without timing or report (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    global ROWS
    ROWS = max(0, args.rows)

    dist = Dist()
    if args.impl == "reference":
        return reference_arm(args, dist)

    import torch
    import lm_head_cross_gh_b200 as gh
    from lm_head_cross_gh_b200 import _build
    if not os.path.exists(gh.LIB_PATH):
        _build.build()
    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    dev = torch.device("cuda", dist.local)
    pk, pk_kind = peaks()

    is_ce = args.workload in CE_WORKLOADS
    case = make_case(args.workload, dist.rank, dev, args.op)
    if args.launches_only:
        for _ in range(args.warmup + args.steps):
            case.step()
        torch.cuda.synchronize()
        dist.close()
        return 0
    m = measure(case, dist, args.steps, args.warmup, pk, pk_kind)

    out = {"metric": METRIC, "value": m["value"], "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": case.dtype,
           "data": "synthetic (seeded; seed = rank)", "config": case.config()}
    out["config"]["parallelism"] = parallelism(dist.world)
    out["roofline"] = m["roofline"]
    if is_ce:
        out["hbm_gbs_step"] = m["hbm_gbs_step"]
    else:
        out["tflops"] = m["tflops"]
    out["gpu_launches"] = m["gpu_launches"]
    out["clocks"] = m["clocks"]

    if not args.no_e2e:
        k = max(1, min(args.steps, 10))
        e_ms = dist.max(time_e2e(case, dist, k))
        out["e2e"] = {"value": dist.sum(case.tokens * k) / (e_ms * 1e-3), "unit": "tokens/s",
                      "h2d_bytes_per_step": case.h2d, "d2h_bytes_per_step": case.d2h,
                      "path": "pinned host -> device copies, gh C ABI call, loss read back, per step"}

    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        v, nrows, dt, threads = run_oracle_timing(case, ORACLE_ROWS[args.workload] *
                                                  (host_threads() if is_ce else 1))
        out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                               "sample": f"first {nrows} rows of the same workload, float64 numpy oracle on "
                                         f"{threads} host threads, {dt:.1f} s"}

    if is_ce and args.workload == "ce_gpt2" and args.op == "fwd_bwd" and not args.no_extra:
        del case
        torch.cuda.empty_cache()
        for key, name, cap in EXTRA_WORKLOADS:
            try:
                extra = make_case(name, dist.rank, dev)
                st = max(3, min(args.steps, cap))
                obj = measure(extra, dist, st, args.warmup, pk, pk_kind)
                obj["config"] = extra.config()
                out[key] = obj
                del extra
            except Exception as e:  # the CE line stands on its own
                out[key] = {"workload": name, "unavailable": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()
    if dist.rank == 0:
        print(json.dumps(out), flush=True)
    dist.close()


def parallelism(world):
    return f"replicas x{world} (independent batches, no collective)"


def reference_arm(args, dist):
    """The float64 oracle on the host cores, on a bounded sample of the same workload."""
    if dist.rank != 0:
        return 0
    is_ce = args.workload in CE_WORKLOADS

    class Dummy:
        kind = "ce" if is_ce else "linear"
    case = Dummy()
    if is_ce:
        case.p = make_ce(args.workload, 0)
        case.cpu_sample = lambda n, c=case: __import__("numpy").arange(min(c.p.B, n))
        case.run_oracle = lambda rows, threads, c=case: ce_oracle_rows(c.p, args.op, rows, threads)
        config = ce_config(case.p, args.op)
    else:
        case.p = make_linear(args.workload, 0)
        case.cpu_sample = lambda n, c=case: __import__("numpy").arange(min(c.p.N, n))
        case.run_oracle = lambda rows, threads, c=case: LinearCase.run_oracle(c, rows, threads)
        config = linear_config(case.p)
    config["parallelism"] = parallelism(1)
    threads = oracle_threads(case)
    rows_per_step = max(1, ORACLE_ROWS[args.workload] // 8) * (threads if is_ce else 1)
    rows = case.cpu_sample(rows_per_step)
    for _ in range(args.warmup):
        case.run_oracle(rows, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        case.run_oracle(rows, threads)
    dt = time.perf_counter() - t0
    value = len(rows) * args.steps / dt
    sample = f"first {len(rows)} rows of {case.p.name} per step, float64 numpy oracle on {threads} host threads"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64", "data": "synthetic (seeded)", "config": config,
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
