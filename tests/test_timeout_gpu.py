"""The bounded-wait failure path, on the GPU, without faulting or hanging it.

Every device-side wait in the library gives up after a time limit: the kernel
records GH_ERR_TIMEOUT in the device status word, stops all its roles, lets the
copies it has in flight land, finishes or abandons its tensor-core work, frees
TMEM and returns, and the CUDA context stays usable.  These tests make one wait
run out on purpose (gh_debug_set: a 1 ms wait limit, and one copy that the
producer leaves out, so nothing ever completes the barrier a consumer waits on)
and check that

* the call reports GH_ERR_TIMEOUT through gh_get_device_status;
* the next normal call, with the default limit back, is correct (against the
  float64 oracle) and leaves the status clean.

Covered: the two-pass cross-entropy ring (a consumer group waits for a piece
that is never copied) and the linear cross-entropy GEMM on both layouts (the
MMA issuer waits for a stage whose operands are never loaded).
"""
import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
import oracle
from ce_check import check_problem_full, grad_to_f64, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture
def short_waits():
    gh.gh_get_device_status()  # start from a clean status word
    gh.gh_debug_set("wait_limit_ns", 1_000_000)
    try:
        yield
    finally:
        gh.gh_debug_set("withhold_ring_piece", -1)
        gh.gh_debug_set("withhold_gemm_stage", -1)
        gh.gh_debug_set("wait_limit_ns", 0)


def test_ring_consumer_wait_runs_out(cuda_device, short_waits, monkeypatch):
    monkeypatch.setenv("GH_CE_PATH", "ring")
    p = gh_synth.ce_normal(1200, 4099, 3.0, dtype="bf16", ignore_frac=0.05, reduction="mean", z_loss=1e-4, seed=31)
    x, t = to_device(p)
    gh.gh_debug_set("withhold_ring_piece", 5)
    gh.gh_ce_fwd_bwd(x, t, p.ignore_index, p.reduction, p.z_loss)
    assert gh.gh_get_device_status() == gh.GH_ERR_TIMEOUT
    gh.gh_debug_set("wait_limit_ns", 0)
    loss, grad = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, p.reduction, p.z_loss)
    torch.cuda.synchronize()
    check_problem_full(p, loss.item(), grad_to_f64(grad), "after the timeout")
    assert gh.gh_get_device_status() == gh.GH_OK


@pytest.mark.parametrize("mode", ["pair", "single"])
@pytest.mark.parametrize("stage", [0, 1])
def test_gemm_mma_wait_runs_out(cuda_device, short_waits, monkeypatch, mode, stage):
    monkeypatch.setenv("GH_GEMM", mode)
    q = gh_synth.linear_ce_normal(700, 128, 3001, chunk=512, ignore_frac=0.05, x_sigma=1.0, w_sigma=0.05,
                                  z_loss=1e-4, seed=32)
    X = torch.from_numpy(q.inputs.view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(q.weight.view(np.int16)).cuda().view(torch.bfloat16)
    T = torch.from_numpy(q.targets).cuda()
    gh.gh_debug_set("withhold_gemm_stage", stage)
    gh.gh_linear_ce(X, W, T, q.ignore_index, q.reduction, q.z_loss, q.chunk, q.accum)
    assert gh.gh_get_device_status() == gh.GH_ERR_TIMEOUT
    gh.gh_debug_set("wait_limit_ns", 0)
    loss, dX, dW = gh.gh_linear_ce(X, W, T, q.ignore_index, q.reduction, q.z_loss, q.chunk, q.accum)
    torch.cuda.synchronize()
    assert gh.gh_get_device_status() == gh.GH_OK
    r = oracle.linear_cross_entropy(gh_synth.bf16_to_f32(q.inputs), gh_synth.bf16_to_f32(q.weight), q.targets,
                                    q.ignore_index, q.reduction, q.z_loss, q.chunk, q.accum)
    assert abs(loss.item() - r["loss"]) <= 1e-3 * abs(r["loss"])
    for got, want in ((dX, r["grad_inputs"]), (dW, r["grad_weight"])):
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(g - want) <= 1e-2 * np.linalg.norm(want)


def test_debug_knobs_reject_unknown(cuda_device):
    with pytest.raises(KeyError):
        gh.gh_debug_set("no_such_knob", 1)
    assert gh.lib().gh_debug_set(99, 1) == gh.GH_ERR_INVALID_ARG
