"""GPU parity of gh_ce_fwd_bwd against the float64 oracle (through the C ABI).

Covers the small fp32 workload, ragged vocabulary sizes around every vector and
chunk boundary, every kernel path (one CTA per row, a cluster of CTAs per row,
the two-pass streaming path for very long rows, and the two-pass ring pipeline,
each case run on the row kernel and on the ring), in-place gradients, a
gradient buffer whose 16-byte phase differs from the logits', ignored and
out-of-range targets, determinism, and the full-size GPT-2 and large-vocabulary
workloads on sampled rows.
"""
import os

import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
import oracle
from ce_check import check_grad, check_loss, check_problem_full, grad_to_f64, loss_atol, row_eps, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["rows", "ring"])
def ce_path(request, monkeypatch):
    """Every case on both forward+backward kernels: the row kernel (a row, or a
    cluster's slices of it, resident in shared memory; the two-pass streaming
    kernel beyond) and the two-pass ring pipeline (the second pass from L2)."""
    monkeypatch.setenv("GH_CE_PATH", request.param)
    return request.param


def run(p, **kw):
    x, t = to_device(p)
    loss, grad = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, p.reduction, p.z_loss, **kw)
    torch.cuda.synchronize()
    return loss.item(), grad


@pytest.mark.parametrize("z", [0.0, 1e-4])
def test_small_fp32_workload(cuda_device, z):
    p = gh_synth.ce_small(z_loss=z)
    loss, grad = run(p)
    check_problem_full(p, loss, grad_to_f64(grad), "ce_small")
    assert gh.gh_get_device_status() == gh.GH_OK


VS = [1, 2, 3, 7, 8, 9, 15, 16, 17, 31, 33, 100, 1000, 1023, 1025, 4097, 8191, 16385, 32769, 50257]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", VS)
def test_ragged_vocab_sizes(cuda_device, dtype, V):
    B = 13 if V < 20000 else 5
    for z, red in ((0.0, "mean"), (1e-3, "sum")):
        p = gh_synth.ce_normal(B, V, 3.0, dtype=dtype, ignore_frac=0.2, reduction=red, z_loss=z, seed=V)
        loss, grad = run(p)
        check_problem_full(p, loss, grad_to_f64(grad), f"{dtype} V={V} z={z}")


@pytest.mark.parametrize("dtype,V,B", [("bf16", 65537, 4), ("bf16", 262144, 3), ("f32", 100003, 3),
                                       ("bf16", 400000, 2)])
def test_cluster_paths(cuda_device, dtype, V, B):
    p = gh_synth.ce_normal(B, V, 4.0, dtype=dtype, ignore_frac=0.0, reduction="mean", z_loss=1e-4, seed=3)
    loss, grad = run(p)
    check_problem_full(p, loss, grad_to_f64(grad), f"cluster {dtype} V={V}")


@pytest.mark.parametrize("dtype,V,B", [("bf16", 5003, 1500), ("f32", 30011, 700), ("bf16", 100003, 700),
                                       ("bf16", 262147, 300),
                                       # slices whose chunk count straddles 1024 from row to row
                                       ("bf16", 8187, 1500), ("f32", 4093, 1500)])
def test_many_rows_per_persistent_cta(cuda_device, dtype, V, B):
    # more rows than resident CTAs: each CTA cycles both slice buffers many
    # times, with ignored rows (no copy, no cluster exchange) interleaved
    p = gh_synth.ce_normal(B, V, 3.0, dtype=dtype, ignore_frac=0.3, reduction="mean", z_loss=1e-4, seed=V)
    loss, grad = run(p)
    check_problem_full(p, loss, grad_to_f64(grad), f"persistent {dtype} V={V} B={B}")


@pytest.mark.parametrize("dtype,V", [("bf16", 1_200_003), ("f32", 600_001)])
def test_streaming_path_for_very_long_rows(cuda_device, dtype, V):
    p = gh_synth.ce_normal(3, V, 3.0, dtype=dtype, ignore_frac=0.0, reduction="sum", z_loss=1e-4, seed=4)
    loss, grad = run(p)
    check_problem_full(p, loss, grad_to_f64(grad), f"stream {dtype} V={V}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_in_place_gradient(cuda_device, dtype):
    p = gh_synth.ce_normal(17, 5003, 2.0, dtype=dtype, ignore_frac=0.2, z_loss=1e-4, seed=5)
    x, t = to_device(p)
    loss, grad = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, p.reduction, p.z_loss, grad=x)
    torch.cuda.synchronize()
    assert grad.data_ptr() == x.data_ptr()
    check_problem_full(p, loss.item(), grad_to_f64(x), "in-place")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gradient_buffer_with_different_alignment(cuda_device, dtype):
    p = gh_synth.ce_normal(9, 3001, 2.0, dtype=dtype, ignore_frac=0.2, z_loss=1e-4, seed=6)
    x, t = to_device(p)
    store = torch.empty(x.numel() + 8, dtype=x.dtype, device=x.device)
    g = store[1:1 + x.numel()].view_as(x)  # 16-byte phase differs from x's
    loss, _ = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, p.reduction, p.z_loss, grad=g)
    torch.cuda.synchronize()
    check_problem_full(p, loss.item(), grad_to_f64(g), "offset grad")


def test_all_rows_ignored_and_single_row(cuda_device):
    p = gh_synth.ce_normal(6, 777, 2.0, dtype="bf16", seed=7)
    p.targets[:] = -100
    loss, grad = run(p)
    assert loss == 0.0 and not grad.any().item()
    q = gh_synth.ce_normal(1, 50257, 3.0, dtype="bf16", z_loss=1e-4, seed=8)
    loss, grad = run(q)
    check_problem_full(q, loss, grad_to_f64(grad), "B=1")


def test_ignore_index_inside_class_range(cuda_device):
    p = gh_synth.ce_normal(20, 300, 2.0, dtype="f32", seed=9, ignore_index=5)
    p.targets[::3] = 5
    loss, grad = run(p)
    check_problem_full(p, loss, grad_to_f64(grad), "ii=5")


def test_out_of_range_target_is_flagged_and_ignored(cuda_device):
    gh.gh_get_device_status()
    p = gh_synth.ce_normal(8, 100, 2.0, dtype="f32", seed=10)
    p.targets[3] = 100
    p.targets[5] = -7
    loss, grad = run(p)
    assert gh.gh_get_device_status() == gh.GH_ERR_TARGET_RANGE
    assert gh.gh_get_device_status() == gh.GH_OK  # reading clears it
    q = gh_synth.CEInputs(p.name, p.dtype, p.logits, p.targets.copy(), p.ignore_index, p.reduction, p.z_loss)
    q.targets[[3, 5]] = p.ignore_index
    check_problem_full(q, loss, grad_to_f64(grad), "out-of-range treated as ignored")


def test_empty_batch_writes_zero_loss(cuda_device):
    x = torch.empty(0, 10, dtype=torch.bfloat16, device="cuda")
    t = torch.empty(0, dtype=torch.int64, device="cuda")
    loss = torch.full((), 7.0, device="cuda")
    gh.gh_ce_fwd_bwd(x, t, loss=loss)
    assert loss.item() == 0.0


@pytest.mark.parametrize("V", [50257, 65543])
def test_nan_logit_poisons_its_row_only(cuda_device, V):
    """A NaN logit in a valid row makes the loss NaN and that row's gradient
    NaN (as the definition's sum over the row does), whichever part of the
    row holds it: on the ring's long rows (65543 bf16 columns, 128 KiB) column
    1000 is evaluated on the FMA-pipe exponential and column 20000 on the MUFU
    one.  Other rows stay finite, and a NaN in an ignored row is not read."""
    p = gh_synth.ce_normal(6, V, 3.0, dtype="bf16", reduction="sum", seed=7)
    x, t = to_device(p)
    t[4] = -100
    x[4, 9] = float("nan")
    loss, grad = gh.gh_ce_fwd_bwd(x, t, -100, "sum", 0.0)
    assert torch.isfinite(loss).item() and torch.isfinite(grad).all().item()
    assert not grad[4].any().item()
    for col in (1000, 20000):
        y = x.clone()
        y[2, col] = float("nan")
        loss, grad = gh.gh_ce_fwd_bwd(y, t, -100, "sum", 0.0)
        torch.cuda.synchronize()
        assert torch.isnan(loss).item(), col
        assert torch.isnan(grad[2].float()).all().item(), col
        keep = [0, 1, 3, 5]
        assert torch.isfinite(grad[keep].float()).all().item(), col
        assert not grad[4].any().item()


def test_results_are_deterministic(cuda_device):
    p = gh_synth.ce_normal(64, 50257, 3.0, dtype="bf16", ignore_frac=0.02, z_loss=1e-4, seed=11)
    x, t = to_device(p)
    l1, g1 = gh.gh_ce_fwd_bwd(x, t, -100, "mean", 1e-4)
    l1 = l1.clone()
    g1 = g1.clone()
    l2, g2 = gh.gh_ce_fwd_bwd(x, t, -100, "mean", 1e-4)
    torch.cuda.synchronize()
    assert l1.item() == l2.item()
    assert torch.equal(g1.view(torch.int16), g2.view(torch.int16))


def test_partial_overlap_rejected_and_alloc_fault(cuda_device, monkeypatch):
    buf = torch.zeros(512, dtype=torch.bfloat16, device="cuda")
    x = buf[:256].view(4, 64)
    t = torch.zeros(4, dtype=torch.int64, device="cuda")
    with pytest.raises(gh.GhError) as e:
        gh.gh_ce_fwd_bwd(x, t, grad=buf[8:8 + 256].view(4, 64))
    assert e.value.status == gh.GH_ERR_INVALID_ARG
    monkeypatch.setenv("GH_FAULT_ALLOC", "1")
    with pytest.raises(gh.GhError) as e:
        gh.gh_ce_fwd_bwd(x, t)
    assert e.value.status == gh.GH_ERR_ALLOC
    monkeypatch.delenv("GH_FAULT_ALLOC")
    gh.gh_ce_fwd_bwd(x, t)
    torch.cuda.synchronize()


def _sampled_check(p, loss, grad, nsample=48, seed=0):
    rng = np.random.default_rng(seed)
    ign = np.nonzero(p.targets == p.ignore_index)[0]
    rows = np.unique(np.concatenate([rng.choice(p.B, nsample, replace=False), ign[:4], [0, p.B - 1]]))
    n_valid, scale = oracle.n_valid_and_scale(p.targets, p.ignore_index, p.reduction, p.V)
    x = p.values_f32(rows).astype(np.float64)
    _, _, g_ref = oracle.ce_rows(x, p.targets[rows], p.ignore_index, p.z_loss, scale)
    g = grad[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    ref = oracle.cross_entropy(p.values_f32(), p.targets, p.ignore_index, p.reduction, p.z_loss,
                               with_grad=False, row_block=64)
    valid = p.targets != p.ignore_index
    eps_all = np.concatenate([row_eps(p.values_f32(slice(r0, r0 + 256))) for r0 in range(0, p.B, 256)])
    check_grad(g, g_ref, p.dtype, scale, p.targets[rows], p.ignore_index, eps_all[rows], p.name)
    check_loss(loss, ref["loss"], loss_atol(eps_all, ref["lse"], valid, p.reduction), p.name)


@pytest.mark.slow
def test_full_size_gpt2_workload_sampled_rows(cuda_device):
    p = gh_synth.ce_gpt2()
    loss, grad = run(p)
    _sampled_check(p, loss, grad)


@pytest.mark.slow
def test_full_size_large_vocab_workload_sampled_rows(cuda_device):
    p = gh_synth.ce_large_vocab()
    loss, grad = run(p)
    _sampled_check(p, loss, grad, nsample=24)
