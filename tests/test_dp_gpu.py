"""Data-parallel shard entry points on one GPU.

gh_ce_fwd_bwd_shard / gh_linear_ce_shard divide the mean by a total count the
caller passes; with a total of twice the local count the loss and gradients
are the oracle's for scale 1 / (2 n_valid).  With the local count they are
bitwise those of gh_ce_fwd_bwd / gh_linear_ce.  gh_linear_ce_shard_f32 returns
the weight gradient's unrounded fp32 sum (rounded once by gh_cast_f32_to_bf16
it is the bf16 entry point's); its sliced form (the last weight-gradient
contraction in ranges of weight rows, a callback after each) is bitwise the
same.  The data-parallel functional
wrappers on a one-rank NCCL group (the all-reduces are then identities) give
the same results as the single-process functions.
"""
import socket

import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
import oracle
from ce_check import check_grad, check_loss, grad_to_f64, loss_atol, row_eps, to_device
from lm_head_cross_gh_b200 import functional as GF

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("path", ["rows", "ring"])
def test_ce_shard_divides_by_the_given_total(cuda_device, monkeypatch, path):
    monkeypatch.setenv("GH_CE_PATH", path)
    p = gh_synth.ce_normal(300, 5003, 3.0, dtype="bf16", ignore_frac=0.1, z_loss=1e-4, seed=11)
    x, t = to_device(p)
    n_local = int((p.targets != p.ignore_index).sum())
    assert gh.gh_count_valid(t, p.V, p.ignore_index).item() == n_local
    total = torch.tensor(2 * n_local, dtype=torch.int64, device="cuda")
    loss, grad = gh.gh_ce_fwd_bwd_shard(x, t, total, p.ignore_index, "mean", 1e-4)
    torch.cuda.synchronize()
    xv = p.values_f32().astype(np.float64)
    scale = 1.0 / (2 * n_local)
    lse, rl, g_ref = oracle.ce_rows(xv, p.targets, p.ignore_index, 1e-4, scale)
    valid = p.targets != p.ignore_index
    eps = row_eps(xv)
    check_loss(loss.item(), float(rl.sum()) * scale, loss_atol(eps, lse, valid, "sum") * scale, "shard loss")
    check_grad(grad_to_f64(grad), g_ref, "bf16", scale, p.targets, p.ignore_index, eps, "shard grad")
    own = torch.tensor(n_local, dtype=torch.int64, device="cuda")
    l1, g1 = gh.gh_ce_fwd_bwd_shard(x, t, own, p.ignore_index, "mean", 1e-4)
    l2, g2 = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, "mean", 1e-4)
    torch.cuda.synchronize()
    assert l1.item() == l2.item() and torch.equal(g1.view(torch.int16), g2.view(torch.int16))


def test_linear_ce_shard_with_the_local_count_is_linear_ce(cuda_device):
    q = gh_synth.linear_ce_normal(700, 128, 3001, chunk=256, ignore_frac=0.05, w_sigma=0.05, z_loss=1e-4, seed=12)
    X = torch.from_numpy(q.inputs.view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(q.weight.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(q.targets).cuda()
    n = gh.gh_count_valid(t, q.V, -100)
    a = gh.gh_linear_ce_shard(X, W, t, n, -100, "mean", 1e-4, 256, "fp32")
    b = gh.gh_linear_ce(X, W, t, -100, "mean", 1e-4, 256, "fp32")
    torch.cuda.synchronize()
    assert a[0].item() == b[0].item() and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


@pytest.mark.parametrize("chunk", [256, 0])
def test_linear_ce_shard_f32_returns_the_unrounded_weight_gradient(cuda_device, chunk):
    """The fp32 shard entry point's weight gradient is the fp32 sum over the
    chunks: against the oracle (scale 1 / (2 n_valid)), and rounded once it is
    bitwise the bf16 shard entry point's."""
    q = gh_synth.linear_ce_normal(700, 128, 3001, chunk=chunk, ignore_frac=0.05, w_sigma=0.05, z_loss=1e-4, seed=15)
    X = torch.from_numpy(q.inputs.view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(q.weight.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(q.targets).cuda()
    n_local = int((q.targets != -100).sum())
    total = torch.tensor(2 * n_local, dtype=torch.int64, device="cuda")
    l32, dx32, dw32 = gh.gh_linear_ce_shard_f32(X, W, t, total, -100, "mean", 1e-4, chunk)
    l16, dx16, dw16 = gh.gh_linear_ce_shard(X, W, t, total, -100, "mean", 1e-4, chunk, "fp32")
    torch.cuda.synchronize()
    assert dw32.dtype == torch.float32
    assert l32.item() == l16.item() and torch.equal(dx32, dx16)
    assert torch.equal(gh.gh_cast_f32_to_bf16(dw32), dw16)
    Xd = gh_synth.bf16_to_f32(q.inputs).astype(np.float64)
    Wd = gh_synth.bf16_to_f32(q.weight).astype(np.float64)
    r = oracle.linear_cross_entropy(Xd, Wd, q.targets, -100, "sum", 1e-4, chunk, "fp32")
    ref = r["grad_weight"] / (2 * n_local)   # "sum" scaled by the batch's mean factor
    got = dw32.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref) <= 1e-2 * np.linalg.norm(ref)


@pytest.mark.parametrize("chunk,slices,max_sms", [(256, 3, 0), (0, 1, 0), (256, 1000, 20), (0, 5, 41)])
def test_linear_ce_shard_f32_sliced_is_bitwise_the_unsliced_call(cuda_device, chunk, slices, max_sms):
    """The last weight-gradient contraction cut into ranges of weight rows (on
    fewer SMs) gives bitwise the single launch's results; the callbacks come in
    order, once per range, cover [0, V) and start at multiples of 128 (whole
    256-row tiles here)."""
    q = gh_synth.linear_ce_normal(700, 128, 3001, chunk=chunk, ignore_frac=0.05, w_sigma=0.05, z_loss=1e-4, seed=16)
    X = torch.from_numpy(q.inputs.view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(q.weight.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(q.targets).cuda()
    total = torch.tensor(int((q.targets != -100).sum()), dtype=torch.int64, device="cuda")
    la, dxa, dwa = gh.gh_linear_ce_shard_f32(X, W, t, total, -100, "mean", 1e-4, chunk)
    ranges = []
    lb, dxb, dwb = gh.gh_linear_ce_shard_f32(X, W, t, total, -100, "mean", 1e-4, chunk,
                                             on_slice=lambda v0, v1: ranges.append((v0, v1)),
                                             dw_slices=slices, max_sms=max_sms)
    torch.cuda.synchronize()
    tiles = (3001 + 255) // 256
    k = min(slices, tiles)
    assert len(ranges) == k and ranges[0][0] == 0 and ranges[-1][1] == 3001
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    assert all(v0 % 256 == 0 and v1 > v0 for v0, v1 in ranges)
    assert la.item() == lb.item() and torch.equal(dxa, dxb)
    assert torch.equal(dwa.view(torch.int32), dwb.view(torch.int32))


def test_linear_ce_shard_f32_sliced_stops_on_a_callback_error(cuda_device):
    q = gh_synth.linear_ce_normal(300, 64, 1500, chunk=0, seed=17)
    X = torch.from_numpy(q.inputs.view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(q.weight.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(q.targets).cuda()
    total = torch.tensor(int((q.targets != -100).sum()), dtype=torch.int64, device="cuda")
    calls = []

    def fail(v0, v1):
        calls.append((v0, v1))
        raise RuntimeError("reduction could not start")

    with pytest.raises(RuntimeError, match="could not start"):
        gh.gh_linear_ce_shard_f32(X, W, t, total, -100, "mean", 0.0, 0, on_slice=fail, dw_slices=3)
    torch.cuda.synchronize()
    assert calls == [(0, 512)]  # the call stopped at the first range


def test_cast_f32_to_bf16_rounds_to_nearest_even(cuda_device):
    g = torch.Generator().manual_seed(0)
    x = torch.randn(100003, generator=g) * torch.exp(torch.randn(100003, generator=g) * 8)
    x[:6] = torch.tensor([0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.0e38, -1.0e-40])
    xd = x.cuda()
    got = gh.gh_cast_f32_to_bf16(xd)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), xd.to(torch.bfloat16).view(torch.int16))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_data_parallel_wrappers_on_one_rank(cuda_device):
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        p = gh_synth.ce_normal(400, 2003, 3.0, dtype="bf16", ignore_frac=0.1, z_loss=1e-4, seed=13)
        x, t = to_device(p)
        xa, xb = x.clone().requires_grad_(True), x.clone().requires_grad_(True)
        la = GF.data_parallel_cross_entropy(xa, t, -100, "mean", 1e-4)
        lb = GF.cross_entropy(xb, t, -100, "mean", 1e-4)
        (la + lb).backward()
        torch.cuda.synchronize()
        assert la.item() == lb.item() and torch.equal(xa.grad, xb.grad)

        q = gh_synth.linear_ce_normal(512, 128, 3001, chunk=0, ignore_frac=0.05, w_sigma=0.05, seed=14)
        X = torch.from_numpy(q.inputs.view(np.int16)).cuda().view(torch.bfloat16)
        W = torch.from_numpy(q.weight.view(np.int16)).cuda().view(torch.bfloat16)
        tq = torch.from_numpy(q.targets).cuda()
        Xa, Wa = X.clone().requires_grad_(True), W.clone().requires_grad_(True)
        Xb, Wb = X.clone().requires_grad_(True), W.clone().requires_grad_(True)
        ma = GF.data_parallel_chunked_linear_cross_entropy(Xa, Wa, tq)
        mb = GF.chunked_linear_cross_entropy(Xb, Wb, tq)
        (ma + mb).backward()
        torch.cuda.synchronize()
        assert ma.item() == mb.item()
        assert torch.equal(Xa.grad, Xb.grad) and torch.equal(Wa.grad, Wb.grad)
    finally:
        dist.destroy_process_group()
