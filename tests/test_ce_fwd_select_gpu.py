"""GPU parity of gh_ce_fwd (loss without gradient) and gh_selective_log_softmax
against the float64 oracle, through the C ABI.

Two kernels serve both calls: the row kernel in a forward-only mode (one CTA
per row, a cluster of CTAs per long row, the two-pass streaming kernel beyond
that; the default below 8 rows per SM) and the ring pipeline (pieces of rows
streamed through a shared-memory ring; the default from 8 rows per SM up).
The `path` fixture runs each case on both (GH_CE_PATH); the ring's own
cases cover every 16-byte phase of a row's start, rows without a whole
16-byte chunk and rows of many pieces.

Tolerances: a row's value is lse - x_t (+ z lse^2) or x_t - lse, so its error is
the error of lse, below eps_i * max(1, |lse_i|) with eps_i = 4e-7 * max(1,
max_j |x_ij|) (the kernel's fp32 exponent arithmetic; see ce_check).  The
reduced loss uses the same bound as gh_ce_fwd_bwd.  Two properties tie the
modes together: gh_ce_fwd's loss equals the forward+backward kernel's (exactly
on the row kernel, which runs the same passes 0 and 1; within 2e-6 relative on
the ring, which sums in another order), and the selected log-probability is
exactly minus the z-free row loss.
"""
import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
import oracle
from ce_check import check_loss, loss_atol, row_eps, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["rows", "ring"])
def path(request, monkeypatch):
    """Both forward-only kernels: the row kernel (clusters for long rows, the
    streaming kernel beyond them) and the ring pipeline (the default from
    8 rows per SM up)."""
    monkeypatch.setenv("GH_CE_PATH", request.param)
    return request.param


def fwd(p, rows=True):
    x, t = to_device(p)
    rl = torch.full((p.B,), 7.0, dtype=torch.float32, device="cuda") if rows else None
    loss, rl = gh.gh_ce_fwd(x, t, p.ignore_index, p.reduction, p.z_loss, row_loss=rl)
    torch.cuda.synchronize()
    return loss.item(), (rl.cpu().numpy().astype(np.float64) if rows else None)


def check_fwd(p, loss, rl, what):
    x = p.values_f32().astype(np.float64)
    ref = oracle.cross_entropy(x, p.targets, p.ignore_index, p.reduction, p.z_loss, with_grad=False)
    eps = row_eps(x).reshape(-1)
    valid = p.targets != p.ignore_index
    check_loss(loss, ref["loss"], loss_atol(eps[:, None], ref["lse"], valid, p.reduction), what)
    if rl is not None:
        tol = 1e-5 * np.abs(ref["row_loss"]) + eps * np.maximum(1.0, np.abs(ref["lse"])) * (1 + 2 * abs(p.z_loss) * np.abs(ref["lse"]))
        err = np.abs(rl - ref["row_loss"])
        assert (err <= tol).all(), f"{what} row loss worst {err.max():.3g}"
        assert (rl[~valid] == 0.0).all(), f"{what} ignored rows must be exactly 0"


VS = [1, 2, 7, 8, 9, 17, 100, 1023, 1025, 8191, 32769, 50257]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", VS)
def test_fwd_ragged_vocab_sizes(cuda_device, path, dtype, V):
    B = 13 if V < 20000 else 5
    for z, red in ((0.0, "mean"), (1e-3, "sum")):
        p = gh_synth.ce_normal(B, V, 3.0, dtype=dtype, ignore_frac=0.2, reduction=red, z_loss=z, seed=V)
        check_fwd(p, *fwd(p), f"fwd {dtype} V={V} z={z}")


@pytest.mark.parametrize("dtype,V,B", [("bf16", 262144, 3), ("f32", 100003, 3), ("bf16", 5003, 1500),
                                       ("bf16", 262147, 300), ("bf16", 1_200_003, 2), ("f32", 600_001, 2)])
def test_fwd_cluster_persistent_and_streaming_paths(cuda_device, path, dtype, V, B):
    p = gh_synth.ce_normal(B, V, 4.0, dtype=dtype, ignore_frac=0.2, reduction="mean", z_loss=1e-4, seed=V + B)
    check_fwd(p, *fwd(p), f"fwd {dtype} V={V} B={B}")


@pytest.mark.parametrize("dtype,V,B", [("bf16", 50257, 64), ("f32", 4093, 300), ("bf16", 262144, 4),
                                       ("bf16", 1_200_003, 2)])
def test_fwd_matches_forward_backward_loss(cuda_device, path, dtype, V, B):
    # the row kernel's forward mode runs the same passes 0 and 1 as its
    # forward+backward mode: identical loss.  The ring folds each thread's
    # chunks online in another order: equal within the loss tolerance.
    p = gh_synth.ce_normal(B, V, 3.0, dtype=dtype, ignore_frac=0.1, reduction="mean", z_loss=1e-4, seed=5)
    x, t = to_device(p)
    l_fb, _ = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, "mean", 1e-4)
    l_f, _ = gh.gh_ce_fwd(x, t, p.ignore_index, "mean", 1e-4)
    torch.cuda.synchronize()
    if path == "rows":
        assert l_f.item() == l_fb.item()
    else:
        assert abs(l_f.item() - l_fb.item()) <= 2e-6 * abs(l_fb.item())


def test_fwd_without_row_output_and_empty(cuda_device, path):
    p = gh_synth.ce_small(z_loss=1e-4)
    loss, _ = fwd(p, rows=False)
    check_fwd(p, loss, None, "fwd no rows")
    x = torch.empty(0, 10, dtype=torch.bfloat16, device="cuda")
    t = torch.empty(0, dtype=torch.int64, device="cuda")
    loss = torch.full((), 7.0, device="cuda")
    gh.gh_ce_fwd(x, t, loss=loss)
    assert loss.item() == 0.0


def test_fwd_all_ignored_and_out_of_range(cuda_device, path):
    gh.gh_get_device_status()
    p = gh_synth.ce_normal(9, 333, 2.0, dtype="bf16", seed=12)
    p.targets[:] = -100
    loss, rl = fwd(p)
    assert loss == 0.0 and not rl.any()
    p = gh_synth.ce_normal(9, 333, 2.0, dtype="f32", seed=13)
    p.targets[2] = 333
    loss, rl = fwd(p)
    assert gh.gh_get_device_status() == gh.GH_ERR_TARGET_RANGE
    assert rl[2] == 0.0
    q = gh_synth.CEInputs(p.name, p.dtype, p.logits, p.targets.copy(), p.ignore_index, p.reduction, p.z_loss)
    q.targets[2] = q.ignore_index
    check_fwd(q, loss, rl, "out-of-range treated as ignored")


# ---- selective_log_softmax ------------------------------------------------------------


def select(x, idx):
    out = gh.gh_selective_log_softmax(x, idx)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def check_select(xv, idx, out, what):
    """xv: float64 values [..., V]; idx int64 [...]; out float64 [...]."""
    V = xv.shape[-1]
    ref = oracle.selective_log_softmax(xv, idx)
    x2 = xv.reshape(-1, V)
    eps = row_eps(x2).reshape(-1)
    m = x2.max(axis=1)
    lse = m + np.log(np.exp(x2 - m[:, None]).sum(axis=1))
    tol = 1e-5 * np.abs(ref.reshape(-1)) + eps * np.maximum(1.0, np.abs(lse))
    err = np.abs(out.reshape(-1) - ref.reshape(-1))
    assert (err <= tol).all(), f"{what} worst {err.max():.3g}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", [1, 3, 8, 9, 100, 1025, 8191, 50257, 65537, 262144, 1_200_003])
def test_select_all_paths(cuda_device, path, dtype, V):
    B = 11 if V < 20000 else 3
    p = gh_synth.ce_normal(B, V, 3.0, dtype=dtype, seed=V + 1)
    x, t = to_device(p)
    check_select(p.values_f32().astype(np.float64), p.targets, select(x, t), f"select {dtype} V={V}")


def test_select_leading_dims_and_many_rows(cuda_device, path):
    p = gh_synth.ce_normal(2 * 350, 4099, 2.0, dtype="bf16", seed=21)
    x, t = to_device(p)
    x3, t3 = x.view(2, 350, 4099), t.view(2, 350)
    out = gh.gh_selective_log_softmax(x3, t3)
    torch.cuda.synchronize()
    assert tuple(out.shape) == (2, 350) and out.dtype == torch.float32
    xv = p.values_f32().astype(np.float64).reshape(2, 350, 4099)
    check_select(xv, p.targets.reshape(2, 350), out.cpu().numpy().astype(np.float64), "select [2,350,V]")


def test_select_is_minus_z_free_row_loss(cuda_device, path):
    # x_t - lse and lse - x_t from the same fp32 values: exact negatives
    p = gh_synth.ce_normal(257, 50257, 3.0, dtype="bf16", seed=22)
    x, t = to_device(p)
    rl = torch.empty(257, dtype=torch.float32, device="cuda")
    gh.gh_ce_fwd(x, t, -100, "sum", 0.0, row_loss=rl)
    out = gh.gh_selective_log_softmax(x, t)
    torch.cuda.synchronize()
    assert torch.equal(out, -rl)


def test_select_out_of_range_index_gives_nan(cuda_device, path):
    gh.gh_get_device_status()
    p = gh_synth.ce_normal(6, 500, 2.0, dtype="f32", seed=23)
    p.targets[1] = 500
    p.targets[4] = -100  # no ignore_index here: a negative index is out of range too
    x, t = to_device(p)
    out = select(x, t)
    assert gh.gh_get_device_status() == gh.GH_ERR_TARGET_RANGE
    assert np.isnan(out[[1, 4]]).all()
    ok = np.array([0, 2, 3, 5])
    check_select(p.values_f32().astype(np.float64)[ok], p.targets[ok], out[ok], "select in-range rows")


def test_select_empty(cuda_device):
    x = torch.empty(0, 10, dtype=torch.float32, device="cuda")
    t = torch.empty(0, dtype=torch.int64, device="cuda")
    out = gh.gh_selective_log_softmax(x, t)
    assert out.shape == (0,)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ring_row_alignments_and_tiny_rows(cuda_device, dtype):
    # the default path (>= 8 rows per SM): every 16-byte phase of the row
    # starts, rows with no whole chunk, rows of one chunk and a ragged piece
    for V in (1, 2, 3, 5, 8, 9, 13, 17, 1021, 8195, 16389):
        p = gh_synth.ce_normal(1300, V, 3.0, dtype=dtype, ignore_frac=0.15, reduction="sum", z_loss=1e-3, seed=V)
        check_fwd(p, *fwd(p), f"ring {dtype} V={V}")
        x, t = to_device(p)
        idx = torch.from_numpy(np.maximum(p.targets, 0)).cuda()
        check_select(p.values_f32().astype(np.float64), np.maximum(p.targets, 0), select(x, idx), f"ring select V={V}")


def test_ring_many_pieces_per_row(cuda_device, monkeypatch):
    monkeypatch.setenv("GH_CE_PATH", "ring")
    # 262147 bf16 = 33 pieces of 16 KiB; more pieces per CTA than ring slots
    p = gh_synth.ce_student_t_spiked(200, 262147, dtype="bf16", reduction="mean", z_loss=1e-4, seed=31)
    check_fwd(p, *fwd(p), "ring spiked 262147")


@pytest.mark.slow
def test_full_size_gpt2_workload_fwd_and_select(cuda_device):
    p = gh_synth.ce_gpt2()
    x, t = to_device(p)
    rl = torch.empty(p.B, dtype=torch.float32, device="cuda")
    loss, _ = gh.gh_ce_fwd(x, t, p.ignore_index, p.reduction, p.z_loss, row_loss=rl)
    sel = gh.gh_selective_log_softmax(x, t.clamp(min=0))
    torch.cuda.synchronize()
    ref = oracle.cross_entropy(p.values_f32(), p.targets, p.ignore_index, p.reduction, p.z_loss,
                               with_grad=False, row_block=64)
    valid = p.targets != p.ignore_index
    eps = np.concatenate([row_eps(p.values_f32(slice(r0, r0 + 256))) for r0 in range(0, p.B, 256)])
    check_loss(loss.item(), ref["loss"], loss_atol(eps, ref["lse"], valid, p.reduction), "gpt2 fwd")
    rows = np.random.default_rng(1).choice(p.B, 64, replace=False)
    xs = p.values_f32(rows).astype(np.float64)
    check_select(xs, np.maximum(p.targets[rows], 0), sel.cpu().numpy().astype(np.float64)[rows], "gpt2 select")
