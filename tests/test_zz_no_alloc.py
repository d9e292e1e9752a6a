"""gh_ce_fwd_bwd_noalloc against gh_ce_fwd_bwd (GPU; collected last on purpose).

The allocation-free entry point serves callers that cannot allocate device
memory inside a call: their memory is owned in full by another allocator, or
allocator calls are forbidden inside their step.  It keeps its scratch in a
fixed device array shared by every call, so these tests check that two calls
in a row (the second one seeing the first one's leftovers in that array) give
the same results as the allocating entry point, within the tolerances the
other parity tests use, and that a batch beyond the array's row limit is
refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
import oracle
from ce_check import check_grad, check_loss, grad_to_f64, loss_atol, row_eps, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["auto", "rows", "ring"])
def ce_path(request, monkeypatch):
    """The row count picks the kernel (the two-pass ring from 8 rows per SM,
    the row kernel below); "rows" and "ring" force one of them, so both
    kernels run with the fixed scratch whatever the batch size."""
    if request.param != "auto":
        monkeypatch.setenv("GH_CE_PATH", request.param)
    else:
        monkeypatch.delenv("GH_CE_PATH", raising=False)
    return request.param


def _call_noalloc(x, t, p, loss, grad):
    L = gh.lib()
    dtype = gh.GH_F32 if x.dtype == torch.float32 else gh.GH_BF16
    st = L.gh_ce_fwd_bwd_noalloc(x.data_ptr(), t.data_ptr(), x.shape[0], x.shape[1], dtype, p.ignore_index,
                                 gh.GH_REDUCTION[p.reduction], float(p.z_loss), loss.data_ptr(), grad.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    return st


def _compare(p, loss_a, grad_a, loss_b, grad_b, what):
    """Result b (no-alloc) against result a (allocating entry point)."""
    x = p.values_f32().astype(np.float64)
    ref = oracle.cross_entropy(x, p.targets, p.ignore_index, p.reduction, p.z_loss, with_grad=False)
    _, scale = oracle.n_valid_and_scale(p.targets, p.ignore_index, p.reduction, p.V)
    eps = row_eps(x)
    valid = p.targets != p.ignore_index
    check_loss(loss_b, loss_a, loss_atol(eps, ref["lse"], valid, p.reduction), what)
    check_grad(grad_b, grad_a, p.dtype, scale, p.targets, p.ignore_index, eps, what)


def test_noalloc_matches_allocating_entry_point_on_two_calls_in_a_row(cuda_device, ce_path):
    # Each problem has a different row count, share of ignored rows or
    # reduction than the one before it, so leftovers of the previous call in
    # the shared scratch (counter or row losses) would change its result.  The
    # 2048-row problem is past 8 rows per SM, where the library picks the ring
    # kernel by itself.
    problems = [
        gh_synth.ce_normal(512, 50257, 3.0, dtype="bf16", ignore_frac=0.02, reduction="mean", z_loss=1e-4, seed=21),
        gh_synth.ce_normal(2048, 4099, 3.0, dtype="bf16", ignore_frac=0.05, reduction="mean", z_loss=1e-4, seed=24),
        gh_synth.ce_normal(300, 4099, 2.0, dtype="f32", ignore_frac=0.30, reduction="mean", z_loss=0.0, seed=22),
        gh_synth.ce_normal(200, 50257, 3.0, dtype="bf16", ignore_frac=0.10, reduction="sum", z_loss=1e-4, seed=23),
    ]
    dev = [to_device(p) for p in problems]
    ref = []
    for p, (x, t) in zip(problems, dev):
        loss_a, grad_a = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, p.reduction, p.z_loss)
        torch.cuda.synchronize()
        ref.append((loss_a.item(), grad_to_f64(grad_a)))
    # the no-alloc calls back to back, nothing in between
    outs = []
    for p, (x, t) in zip(problems, dev):
        loss_b = torch.full((), float("nan"), dtype=torch.float32, device=x.device)
        grad_b = torch.full_like(x, float("nan"))
        assert _call_noalloc(x, t, p, loss_b, grad_b) == gh.GH_OK
        outs.append((loss_b, grad_b))
    torch.cuda.synchronize()
    for i, (p, (la, ga), (lb, gb)) in enumerate(zip(problems, ref, outs)):
        _compare(p, la, ga, lb.item(), grad_to_f64(gb), f"call {i}")
    assert gh.gh_get_device_status() == gh.GH_OK


def test_noalloc_refuses_batches_beyond_its_scratch(cuda_device):
    B = gh.GH_NOALLOC_MAX_ROWS + 1
    x = torch.zeros(B, 8, dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(B, dtype=torch.int64, device="cuda")
    loss = torch.full((), 5.0, device="cuda")
    grad = torch.full_like(x, 1.0)
    p = gh_synth.CEInputs("limit", "bf16", np.zeros((0, 8), np.uint16), np.zeros(0, np.int64), -100, "mean", 0.0)
    assert _call_noalloc(x, t, p, loss, grad) == gh.GH_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert loss.item() == 5.0 and bool((grad == 1.0).all())  # nothing ran
    with pytest.raises(gh.GhError):
        gh.gh_ce_fwd_bwd_noalloc(x, t, loss=loss, grad=grad)
