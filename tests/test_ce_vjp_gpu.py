"""GPU parity of gh_ce_vjp (the per-row cross-entropy's logits gradient for an
upstream gradient per row, from the forward's row loss) against the oracle.

Reference: ``oracle.ce_vjp`` -- for a valid row, grad = g_r * (softmax(x_r) -
onehot(t_r)); ignored rows are zero.

Tolerance per element: one rounding of the output (2^-8 |ref| for bf16, 2e-5
|ref| for fp32) plus |g_r| p_rj times the relative error of exp(x - lse):
eps_r (the kernel's fp32 exponent arithmetic, as for the other CE kernels) plus
the error of recovering lse as row_loss + x_t in fp32 (2^-22 max(1, |lse|,
|x_t|) covers the rounding of the given loss and of the sum).  A dropped
target term, a wrong sign of g or a wrong row's lse gives errors of order
|g| p or |g|, far above it.
"""
import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
import oracle
from ce_check import row_eps, to_device

pytestmark = pytest.mark.gpu


def reference(p, g):
    x = p.values_f32().astype(np.float64)
    lse, _, _ = oracle.ce_rows(x, p.targets, p.ignore_index, 0.0, 1.0, with_grad=False)
    return oracle.ce_vjp(x, p.targets, p.ignore_index, g), lse, x


def check(p, g, out, what, row_loss=None):
    ref, lse, x = reference(p, g)
    valid = p.targets != p.ignore_index
    pm = np.exp(x - lse[:, None])
    xt = np.where(valid, x[np.arange(p.B), np.where(valid, p.targets, 0)], 0.0)
    eps = row_eps(x).reshape(-1) + 2.0 ** -22 * np.maximum(1.0, np.maximum(np.abs(lse), np.abs(xt)))
    rel = 2.0 ** -8 if p.dtype == "bf16" else 2e-5
    bound = rel * np.abs(ref) + (np.abs(g) * eps)[:, None] * pm + 1e-30
    err = np.abs(out - ref)
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of bound, worst {err[bad].max():.3g}"
    assert not out[~valid].any(), f"{what}: ignored rows must be zero"


def run(p, g, row_loss=None, **kw):
    x, t = to_device(p)
    if row_loss is None:
        rl = torch.empty(p.B, dtype=torch.float32, device="cuda")
        gh.gh_ce_fwd(x, t, p.ignore_index, "sum", 0.0, row_loss=rl)
    else:
        rl = torch.from_numpy(row_loss.astype(np.float32)).cuda()
    gd = torch.from_numpy(g.astype(np.float32)).cuda()
    out = gh.gh_ce_vjp(x, t, rl, gd, p.ignore_index, **kw)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", [1, 2, 7, 8, 9, 17, 100, 1023, 1025, 8191, 50257])
def test_vjp_ragged_vocab_sizes(cuda_device, dtype, V):
    B = 37 if V < 20000 else 9
    p = gh_synth.ce_normal(B, V, 3.0, dtype=dtype, ignore_frac=0.2, seed=V)
    g = np.random.default_rng(V).normal(size=B)
    g[::5] = 0.0
    out = run(p, g).float().cpu().numpy().astype(np.float64)
    check(p, g, out, f"{dtype} V={V}")


def test_vjp_with_oracle_row_loss_and_many_rows(cuda_device):
    p = gh_synth.ce_normal(1500, 5003, 2.0, dtype="bf16", ignore_frac=0.1, seed=41)
    g = np.random.default_rng(1).uniform(-2, 2, size=p.B)
    x = p.values_f32().astype(np.float64)
    _, rl, _ = oracle.ce_rows(x, p.targets, p.ignore_index, 0.0, 1.0, with_grad=False)
    out = run(p, g, row_loss=rl).float().cpu().numpy().astype(np.float64)
    check(p, g, out, "oracle row loss")


def test_vjp_in_place_and_shifted_gradient_buffer(cuda_device):
    p = gh_synth.ce_normal(40, 3001, 3.0, dtype="bf16", ignore_frac=0.1, seed=42)
    g = np.random.default_rng(2).normal(size=p.B)
    x, t = to_device(p)
    rl = torch.empty(p.B, dtype=torch.float32, device="cuda")
    gh.gh_ce_fwd(x, t, p.ignore_index, "sum", 0.0, row_loss=rl)
    gd = torch.from_numpy(g.astype(np.float32)).cuda()
    xi = x.clone()
    gh.gh_ce_vjp(xi, t, rl, gd, p.ignore_index, grad=xi)
    buf = torch.empty(x.numel() + 8, dtype=x.dtype, device="cuda")
    gs = buf[3:3 + x.numel()].view_as(x)  # another 16-byte phase than the logits
    gh.gh_ce_vjp(x, t, rl, gd, p.ignore_index, grad=gs)
    torch.cuda.synchronize()
    check(p, g, xi.float().cpu().numpy().astype(np.float64), "in place")
    check(p, g, gs.float().cpu().numpy().astype(np.float64), "shifted buffer")


def test_vjp_with_unit_g_is_the_summed_loss_gradient(cuda_device):
    # g = 1 and the z-free row loss: the gradient of the summed loss, which
    # gh_ce_fwd_bwd computes with its own passes
    p = gh_synth.ce_normal(300, 50257, 3.0, dtype="bf16", ignore_frac=0.05, seed=43)
    x, t = to_device(p)
    _, gfb = gh.gh_ce_fwd_bwd(x, t, p.ignore_index, "sum", 0.0)
    out = run(p, np.ones(p.B))
    torch.cuda.synchronize()
    a = out.float().cpu().numpy().astype(np.float64)
    b = gfb.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 1e-9)


def test_vjp_out_of_range_target_and_empty(cuda_device):
    gh.gh_get_device_status()
    p = gh_synth.ce_normal(6, 300, 2.0, dtype="f32", seed=44)
    p.targets[2] = 300
    g = np.ones(p.B)
    x, t = to_device(p)
    rl = torch.zeros(p.B, dtype=torch.float32, device="cuda")
    q = gh_synth.CEInputs(p.name, p.dtype, p.logits, p.targets.copy(), p.ignore_index, p.reduction, p.z_loss)
    q.targets[2] = q.ignore_index
    xq, tq = to_device(q)
    gh.gh_ce_fwd(xq, tq, q.ignore_index, "sum", 0.0, row_loss=rl)
    out = gh.gh_ce_vjp(x, t, rl, torch.ones(p.B, device="cuda"), p.ignore_index)
    torch.cuda.synchronize()
    assert gh.gh_get_device_status() == gh.GH_ERR_TARGET_RANGE
    check(q, g, out.cpu().numpy().astype(np.float64), "out-of-range row zero")
    e = gh.gh_ce_vjp(torch.empty(0, 5, device="cuda"), torch.empty(0, dtype=torch.int64, device="cuda"),
                     torch.empty(0, device="cuda"), torch.empty(0, device="cuda"))
    assert e.shape == (0, 5)
