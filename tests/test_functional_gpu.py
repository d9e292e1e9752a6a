"""The Greyhound-style functional API (autograd over the C ABI).

GPU: cross_entropy's backward returns exactly the gradient gh_ce_fwd_bwd
computes (and that gradient times the upstream gradient when it is not 1);
without grad it uses the forward-only kernel and gives the same loss; the
linear cross-entropy and the generic chunked loss give the gradients of their
direct calls.  CPU: autograd_loss_and_logits_grad reproduces the closed-form
cross-entropy gradient softmax - onehot.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gh_synth
import lm_head_cross_gh_b200 as gh
from lm_head_cross_gh_b200 import functional as GF


def test_autograd_adapter_cpu():
    torch.manual_seed(0)
    x = torch.randn(7, 11, dtype=torch.float64)
    t = torch.randint(0, 11, (7,))
    loss, g = GF.autograd_loss_and_logits_grad(lambda z, tt: F.cross_entropy(z, tt, reduction="sum"))(x, t)
    p = torch.softmax(x.float(), dim=1)
    p[torch.arange(7), t] -= 1.0
    assert torch.allclose(g.float(), p, atol=1e-6) and g.dtype == x.dtype
    ref = F.cross_entropy(x, t, reduction="sum")
    assert abs(loss.item() - ref.item()) < 1e-5


@pytest.mark.gpu
def test_cross_entropy_autograd_matches_the_kernel(cuda_device):
    p = gh_synth.ce_normal(6 * 100, 5003, 3.0, dtype="bf16", ignore_frac=0.1, z_loss=1e-4, seed=3)
    x = torch.from_numpy(p.logits.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(p.targets).cuda()
    ref_loss, ref_grad = gh.gh_ce_fwd_bwd(x, t, -100, "mean", 1e-4)
    xl = x.clone().view(6, 100, 5003).requires_grad_(True)
    loss = GF.cross_entropy(xl, t.view(6, 100), -100, "mean", 1e-4)
    loss.backward()
    torch.cuda.synchronize()
    assert loss.item() == ref_loss.item()
    assert torch.equal(xl.grad.view(600, 5003).view(torch.int16), ref_grad.view(torch.int16))
    xl.grad = None
    (3.0 * GF.cross_entropy(xl, t.view(6, 100), -100, "mean", 1e-4)).backward()
    assert torch.allclose(xl.grad.view(600, 5003).float(), 3.0 * ref_grad.float(), rtol=1e-2, atol=1e-9)
    with torch.no_grad():
        l2 = GF.cross_entropy(x, t, -100, "mean", 1e-4)
    assert abs(l2.item() - ref_loss.item()) <= 1e-5 * abs(ref_loss.item())


@pytest.mark.gpu
def test_backward_is_captured_in_a_cuda_graph(cuda_device):
    """The backward multiplies the saved gradient by the upstream gradient on
    the device, without reading it back to the host, so it can be captured in
    a CUDA graph; each replay uses the upstream gradient's current value."""
    p = gh_synth.ce_normal(300, 2003, 3.0, dtype="bf16", ignore_frac=0.1, z_loss=1e-4, seed=9)
    x0 = torch.from_numpy(p.logits.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(p.targets).cuda()
    _, ref_grad = gh.gh_ce_fwd_bwd(x0, t, -100, "mean", 1e-4)
    x = x0.clone().requires_grad_(True)
    g = torch.full((), 2.0, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        loss = GF.cross_entropy(x, t, -100, "mean", 1e-4)
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        (gx,) = torch.autograd.grad(loss, x, grad_outputs=g, retain_graph=True)
    for scale in (2.0, -0.5):
        g.fill_(scale)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(gx, ref_grad * torch.tensor(scale, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.gpu
def test_linear_and_generic_chunked_losses_autograd(cuda_device):
    q = gh_synth.linear_ce_normal(512, 128, 3001, chunk=0, ignore_frac=0.05, x_sigma=1.0, w_sigma=0.05,
                                  reduction="sum", z_loss=0.0, seed=4)
    X = torch.from_numpy(q.inputs.view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(q.weight.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(q.targets).cuda()
    l_ref, dx_ref, dw_ref = gh.gh_linear_ce(X, W, t, -100, "sum", 0.0, 0, "fp32")
    Xg, Wg = X.clone().requires_grad_(True), W.clone().requires_grad_(True)
    loss = GF.chunked_linear_cross_entropy(Xg, Wg, t, -100, "sum", 0.0, "fp32")
    loss.backward()
    torch.cuda.synchronize()
    assert loss.item() == l_ref.item()
    assert torch.equal(Xg.grad, dx_ref) and torch.equal(Wg.grad, dw_ref)

    fn = GF.autograd_loss_and_logits_grad(lambda z, tt: F.cross_entropy(z, tt, ignore_index=-100, reduction="sum"))
    Xh, Wh = X.clone().requires_grad_(True), W.clone().requires_grad_(True)
    loss2 = GF.chunked_linear_loss(Xh, Wh, fn, t, chunk_size=128)
    loss2.backward()
    torch.cuda.synchronize()
    assert abs(loss2.item() - l_ref.item()) <= 1e-3 * abs(l_ref.item())
    for a, b in ((Xh.grad, dx_ref), (Wh.grad, dw_ref)):
        a64, b64 = a.float().cpu().double(), b.float().cpu().double()
        assert (a64 - b64).norm() <= 1e-2 * b64.norm()


@pytest.mark.gpu
def test_selective_log_softmax_function(cuda_device):
    x = torch.randn(4, 9, 333, device="cuda")
    i = torch.randint(0, 333, (4, 9), device="cuda")
    out = GF.selective_log_softmax(x, i)
    ref = torch.gather(torch.log_softmax(x.double(), dim=-1), -1, i[..., None])[..., 0]
    assert torch.allclose(out.double(), ref, atol=1e-5)
