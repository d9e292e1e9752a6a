"""GPU parity of gh_chunked_linear_loss (the chunk loop of the linear
cross-entropy with a caller-provided loss per chunk).

1. Cross-entropy written as a per-chunk callback in plain PyTorch gives the
   same loss and gradients as gh_linear_ce (sum reduction), within the linear
   cross-entropy's bars (1e-3 relative loss, 1e-2 relative Frobenius).
2. A loss that is not cross-entropy, L = sum(w_r * logits_r^2) / 2 with a
   per-row weight w (a tensor argument sliced per chunk), against its closed
   form in float64: G = w * bf16(X W^T), dX = G W, dW = G^T X.
3. An exception in the callback stops the loop and is raised to the caller.
"""
import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
import oracle

pytestmark = pytest.mark.gpu


def dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def ce_chunk(logits, targets, ignore_index=-100):
    """Summed cross-entropy of one chunk and its logits gradient, in fp32."""
    x = logits.float()
    valid = targets != ignore_index
    t = torch.where(valid, targets, torch.zeros_like(targets))
    lse = torch.logsumexp(x, dim=1)
    loss = ((lse - x.gather(1, t[:, None])[:, 0]) * valid).sum()
    g = torch.softmax(x, dim=1)
    g[torch.arange(x.shape[0], device=x.device), t] -= 1.0
    g = g * valid[:, None]
    return loss, g.to(torch.bfloat16)


@pytest.mark.parametrize("N,D,V,chunk,accum", [(300, 64, 1000, 128, "fp32"), (1000, 256, 5003, 384, "weight"),
                                               (2048, 768, 8191, 1024, "fp32")])
def test_cross_entropy_as_a_callback_matches_linear_ce(cuda_device, N, D, V, chunk, accum):
    p = gh_synth.linear_ce_normal(N, D, V, chunk=chunk, ignore_frac=0.05, x_sigma=1.0, w_sigma=0.5 / np.sqrt(D),
                                  accum=accum, reduction="sum", z_loss=0.0, seed=N)
    X, W = dev_bf16(p.inputs), dev_bf16(p.weight)
    t = torch.from_numpy(p.targets).cuda()
    l1, x1, w1 = gh.gh_chunked_linear_loss(X, W, ce_chunk, t, chunk=chunk, accum=accum)
    l2, x2, w2 = gh.gh_linear_ce(X, W, t, -100, "sum", 0.0, chunk, accum)
    torch.cuda.synchronize()
    r = oracle.linear_cross_entropy(gh_synth.bf16_to_f32(p.inputs).astype(np.float64),
                                    gh_synth.bf16_to_f32(p.weight).astype(np.float64), p.targets, -100, "sum", 0.0,
                                    chunk, accum)
    assert abs(l1.item() - r["loss"]) <= 1e-3 * abs(r["loss"])
    assert abs(l1.item() - l2.item()) <= 1e-3 * abs(l2.item())
    dx = x1.float().cpu().numpy().astype(np.float64)
    dw = w1.float().cpu().numpy().astype(np.float64)
    assert rel_fro(dx, r["grad_inputs"]) <= 1e-2
    assert rel_fro(dw, r["grad_weight"]) <= 1e-2
    assert rel_fro(dx, x2.float().cpu().numpy().astype(np.float64)) <= 1e-2


def test_a_non_cross_entropy_loss_with_a_sliced_row_argument(cuda_device):
    N, D, V, chunk = 700, 128, 3001, 256
    rng = np.random.default_rng(9)
    Xf = rng.normal(size=(N, D)).astype(np.float32)
    Wf = (rng.normal(size=(V, D)) * 0.05).astype(np.float32)
    w = rng.uniform(0.5, 1.5, size=N).astype(np.float32)
    Xb, Wb = gh_synth.f32_to_bf16(Xf), gh_synth.f32_to_bf16(Wf)
    X, W = dev_bf16(Xb), dev_bf16(Wb)
    wt = torch.from_numpy(w).cuda()

    def sq(logits, row_w):
        x = logits.float()
        return 0.5 * (row_w[:, None] * x * x).sum(), (row_w[:, None] * x).to(torch.bfloat16)

    loss, dX, dW = gh.gh_chunked_linear_loss(X, W, sq, wt, chunk=chunk)
    torch.cuda.synchronize()
    X64 = gh_synth.bf16_to_f32(Xb).astype(np.float64)
    W64 = gh_synth.bf16_to_f32(Wb).astype(np.float64)
    Lg = gh_synth.bf16_to_f32(gh_synth.f32_to_bf16((X64 @ W64.T).astype(np.float32))).astype(np.float64)
    G = w[:, None].astype(np.float64) * Lg
    ref_loss = 0.5 * float((w[:, None] * Lg * Lg).sum())
    assert abs(loss.item() - ref_loss) <= 1e-3 * abs(ref_loss)
    assert rel_fro(dX.float().cpu().numpy().astype(np.float64), G @ W64) <= 1e-2
    assert rel_fro(dW.float().cpu().numpy().astype(np.float64), G.T @ X64) <= 1e-2


def test_callback_error_is_raised(cuda_device):
    X = torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(100, 64, dtype=torch.bfloat16, device="cuda")

    def bad(logits):
        raise KeyError("boom")

    with pytest.raises(KeyError):
        gh.gh_chunked_linear_loss(X, W, bad, chunk=128)
    torch.cuda.synchronize()
    # the library stays usable
    loss, _, _ = gh.gh_chunked_linear_loss(X, W, lambda x: (x.float().sum(), torch.zeros_like(x)), chunk=128)
    torch.cuda.synchronize()
    assert loss.item() == 0.0
