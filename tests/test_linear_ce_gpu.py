"""GPU parity of gh_linear_ce (chunked linear cross-entropy) against the oracle.

Tolerances: the stated bars are loss within 1e-3 relative and grad_inputs /
grad_weight within 1e-2 relative Frobenius error (bf16 GEMMs).  The GPU rounds
the chunk logits and the logits gradient to bf16 before the two gradient
GEMMs, so each element of G carries ~2^-9 relative error; a dropped term
(z-loss factor, a transposed operand, a wrong chunk offset) produces errors
of order 1, far above the bars.  The tests also check the identity
<grad_W, W> = <grad_X, X> of the GPU's own outputs.
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


def run(p):
    X, W = dev_bf16(p.inputs), dev_bf16(p.weight)
    t = torch.from_numpy(p.targets).cuda()
    loss, dX, dW = gh.gh_linear_ce(X, W, t, p.ignore_index, p.reduction, p.z_loss, p.chunk, p.accum)
    torch.cuda.synchronize()
    return loss.item(), dX.float().cpu().numpy().astype(np.float64), dW.float().cpu().numpy().astype(np.float64)


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def check(p, loss, dX, dW, what, loss_rtol=1e-3, grad_rtol=1e-2):
    X = gh_synth.bf16_to_f32(p.inputs).astype(np.float64)
    W = gh_synth.bf16_to_f32(p.weight).astype(np.float64)
    r = oracle.linear_cross_entropy(X, W, p.targets, p.ignore_index, p.reduction, p.z_loss, p.chunk, p.accum)
    assert abs(loss - r["loss"]) <= loss_rtol * abs(r["loss"]) + 1e-6, f"{what} loss {loss} vs {r['loss']}"
    ex, ew = rel_fro(dX, r["grad_inputs"]), rel_fro(dW, r["grad_weight"])
    assert ex <= grad_rtol, f"{what} grad_inputs rel fro {ex}"
    assert ew <= grad_rtol, f"{what} grad_weight rel fro {ew}"
    ign = p.targets == p.ignore_index
    assert not dX[ign].any(), f"{what} ignored rows of grad_inputs must be zero"
    a, b = float(np.sum(dW * W)), float(np.sum(dX * X))
    assert abs(a - b) <= 2e-2 * max(abs(a), abs(b), 1e-12), f"{what} <dW,W>={a} <dX,X>={b}"
    return ex, ew


@pytest.mark.parametrize("accum", ["fp32", "weight"])
@pytest.mark.parametrize("reduction,z", [("mean", 1e-4), ("sum", 0.0)])
def test_small_three_ragged_chunks(cuda_device, accum, reduction, z):
    p = gh_synth.linear_ce_normal(300, 64, 1000, chunk=128, ignore_frac=0.05, x_sigma=1.0, w_sigma=0.2,
                                  accum=accum, reduction=reduction, z_loss=z, seed=1)
    check(p, *run(p), f"small {accum} {reduction}")


@pytest.mark.parametrize("N,D,V,chunk", [
    (256, 128, 517, 256),     # one chunk, V not a multiple of 8 (padded chunk rows)
    (129, 8, 64, 64),         # minimal D, ragged chunk of one row
    (200, 72, 300, 0),        # D not a multiple of 64, default chunk
    (640, 256, 2049, 384),    # several full N tiles, V just past a tile
    (1000, 768, 5003, 384),   # GPT-2 width, ragged everything
])
def test_shapes(cuda_device, N, D, V, chunk):
    p = gh_synth.linear_ce_normal(N, D, V, chunk=chunk, ignore_frac=0.1, x_sigma=1.0, w_sigma=0.5 / np.sqrt(D),
                                  accum="fp32", reduction="mean", z_loss=1e-4, seed=N + V)
    check(p, *run(p), f"N={N} D={D} V={V} chunk={chunk}")


def test_chunk_size_does_not_change_results(cuda_device):
    base = gh_synth.linear_ce_normal(512, 128, 3001, chunk=512, ignore_frac=0.1, w_sigma=0.05, seed=7)
    l1, x1, w1 = run(base)
    base.chunk = 128
    l2, x2, w2 = run(base)
    assert abs(l1 - l2) <= 1e-5 * abs(l1)
    # grad_inputs rows do not depend on the chunking at all (same kernels per row)
    np.testing.assert_array_equal(x1, x2)
    assert rel_fro(w2, w1) < 5e-3


def test_all_tokens_ignored_and_empty(cuda_device):
    p = gh_synth.linear_ce_normal(130, 64, 200, chunk=64, seed=3)
    p.targets[:] = -100
    loss, dX, dW = run(p)
    assert loss == 0.0 and not dX.any() and not dW.any()
    X = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.ones(200, 64, dtype=torch.bfloat16, device="cuda")
    t = torch.empty(0, dtype=torch.int64, device="cuda")
    loss, dX, dW = gh.gh_linear_ce(X, W, t)
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and not dW.any().item()


@pytest.mark.slow
def test_full_size_gpt2_head(cuda_device):
    p = gh_synth.linear_ce_gpt2()
    ex, ew = check(p, *run(p), "gpt2 head")
    print(f"gpt2 head: grad_inputs rel fro {ex:.2e}, grad_weight rel fro {ew:.2e}")


@pytest.mark.slow
def test_full_size_llama3_8b_head_sampled(cuda_device):
    """Llama-3-8B head at full size: sampled grad_inputs rows against the oracle
    (each needs only its own logits row) and the <dW, W> = <dX, X> identity."""
    p = gh_synth.linear_ce_llama3_8b()
    loss, dX, dW = run(p)
    X = gh_synth.bf16_to_f32(p.inputs).astype(np.float64)
    W = gh_synth.bf16_to_f32(p.weight).astype(np.float64)
    n_valid, scale = oracle.n_valid_and_scale(p.targets, p.ignore_index, p.reduction, p.V)
    rows = np.random.default_rng(0).choice(p.N, 8, replace=False)
    Z = X[rows] @ W.T
    lse, row_loss, G = oracle.ce_rows(Z, p.targets[rows], p.ignore_index, p.z_loss, scale)
    ref = G @ W
    assert rel_fro(dX[rows], ref) <= 1e-2
    a, b = float(np.sum(dW * W)), float(np.sum(dX * X))
    assert abs(a - b) <= 2e-2 * max(abs(a), abs(b))
    assert np.isfinite(loss) and 0 < loss < 2 * np.log(p.V)


@pytest.mark.parametrize("accum", ["weight", "fp32"])
def test_weight_accumulation_order_golden(cuda_device, accum):
    """The hand-derived two-chunk example of tests/golden/linear_ce_weight_accum.json,
    bit for bit: 'weight' rounds the running bf16 sum after each chunk, 'fp32'
    rounds once at the end.  D is padded from 2 to 8 with zero columns (the
    library needs 16-byte rows); the padding columns' gradients are zero."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "linear_ce_weight_accum.json")) as f:
        g = json.load(f)
    X = np.zeros((g["N"], 8), np.float32)
    X[:, :g["D"]] = np.array(g["inputs"], np.float32)
    W = np.zeros((g["V"], 8), np.float32)
    Xd = torch.from_numpy(X).cuda().to(torch.bfloat16)
    Wd = torch.from_numpy(W).cuda().to(torch.bfloat16)
    t = torch.tensor(g["targets"], dtype=torch.int64, device="cuda")
    loss, dX, dW = gh.gh_linear_ce(Xd, Wd, t, g["ignore_index"], g["reduction"], g["z_loss"], g["chunk"], accum)
    torch.cuda.synchronize()
    key = "grad_weight_weight_accum_bf16_bits" if accum == "weight" else "grad_weight_fp32_accum_bf16_bits"
    want = np.array([[int(b, 16) for b in row] for row in g[key]], dtype=np.uint16)
    got = dW.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got[:, :g["D"]], want)
    assert not got[:, g["D"]:].any()
    assert not dX.float().cpu().numpy().any()
    assert abs(loss.item() - 4 * np.log(2.0)) <= 1e-6
