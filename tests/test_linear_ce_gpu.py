"""GPU parity of gh_linear_ce (chunked linear cross-entropy) against the oracle,
on both GEMM layouts (CTA pairs and single CTAs).

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


@pytest.fixture(autouse=True, params=["pair", "single"])
def gemm_mode(request, monkeypatch):
    """Every case on both GEMM layouts: 256 x 256 tiles on a pair of CTAs
    (cta_group::2, the default) and 128 x 256 tiles on one CTA."""
    monkeypatch.setenv("GH_GEMM", request.param)
    return request.param


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
    (50, 16, 17, 32),         # V inside one 64-column block of the exponentials
    (40, 16, 1, 0),           # one class: zero loss (z = 1e-4 aside) and gradients
    (200, 72, 300, 0),        # D not a multiple of 64, default chunk
    (640, 256, 2049, 384),    # several full N tiles, V just past a tile
    (1000, 768, 5003, 384),   # GPT-2 width, ragged everything
    (4096, 1280, 4099, 0),    # dX tiles past one wave: K split with more units than SMs
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


def _stored_llama_lse(p):
    """Every row's lse from tests/golden/linear_ce_llama3_8b_lse.npz (written by
    tests/golden/make_llama3_8b_lse.py with the oracle), after checking that it
    was made from these exact inputs."""
    import importlib.util
    import os
    here = os.path.join(os.path.dirname(__file__), "golden")
    spec = importlib.util.spec_from_file_location("make_llama3_8b_lse", os.path.join(here, "make_llama3_8b_lse.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    stored = np.load(os.path.join(here, "linear_ce_llama3_8b_lse.npz"))
    assert str(stored["inputs_sha256"]) == mk.inputs_digest(p), \
        "the stored lse was made from other inputs: rerun tests/golden/make_llama3_8b_lse.py"
    return stored["lse"]


def _rows_f64(t, idx):
    return t[torch.as_tensor(idx, device=t.device)].float().cpu().numpy().astype(np.float64)


@pytest.mark.slow
def test_full_size_llama3_8b_head(cuda_device):
    """Llama-3-8B head at full size ([16384, 4096] x [128256, 4096], 5% ignored,
    chunk 4096, fp32 accumulation, mean, z 1e-4) against the oracle:

    * the loss within 1e-3 relative, from every row's oracle lse (stored) and
      target logit;
    * 64 sampled rows of grad_inputs, each within 1e-2 relative Frobenius error
      (each needs only its own logits row), and every ignored row exactly zero;
    * 64 sampled vocabulary rows of grad_weight, each within 1e-2 relative
      Frobenius error: half are targets of sampled valid rows (their column of
      the logits gradient carries one-hot terms), half drawn uniformly.
    """
    p = gh_synth.linear_ce_llama3_8b()
    lse = _stored_llama_lse(p)
    Xd, Wd = dev_bf16(p.inputs), dev_bf16(p.weight)
    t = torch.from_numpy(p.targets).cuda()
    loss, dX, dW = gh.gh_linear_ce(Xd, Wd, t, p.ignore_index, p.reduction, p.z_loss, p.chunk, p.accum)
    torch.cuda.synchronize()
    assert gh.gh_get_device_status() == gh.GH_OK
    X = gh_synth.bf16_to_f32(p.inputs).astype(np.float64)
    W = gh_synth.bf16_to_f32(p.weight).astype(np.float64)
    kw = dict(ignore_index=p.ignore_index, reduction=p.reduction, z_loss=p.z_loss)

    ref_loss = oracle.loss_from_lse(X, W, p.targets, lse, **kw)
    assert abs(loss.item() - ref_loss) <= 1e-3 * abs(ref_loss), (loss.item(), ref_loss)

    rng = np.random.default_rng(0)
    valid = np.nonzero(p.targets != p.ignore_index)[0]
    ign = np.nonzero(p.targets == p.ignore_index)[0]
    rows = rng.choice(valid, 64, replace=False)
    ref_dx = oracle.grad_input_rows(X, W, p.targets, rows, **kw)
    got_dx = _rows_f64(dX, rows)
    for k, r in enumerate(rows):
        e = rel_fro(got_dx[k], ref_dx[k])
        assert e <= 1e-2, f"grad_inputs row {r}: rel fro {e}"
    assert not dX[torch.as_tensor(ign, device="cuda")].any().item(), "ignored rows of grad_inputs must be zero"

    vocab = np.unique(np.concatenate([p.targets[rng.choice(valid, 32, replace=False)],
                                      rng.choice(p.V, 40, replace=False)]))
    assert len(vocab) >= 64
    ref_dw = oracle.grad_weight_rows(X, W, p.targets, lse, vocab, **kw)
    got_dw = _rows_f64(dW, vocab)
    for k, v in enumerate(vocab):
        e = rel_fro(got_dw[k], ref_dw[k])
        assert e <= 1e-2, f"grad_weight row {v}: rel fro {e}"


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


def _bf16_bits(a):
    return gh_synth.f32_to_bf16(np.asarray(a, np.float32))


@pytest.mark.parametrize("accum", ["fp32", "weight"])
def test_rows_outside_the_exponent_window(cuda_device, accum):
    """The logits epilogue stores exp(x) (reference 0) and keeps a row only while
    its lse lies in [-40, 40]; rows beyond (here lse ~ +190 and ~ -95, next to
    ordinary rows in the same chunk) make the chunk recompute with the row max
    as the reference.  An ignored row with huge logits must neither trigger
    anything nor leak into the gradients.  All results against the oracle."""
    rng = np.random.default_rng(5)
    N, D, V = 300, 64, 1000
    X = rng.normal(0.0, 1.0, (N, D)).astype(np.float32)
    W = rng.normal(0.0, 0.2, (V, D)).astype(np.float32)
    W[:, 0] = 1.0                       # a shared direction: X[i, 0] shifts every logit of row i
    X[:, 0] = 0.0
    X[3] *= 40.0                        # logits ~ N(0, 64^2): lse far above 40
    X[130, 0] = -100.0                  # every logit near -100: lse below -40
    X[131] *= 40.0                      # huge logits on a row that is ignored
    X[260, 0] = 45.0                    # lse just past the window, in the last chunk
    t = rng.integers(0, V, N).astype(np.int64)
    t[131] = -100
    t[[7, 50, 200]] = -100
    p = gh_synth.LinearCEInputs("window", _bf16_bits(X), _bf16_bits(W), t, 128, accum, -100, "mean", 1e-4)
    check(p, *run(p), f"window {accum}")
    assert gh.gh_get_device_status() == gh.GH_OK


def test_z_loss_factor_near_zero(cuda_device):
    """A z-loss multiplier for which 1 + 2 z lse is nearly 0 on one row: that
    row's gradient is almost exactly -scale at the target and ~0 elsewhere."""
    rng = np.random.default_rng(6)
    N, D, V = 200, 32, 500
    X = rng.normal(0.0, 1.0, (N, D)).astype(np.float32)
    W = rng.normal(0.0, 0.3, (V, D)).astype(np.float32)
    Xb, Wb = _bf16_bits(X), _bf16_bits(W)
    t = rng.integers(0, V, N).astype(np.int64)
    lse = oracle.row_lse(gh_synth.bf16_to_f32(Xb).astype(np.float64), gh_synth.bf16_to_f32(Wb).astype(np.float64))
    z = float(np.float32(-0.5 / lse[17]))
    p = gh_synth.LinearCEInputs("zfactor", Xb, Wb, t, 64, "fp32", -100, "sum", z)
    check(p, *run(p), "z factor near zero")
