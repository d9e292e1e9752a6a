"""Pins for the float64 chunked linear cross-entropy oracle (CPU only).

The chunked oracle is checked against a materialised brute force, against
PyTorch autograd through ``F.linear`` + ``F.cross_entropy`` (z = 0), against
central finite differences (z > 0), and against identities any correct
implementation satisfies.
"""
import numpy as np
import pytest
import torch

import oracle


def _problem(N, D, V, seed, ignore_frac=0.2, xs=1.0, ws=0.3):
    rng = np.random.default_rng(seed)
    X = rng.normal(0, xs, size=(N, D))
    W = rng.normal(0, ws, size=(V, D))
    t = rng.integers(0, V, size=N)
    k = int(ignore_frac * N)
    if k:
        t[rng.choice(N, k, replace=False)] = -100
    return X, W, t


@pytest.mark.parametrize("chunk", [1, 3, 7, 16, 0])
@pytest.mark.parametrize("reduction", ["mean", "sum"])
@pytest.mark.parametrize("z", [0.0, 1e-2])
def test_chunked_equals_materialised(chunk, reduction, z):
    X, W, t = _problem(16, 8, 23, seed=1)
    a = oracle.linear_cross_entropy(X, W, t, reduction=reduction, z_loss=z, chunk=chunk)
    b = oracle.linear_cross_entropy_materialised(X, W, t, reduction=reduction, z_loss=z)
    assert a["loss"] == pytest.approx(b["loss"], rel=1e-12)
    np.testing.assert_allclose(a["grad_inputs"], b["grad_inputs"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(a["grad_weight"], b["grad_weight"], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("reduction", ["mean", "sum"])
def test_matches_torch_autograd(reduction):
    X, W, t = _problem(20, 12, 37, seed=2)
    r = oracle.linear_cross_entropy(X, W, t, reduction=reduction, chunk=6)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    loss = torch.nn.functional.cross_entropy(torch.nn.functional.linear(Xt, Wt), torch.tensor(t),
                                             ignore_index=-100, reduction=reduction)
    loss.backward()
    assert r["loss"] == pytest.approx(loss.item(), rel=1e-13)
    np.testing.assert_allclose(r["grad_inputs"], Xt.grad.numpy(), rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(r["grad_weight"], Wt.grad.numpy(), rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("z", [1e-2, 0.2])
def test_finite_differences_inputs_and_weight(z):
    X, W, t = _problem(5, 3, 7, seed=3, ignore_frac=0.2)
    r = oracle.linear_cross_entropy(X, W, t, reduction="mean", z_loss=z, chunk=2)

    def L(Xa, Wa):
        return oracle.linear_cross_entropy(Xa, Wa, t, reduction="mean", z_loss=z, chunk=2)["loss"]

    h = 1e-6
    for A, G, is_x in ((X, r["grad_inputs"], True), (W, r["grad_weight"], False)):
        fd = np.zeros_like(A)
        for idx in np.ndindex(A.shape):
            Ap = A.copy(); Ap[idx] += h
            Am = A.copy(); Am[idx] -= h
            fd[idx] = ((L(Ap, W) - L(Am, W)) if is_x else (L(X, Ap) - L(X, Am))) / (2 * h)
        np.testing.assert_allclose(G, fd, rtol=1e-6, atol=1e-8)


def test_grad_weight_columns_sum_to_zero_without_z_loss():
    # each valid G row sums to 0 when z = 0, so sum_v grad_W[v, :] = sum_i 0 * X_i = 0
    X, W, t = _problem(30, 10, 41, seed=4)
    r = oracle.linear_cross_entropy(X, W, t, z_loss=0.0, chunk=8)
    np.testing.assert_allclose(r["grad_weight"].sum(axis=0), 0.0, atol=1e-14)


def test_grad_weight_column_sums_with_z_loss():
    # sum_v G_iv = scale * 2 z lse_i, so sum_v grad_W[v, :] = sum_i scale * 2 z lse_i X_i
    X, W, t = _problem(30, 10, 41, seed=5)
    z = 0.05
    r = oracle.linear_cross_entropy(X, W, t, z_loss=z, chunk=8)
    valid = t != -100
    scale = 1.0 / valid.sum()
    expect = ((scale * 2 * z * r["lse"]) * valid) @ X
    np.testing.assert_allclose(r["grad_weight"].sum(axis=0), expect, rtol=1e-11, atol=1e-14)


def test_inner_product_identity():
    # <grad_W, W> = sum_iv G_iv Z_iv = <grad_X, X>
    X, W, t = _problem(25, 9, 33, seed=6)
    r = oracle.linear_cross_entropy(X, W, t, z_loss=1e-3, chunk=7)
    a = float(np.sum(r["grad_weight"] * W))
    b = float(np.sum(r["grad_inputs"] * X))
    assert a == pytest.approx(b, rel=1e-11)


def test_weight_accumulation_single_chunk_is_one_rounding():
    X, W, t = _problem(12, 6, 19, seed=7)
    a = oracle.linear_cross_entropy(X, W, t, chunk=0, accum="fp32")
    b = oracle.linear_cross_entropy(X, W, t, chunk=0, accum="weight")
    np.testing.assert_array_equal(b["grad_weight"], oracle.bf16_round(a["grad_weight"]))


def test_weight_accumulation_rounds_between_chunks():
    X, W, t = _problem(64, 16, 50, seed=8, ignore_frac=0.0)
    a = oracle.linear_cross_entropy(X, W, t, chunk=8, accum="fp32")
    b = oracle.linear_cross_entropy(X, W, t, chunk=8, accum="weight")
    # every value of the bf16 accumulator is a bf16 number ...
    np.testing.assert_array_equal(b["grad_weight"], oracle.bf16_round(b["grad_weight"]))
    # ... it differs from the wide accumulator by at most a few bf16 roundings,
    diff = np.abs(b["grad_weight"] - a["grad_weight"])
    bound = 8 * 2.0 ** -8 * np.abs(a["grad_weight"]) + 8 * 2.0 ** -8 * np.abs(a["grad_weight"]).max() / 8
    assert np.all(diff <= bound)
    # ... and it is not the single final rounding (rounding happened in between)
    assert not np.array_equal(b["grad_weight"], oracle.bf16_round(a["grad_weight"]))
    # grad_inputs and loss do not depend on the weight-gradient accumulator
    np.testing.assert_array_equal(a["grad_inputs"], b["grad_inputs"])
    assert a["loss"] == b["loss"]


def test_zero_and_ignored_rows():
    X, W, t = _problem(10, 4, 9, seed=9, ignore_frac=0.0)
    t[[2, 5]] = -100
    r = oracle.linear_cross_entropy(X, W, t, chunk=3)
    assert not r["grad_inputs"][[2, 5]].any()
    t[:] = -100
    r = oracle.linear_cross_entropy(X, W, t, chunk=3)
    assert r["loss"] == 0.0 and not r["grad_inputs"].any() and not r["grad_weight"].any()


def _golden_weight_accum():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "linear_ce_weight_accum.json")) as f:
        return json.load(f)


def _bits_to_f64(bits):
    return np.array([[np.uint32(int(b, 16) << 16).view(np.float32) for b in row] for row in bits], dtype=np.float64)


def test_weight_accumulation_order_golden():
    """Hand-derived two-chunk example (tests/golden/linear_ce_weight_accum.json):
    'weight' accumulation rounds the running sum after each chunk, which gives
    different bits from rounding each chunk's product first and from a single
    final rounding ('fp32')."""
    g = _golden_weight_accum()
    X = np.array(g["inputs"], dtype=np.float64)
    W = np.array(g["weight"], dtype=np.float64)
    t = np.array(g["targets"], dtype=np.int64)
    w = oracle.linear_cross_entropy(X, W, t, g["ignore_index"], g["reduction"], g["z_loss"], g["chunk"], "weight")
    f = oracle.linear_cross_entropy(X, W, t, g["ignore_index"], g["reduction"], g["z_loss"], g["chunk"], "fp32")
    np.testing.assert_array_equal(w["grad_weight"], _bits_to_f64(g["grad_weight_weight_accum_bf16_bits"]))
    np.testing.assert_array_equal(oracle.bf16_round(f["grad_weight"]),
                                  _bits_to_f64(g["grad_weight_fp32_accum_bf16_bits"]))
    assert not np.array_equal(w["grad_weight"], _bits_to_f64(g["wrong_reading_round_product_first_bits"]))
    assert w["loss"] == pytest.approx(4 * np.log(2.0), rel=1e-15)
    np.testing.assert_array_equal(w["grad_inputs"], np.array(g["grad_inputs"]))
    # the inputs are the bf16 values the expressions name
    np.testing.assert_array_equal(X, oracle.bf16_round(X))


@pytest.mark.parametrize("reduction,z", [("mean", 1e-2), ("sum", 0.0)])
def test_sampled_outputs_equal_the_full_oracle(reduction, z):
    """row_lse, loss_from_lse, grad_input_rows and grad_weight_rows (the forms
    used on problems too large to materialise) equal the corresponding slices
    of the chunked oracle, which is pinned above against torch autograd,
    finite differences and the materialised brute force."""
    X, W, t = _problem(40, 10, 57, seed=11, ignore_frac=0.2)
    t[3] = 5
    t[7] = 5  # two rows share a target: its column gets both one-hot terms
    r = oracle.linear_cross_entropy(X, W, t, reduction=reduction, z_loss=z, chunk=9)
    lse = oracle.row_lse(X, W, row_block=7)
    np.testing.assert_allclose(lse, r["lse"], rtol=1e-14)
    assert oracle.loss_from_lse(X, W, t, lse, reduction=reduction, z_loss=z) == pytest.approx(r["loss"], rel=1e-13)
    rows = np.array([0, 3, 7, 39, 12])
    np.testing.assert_allclose(oracle.grad_input_rows(X, W, t, rows, reduction=reduction, z_loss=z),
                               r["grad_inputs"][rows], rtol=1e-12, atol=1e-15)
    vocab = np.array([5, 0, 56, 31])
    np.testing.assert_allclose(oracle.grad_weight_rows(X, W, t, lse, vocab, reduction=reduction, z_loss=z),
                               r["grad_weight"][vocab], rtol=1e-12, atol=1e-15)
