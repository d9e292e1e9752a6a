"""Pins for the float64 cross-entropy oracle (CPU only).

Each test checks the oracle against something other than itself: a closed
form, an invariant of the definition, central finite differences, or
``torch.nn.functional.cross_entropy`` (the ordinary loss the Greyhound page
names next to ``autograd_loss_and_logits_grad``).  Together they make a dropped
term, a sign error, a wrong index or a transposed operand fail somewhere.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(B, V, seed, sigma=2.0, ignore_frac=0.2, ii=-100):
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, sigma, size=(B, V))
    t = rng.integers(0, V, size=B)
    k = int(ignore_frac * B)
    if k:
        t[rng.choice(B, k, replace=False)] = ii
    return x, t


def _loss_only(x, t, ii, red, z):
    return oracle.cross_entropy(x, t, ii, red, z, with_grad=False)["loss"]


# -- closed forms -------------------------------------------------------------

def test_golden_four_class_worked_example():
    with open(os.path.join(GOLDEN, "ce_closed_form.json")) as f:
        g = json.load(f)
    x = np.log(np.array([[1.0, 2.0, 3.0, 4.0]]))
    t = np.array([g["target"]])
    r = oracle.cross_entropy(x, t, reduction="sum", z_loss=0.0)
    assert r["loss"] == pytest.approx(math.log(2.5), rel=1e-15)
    assert r["lse"][0] == pytest.approx(math.log(10.0), rel=1e-15)
    np.testing.assert_allclose(r["grad"][0], g["grad_z0"], rtol=0, atol=1e-15)
    z = g["z_cases"][0]["z"]
    rz = oracle.cross_entropy(x, t, reduction="sum", z_loss=z)
    assert rz["loss"] == pytest.approx(math.log(2.5) + z * math.log(10.0) ** 2, rel=1e-15)
    expect = (1.0 + 2.0 * z * math.log(10.0)) * np.array(g["softmax"]) - np.array([0, 0, 0, 1.0])
    np.testing.assert_allclose(rz["grad"][0], expect, rtol=0, atol=1e-15)


@pytest.mark.parametrize("V", [1, 2, 7, 1024, 50257])
@pytest.mark.parametrize("c", [0.0, -3.5, 12.25])
@pytest.mark.parametrize("z", [0.0, 1e-4, 0.3])
def test_uniform_logits_give_log_V(V, c, z):
    B = 4
    x = np.full((B, V), c)
    t = np.array([0, V - 1, -100, V // 2])
    r = oracle.cross_entropy(x, t, reduction="mean", z_loss=z)
    lse = c + math.log(V)
    assert r["loss"] == pytest.approx(math.log(V) + z * lse * lse, rel=1e-13, abs=1e-13)
    scale = 1.0 / 3
    g = r["grad"]
    k = scale * (1 + 2 * z * lse) / V
    for i, ti in enumerate(t):
        if ti == -100:
            assert not g[i].any()
            continue
        expect = np.full(V, k)
        expect[ti] -= scale
        np.testing.assert_allclose(g[i], expect, rtol=1e-13, atol=1e-16)


# -- library special case (z = 0) ----------------------------------------------

@pytest.mark.parametrize("reduction", ["mean", "sum"])
@pytest.mark.parametrize("B,V,ii", [(1, 5, -100), (16, 33, -100), (64, 1024, -100), (9, 17, 3)])
def test_matches_torch_cross_entropy(reduction, B, V, ii):
    x, t = _rand_problem(B, V, seed=B * 1000 + V, ii=ii)
    r = oracle.cross_entropy(x, t, ignore_index=ii, reduction=reduction, z_loss=0.0)
    xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    lt = torch.nn.functional.cross_entropy(xt, torch.tensor(t), ignore_index=ii, reduction=reduction)
    lt.backward()
    assert r["loss"] == pytest.approx(lt.item(), rel=1e-13, abs=1e-15)
    np.testing.assert_allclose(r["grad"], xt.grad.numpy(), rtol=1e-12, atol=1e-15)


# -- finite differences (z > 0 has no library counterpart) --------------------

@pytest.mark.parametrize("reduction", ["mean", "sum"])
@pytest.mark.parametrize("z", [0.0, 1e-2, 0.25])
def test_grad_matches_central_differences(reduction, z):
    x, t = _rand_problem(4, 6, seed=7, ignore_frac=0.25)
    r = oracle.cross_entropy(x, t, reduction=reduction, z_loss=z)
    h = 1e-6
    fd = np.zeros_like(x)
    for i in range(x.shape[0]):
        for j in range(x.shape[1]):
            xp = x.copy(); xp[i, j] += h
            xm = x.copy(); xm[i, j] -= h
            fd[i, j] = (_loss_only(xp, t, -100, reduction, z) - _loss_only(xm, t, -100, reduction, z)) / (2 * h)
    np.testing.assert_allclose(r["grad"], fd, rtol=1e-7, atol=1e-8)


# -- invariants ---------------------------------------------------------------

@pytest.mark.parametrize("z", [0.0, 1e-4, 0.1])
def test_gradient_row_sums(z):
    # sum_j g_ij = scale * ((1 + 2 z lse) * 1 - 1) = scale * 2 z lse
    x, t = _rand_problem(32, 129, seed=3)
    r = oracle.cross_entropy(x, t, reduction="mean", z_loss=z)
    n = int((t != -100).sum())
    for i in range(32):
        s = r["grad"][i].sum()
        if t[i] == -100:
            assert s == 0.0
        else:
            assert s == pytest.approx(2 * z * r["lse"][i] / n, abs=1e-14)


def test_ignored_rows_exactly_zero_and_mean_denominator():
    x, t = _rand_problem(50, 40, seed=11, ignore_frac=0.3)
    rm = oracle.cross_entropy(x, t, reduction="mean", z_loss=1e-3)
    rs = oracle.cross_entropy(x, t, reduction="sum", z_loss=1e-3)
    ign = t == -100
    assert ign.sum() == 15
    assert np.all(rm["grad"][ign] == 0.0) and np.all(rs["grad"][ign] == 0.0)
    assert np.all(rm["row_loss"][ign] == 0.0)
    assert rs["loss"] / rm["loss"] == pytest.approx(35.0, rel=1e-14)
    np.testing.assert_allclose(rs["grad"], 35.0 * rm["grad"], rtol=1e-13, atol=0)


def test_all_rows_ignored_gives_zero():
    x, t = _rand_problem(5, 9, seed=1, ignore_frac=0.0)
    t[:] = -100
    for red in ("mean", "sum"):
        r = oracle.cross_entropy(x, t, reduction=red, z_loss=1e-4)
        assert r["loss"] == 0.0 and r["n_valid"] == 0
        assert not r["grad"].any()


def test_ignore_index_inside_class_range_is_ignored():
    x, t = _rand_problem(6, 8, seed=2, ignore_frac=0.0)
    t[:] = [3, 1, 3, 0, 3, 7]
    r = oracle.cross_entropy(x, t, ignore_index=3, reduction="mean")
    assert r["n_valid"] == 3
    assert not r["grad"][[0, 2, 4]].any()


def test_out_of_range_target_raises():
    x, t = _rand_problem(3, 4, seed=0, ignore_frac=0.0)
    t[1] = 4
    with pytest.raises(ValueError):
        oracle.cross_entropy(x, t)
    t[1] = -1
    with pytest.raises(ValueError):
        oracle.cross_entropy(x, t)


def test_shift_invariance_without_z_loss():
    x, t = _rand_problem(8, 31, seed=5)
    shift = np.random.default_rng(0).normal(0, 50, size=(8, 1))
    a = oracle.cross_entropy(x, t, z_loss=0.0)
    b = oracle.cross_entropy(x + shift, t, z_loss=0.0)
    assert a["loss"] == pytest.approx(b["loss"], rel=1e-12)
    np.testing.assert_allclose(a["grad"], b["grad"], rtol=1e-9, atol=1e-14)
    # with z > 0 the loss must move with the shift (lse**2 is not shift-invariant)
    c = oracle.cross_entropy(x, t, z_loss=0.1)
    d = oracle.cross_entropy(x + shift, t, z_loss=0.1)
    assert abs(c["loss"] - d["loss"]) > 1e-3


@pytest.mark.parametrize("z", [0.0, 1e-4])
def test_gradient_bounds_and_sign(z):
    x, t = _rand_problem(40, 77, seed=8, sigma=4.0)
    r = oracle.cross_entropy(x, t, reduction="mean", z_loss=z)
    n = int((t != -100).sum())
    s = 1.0 / n
    for i in range(40):
        if t[i] == -100:
            continue
        hi = s * (1 + 2 * z * r["lse"][i])
        g = r["grad"][i]
        assert g.min() >= -s - 1e-18 and g.max() <= hi + 1e-18
        neg = np.nonzero(g < 0)[0]
        assert set(neg.tolist()) <= {int(t[i])}


def test_large_spike_at_target_gives_near_zero_loss():
    rng = np.random.default_rng(4)
    V = 4096
    x = 4.0 * rng.standard_t(3, size=(2, V))
    t = np.array([10, 20])
    x[0, 10] += 1000.0  # target spike: every other term is below exp(-900)
    x[1, 30] += 1000.0  # non-target spike: loss is the spike's height above x_t
    r = oracle.cross_entropy(x, t, reduction="sum", z_loss=0.0)
    assert 0.0 <= r["row_loss"][0] < 1e-300
    assert r["row_loss"][1] == pytest.approx(x[1, 30] - x[1, 20], rel=1e-12)


def test_lse_between_max_and_max_plus_log_V():
    # max_j x_j <= lse <= max_j x_j + log V for every row, heavy tails included
    rng = np.random.default_rng(14)
    x = 4.0 * rng.standard_t(3, size=(64, 999))
    t = rng.integers(0, 999, size=64)
    r = oracle.cross_entropy(x, t, reduction="sum")
    m = x.max(axis=1)
    assert np.all(r["lse"] >= m) and np.all(r["lse"] <= m + math.log(999) + 1e-12)


def test_extreme_logits_stay_finite():
    x = np.array([[1e4, -1e4, 0.0, 1e4 - 1.0], [-3e4, -3e4, -3e4, -3e4]])
    t = np.array([1, 2])
    r = oracle.cross_entropy(x, t, reduction="sum", z_loss=0.0)
    assert np.isfinite(r["loss"]) and np.isfinite(r["grad"]).all()
    assert r["row_loss"][1] == pytest.approx(math.log(4.0), rel=1e-12)


# -- rounding helper and selective log-softmax ---------------------------------

def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-30, 2000) * 1e-8,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, 1e-40])])
    v32 = v.astype(np.float32)
    expect = torch.tensor(v32).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_round(v32.astype(np.float64))
    np.testing.assert_array_equal(got, expect)


def test_selective_log_softmax_matches_torch():
    rng = np.random.default_rng(9)
    x = rng.normal(0, 3, size=(3, 5, 41))
    idx = rng.integers(0, 41, size=(3, 5))
    got = oracle.selective_log_softmax(x, idx)
    xt = torch.tensor(x)
    expect = torch.gather(xt.log_softmax(-1), -1, torch.tensor(idx).unsqueeze(-1)).squeeze(-1)
    np.testing.assert_allclose(got, expect.numpy(), rtol=1e-13, atol=1e-13)


def test_selective_log_softmax_equals_negative_row_loss():
    x, t = _rand_problem(12, 50, seed=12, ignore_frac=0.0)
    r = oracle.cross_entropy(x, t, reduction="sum")
    np.testing.assert_allclose(oracle.selective_log_softmax(x, t), -r["row_loss"], rtol=1e-14)


# -- the VJP ------------------------------------------------------------------

def test_vjp_matches_central_differences_of_the_weighted_row_losses():
    # d/dx sum_r g_r * (lse_r - x_{r,t_r}) by central differences, ignored rows included
    x, t = _rand_problem(5, 7, seed=21, ignore_frac=0.4)
    g = np.random.default_rng(3).normal(size=5)
    out = oracle.ce_vjp(x, t, -100, g)

    def f(xx):
        _, rl, _ = oracle.ce_rows(xx, t, -100, 0.0, 1.0, with_grad=False)
        return float((g * rl).sum())

    h = 1e-6
    fd = np.zeros_like(x)
    for i in range(x.shape[0]):
        for j in range(x.shape[1]):
            xp = x.copy(); xp[i, j] += h
            xm = x.copy(); xm[i, j] -= h
            fd[i, j] = (f(xp) - f(xm)) / (2 * h)
    np.testing.assert_allclose(out, fd, rtol=1e-7, atol=1e-8)
    assert not out[t == -100].any()


def test_vjp_matches_torch_autograd_and_the_scaled_row_gradient():
    x, t = _rand_problem(9, 13, seed=22, ignore_frac=0.2)
    g = np.random.default_rng(4).uniform(-2, 2, size=9)
    xt = torch.tensor(x, requires_grad=True)
    tt = torch.tensor(np.where(t == -100, -100, t))
    rl = torch.nn.functional.cross_entropy(xt, tt, ignore_index=-100, reduction="none")
    (rl * torch.tensor(g)).sum().backward()
    out = oracle.ce_vjp(x, t, -100, g)
    np.testing.assert_allclose(out, xt.grad.numpy(), rtol=1e-12, atol=1e-14)
    # with z = 0 the unscaled row gradient times g is the VJP
    _, _, G = oracle.ce_rows(x, t, -100, 0.0, 1.0)
    np.testing.assert_allclose(out, G * g[:, None], rtol=1e-12, atol=1e-15)
