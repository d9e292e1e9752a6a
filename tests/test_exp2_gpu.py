"""The two routes the cross-entropy kernels take to 2^y, checked on their own
through gh_exp2_eval (float64 numpy as the reference).

* "fma": the FMA-pipe form the two-pass ring uses for a quarter of the first
  pass's exponentials on long rows (Cody-Waite split y = r + f with r =
  round(y), a degree-5 polynomial for 2^f on [-0.5, 0.5], 2^r in the exponent
  field).  Over y in [-125, 0] its relative error is at most 2.2e-7 (the fit,
  plus Horner rounding) and its mean signed error is about 5e-8, so a sum of
  many terms is not biased; below -125 it returns 2^-125 (the clamp), and a
  NaN stays NaN.
* "mufu": ex2.approx.ftz.f32, the instruction every other exponential uses; the
  two routes agree to the sum of their errors.
"""
import numpy as np
import pytest
import torch

import lm_head_cross_gh_b200 as gh

pytestmark = pytest.mark.gpu

FMA_REL = 3.0e-7        # the polynomial's 2.1e-7 with margin for its fp32 Horner steps
MUFU_REL = 2.0 ** -20   # ex2.approx is specified to about 2^-22; 4x margin


def arguments():
    grid = np.linspace(-125.0, 0.0, 2_000_001).astype(np.float32)
    rnd = (-np.random.default_rng(11).random(1_000_000) * 125.0).astype(np.float32)
    near_int = (np.arange(-125, 1, dtype=np.float32)[:, None]
                + np.array([-0.5, -0.4999999, -1e-6, 0.0, 1e-6, 0.4999999, 0.5], np.float32)).ravel()
    near_int = near_int[(near_int >= -125.0) & (near_int <= 0.0)]
    return np.concatenate([grid, rnd, near_int])


def eval2(y: np.ndarray, method: str) -> np.ndarray:
    out = gh.gh_exp2_eval(torch.from_numpy(y).cuda(), method)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_fma_route_against_float64(cuda_device):
    y = arguments()
    ref = np.exp2(y.astype(np.float64))
    rel = eval2(y, "fma").astype(np.float64) / ref - 1.0
    worst = float(np.abs(rel).max())
    assert worst <= FMA_REL, f"max relative error {worst:.3g} at y = {y[np.abs(rel).argmax()]}"
    assert abs(float(rel.mean())) < 1.0e-7, f"mean signed error {rel.mean():.3g}"


def test_mufu_route_against_float64_and_the_fma_route(cuda_device):
    y = arguments()
    ref = np.exp2(y.astype(np.float64))
    mufu = eval2(y, "mufu").astype(np.float64)
    fma = eval2(y, "fma").astype(np.float64)
    worst = float(np.abs(mufu / ref - 1.0).max())
    assert worst <= MUFU_REL, f"ex2.approx max relative error {worst:.3g}"
    gap = float(np.abs(fma / mufu - 1.0).max())
    assert gap <= MUFU_REL + FMA_REL, f"routes differ by {gap:.3g}"


def test_fma_route_special_arguments(cuda_device):
    y = np.array([0.0, -125.0, -125.5, -126.0, -1000.0, -np.inf, np.nan, -np.nan], np.float32)
    out = eval2(y, "fma")
    assert abs(out[0] - 1.0) <= 2.0 ** -23                       # 2^0 within one fp32 step
    assert np.all(out[2:6] == out[1])                            # clamped at -125
    assert abs(float(out[1]) / 2.0 ** -125 - 1.0) <= FMA_REL
    assert np.isnan(out[6:]).all()
    assert np.isnan(eval2(y[6:], "mufu")).all()


def test_odd_lengths_and_empty(cuda_device):
    for n in (0, 1, 2, 3, 257, 513):
        y = (-np.arange(n, dtype=np.float32) * np.float32(124.0 / max(n, 1)))  # inside [-125, 0]
        out = eval2(y, "fma") if n else gh.gh_exp2_eval(torch.empty(0, device="cuda"), "fma").cpu().numpy()
        assert out.shape == (n,)
        if n:
            assert np.all(np.abs(out / np.exp2(y.astype(np.float64)) - 1.0) <= FMA_REL)
