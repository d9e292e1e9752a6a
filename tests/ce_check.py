"""Helpers shared by the GPU parity tests: device upload and tolerance checks.

Tolerances, derived from the kernels' fp32 arithmetic:

* Every exponent is evaluated as 2^(x*log2e - lse*log2e) with one fused
  multiply-add, whose argument carries an absolute rounding error of about
  2^-24 * |x| * log2e; the resulting relative error of p = exp(x - lse) and of
  lse itself is below eps_i = 4e-7 * max(1, max_j |x_ij|) for row i
  (ex2.approx adds ~2^-22).
* loss: |loss - ref| <= 1e-5 |ref| + sum_i eps_i * max(1, |lse_i|) over valid
  rows (divided by n_valid for "mean").  The 1e-5 relative part is the stated bar for fp32
  logits and tighter than the stated 1e-3 for bf16 (the loss is computed in
  fp32 from the exact input values, so bf16 inputs do not widen it).
* gradient, with q = |g_ref| + scale * onehot (the magnitude of
  scale * (1 + 2 z lse) * p, before the target's -scale):
  fp32: |g - g_ref| <= 2e-5 |g_ref| + eps * q + 2^-30 * scale;
  bf16: the stated bar max |g - g_ref| <= 2e-3 over elements with
  |g_ref| < 0.512 (above that a single bf16 rounding, up to 2^-8 |g|, exceeds
  2e-3: "sum" reduction gives |g| up to ~1), plus the per-element bound
  |g - g_ref| <= 2^-8 |g_ref| + (eps + 2^-11) q + 2^-24 * scale: one bf16
  rounding of the output plus one fp16 rounding of the cached exp(x - m)
  (2^-11 relative, applied before the target's -scale, hence on q),
  plus a bias check: the mean signed relative error over elements with
  |g_ref| > 1e-3 * scale stays below 2.5e-4, which unbiased rounding meets and
  a dropped factor (e.g. the z-loss's 1 + 2 z lse) does not.
"""
import numpy as np
import torch

import oracle


def to_device(p, device="cuda"):
    """(logits, targets) CUDA tensors of a gh_synth.CEInputs."""
    if p.dtype == "f32":
        x = torch.from_numpy(np.ascontiguousarray(p.logits)).to(device)
    else:
        x = torch.from_numpy(np.ascontiguousarray(p.logits).view(np.int16)).to(device).view(torch.bfloat16)
    t = torch.from_numpy(np.ascontiguousarray(p.targets)).to(device)
    return x, t


def grad_to_f64(g: torch.Tensor) -> np.ndarray:
    return g.float().cpu().numpy().astype(np.float64)


def row_eps(x: np.ndarray) -> np.ndarray:
    """Per-row relative error bound eps_i = 4e-7 * max(1, max_j |x_ij|), shape [rows, 1]."""
    if x.shape[1] == 0:
        return np.full((x.shape[0], 1), 4e-7)
    return (4e-7 * np.maximum(1.0, np.abs(x).max(axis=1)))[:, None]


def loss_atol(eps_rows: np.ndarray, lse: np.ndarray, valid: np.ndarray, reduction: str) -> float:
    """Absolute loss tolerance: sum over valid rows of eps_i * max(1, |lse_i|) (averaged for mean)."""
    e = eps_rows.reshape(-1)[valid] * np.maximum(1.0, np.abs(lse[valid]))
    tot = float(e.sum())
    return tot / max(int(valid.sum()), 1) if reduction == "mean" else tot


def check_loss(loss_gpu: float, loss_ref: float, atol: float, what=""):
    tol = 1e-5 * abs(loss_ref) + atol
    assert abs(loss_gpu - loss_ref) <= tol, f"{what} loss {loss_gpu!r} vs oracle {loss_ref!r} (tol {tol:.3g})"


def check_grad(g: np.ndarray, g_ref: np.ndarray, dtype: str, scale: float, targets: np.ndarray,
               ignore_index: int, eps: float, what=""):
    err = np.abs(g - g_ref)
    q = np.abs(g_ref).copy()
    valid = np.nonzero(targets != ignore_index)[0]
    q[valid, targets[valid]] += scale
    if dtype == "bf16":
        # the stated 2e-3 max-abs bar, wherever one bf16 rounding (2^-8 |g|) can meet it
        small = np.abs(g_ref) < 2e-3 * 2.0 ** 8
        assert (err[small].max() if small.any() else 0.0) <= 2e-3, f"{what} max-abs {err[small].max()}"
        bound = 2.0 ** -8 * np.abs(g_ref) + (eps + 2.0 ** -11) * q + 2.0 ** -24 * scale
    else:
        bound = 2e-5 * np.abs(g_ref) + eps * q + 2.0 ** -30 * scale
    bad = err > bound
    if bad.any():
        i = np.argmax(np.where(bad, err / np.maximum(bound, 1e-300), 0))
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside the bound; worst "
                             f"err {err.flat[i]:.3g} bound {bound.flat[i]:.3g} ref {g_ref.flat[i]:.3g}")
    if dtype == "bf16":
        big = np.abs(g_ref) > 1e-3 * scale
        if big.sum() > 1000:
            bias = float(np.mean((g[big] - g_ref[big]) / g_ref[big]))
            assert abs(bias) < 2.5e-4, f"{what} mean relative error {bias}"


def check_problem_full(p, loss_gpu: float, grad_gpu: np.ndarray, what=""):
    """Whole-problem parity against the oracle (small problems)."""
    x = p.values_f32().astype(np.float64)
    ref = oracle.cross_entropy(x, p.targets, p.ignore_index, p.reduction, p.z_loss)
    n_valid, scale = oracle.n_valid_and_scale(p.targets, p.ignore_index, p.reduction, p.V)
    eps = row_eps(x)
    valid = p.targets != p.ignore_index
    check_loss(loss_gpu, ref["loss"], loss_atol(eps, ref["lse"], valid, p.reduction), what)
    check_grad(grad_gpu, ref["grad"], p.dtype, scale, p.targets, p.ignore_index, eps, what)
    assert not grad_gpu[~valid].any(), f"{what} ignored rows must be exactly zero"
    return ref
