"""Float64 oracle for the chunked linear cross-entropy (test infrastructure only).

Follows the Greyhound functional API page, ``chunked_linear_loss`` and
``chunked_linear_cross_entropy``: logits ``inputs @ weight.T`` are evaluated in
row chunks; for each chunk the fused cross-entropy gives the chunk's loss and
logits gradient G_c; ``grad_inputs[chunk] = G_c @ weight`` and
``grad_weight += G_c.T @ inputs[chunk]``.  The returned loss is the sum of the
chunks' losses; with ``reduction="mean"`` every chunk divides by the global
number of valid tokens (the reading under which chunking does not change the
result).

Accumulation of ``grad_weight`` (``grad_weight_accum_dtype``):

* ``"fp32"`` keeps a wide accumulator and casts once at the end.  The oracle's
  accumulator is float64 and it returns it unrounded; the output dtype's final
  rounding is left to the comparison.
* ``"weight"`` accumulates in the parameter dtype (bf16), which "rounds
  between chunks": after each chunk the oracle adds the chunk's product to the
  accumulator and rounds the sum to bf16.

Inputs are the exact float64 values of the bf16 tensors the GPU sees.
"""
from __future__ import annotations

import numpy as np

from .ce import bf16_round, ce_rows, cross_entropy, n_valid_and_scale


def linear_cross_entropy(X: np.ndarray, W: np.ndarray, targets: np.ndarray,
                         ignore_index: int = -100, reduction: str = "mean",
                         z_loss: float = 0.0, chunk: int = 0, accum: str = "fp32"):
    """Chunked linear cross-entropy.  Returns dict(loss, grad_inputs, grad_weight, lse).

    ``chunk`` is the number of rows per logits chunk (<= 0 or >= N: one chunk).
    """
    if accum not in ("fp32", "weight"):
        raise ValueError("accum must be 'fp32' or 'weight'")
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    t = np.asarray(targets, dtype=np.int64)
    N, D = X.shape
    V, D2 = W.shape
    if D != D2:
        raise ValueError("inputs and weight disagree on D")
    n_valid, scale = n_valid_and_scale(t, ignore_index, reduction, V)
    if chunk <= 0 or chunk > N:
        chunk = max(N, 1)
    loss_sum = 0.0
    lse = np.empty(N)
    dX = np.zeros((N, D))
    dW = np.zeros((V, D))
    for c0 in range(0, N, chunk):
        c1 = min(N, c0 + chunk)
        Z = X[c0:c1] @ W.T
        l, row_loss, G = ce_rows(Z, t[c0:c1], ignore_index, z_loss, scale)
        lse[c0:c1] = l
        loss_sum += float(np.sum(row_loss))
        dX[c0:c1] = G @ W
        part = G.T @ X[c0:c1]
        if accum == "fp32":
            dW += part
        else:
            dW = bf16_round(dW + part)
    loss = loss_sum / max(n_valid, 1) if reduction == "mean" else loss_sum
    return {"loss": loss, "grad_inputs": dX, "grad_weight": dW, "lse": lse, "n_valid": n_valid}


def linear_cross_entropy_materialised(X: np.ndarray, W: np.ndarray, targets: np.ndarray,
                                      ignore_index: int = -100, reduction: str = "mean",
                                      z_loss: float = 0.0):
    """Brute force: the full logits ``X @ W.T``, then cross-entropy, then both GEMMs."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    Z = X @ W.T
    r = cross_entropy(Z, targets, ignore_index, reduction, z_loss)
    G = r["grad"]
    return {"loss": r["loss"], "grad_inputs": G @ W, "grad_weight": G.T @ X,
            "lse": r["lse"], "n_valid": r["n_valid"]}


# ---------------------------------------------------------------------------
# Sampled outputs: the same definitions evaluated for chosen rows or chosen
# vocabulary entries, for problems too large to materialise (the Llama-3-8B
# head's logits are 16384 x 128256).  Every one equals the corresponding
# slice of ``linear_cross_entropy`` with fp32 accumulation.
# ---------------------------------------------------------------------------

def row_lse(X: np.ndarray, W: np.ndarray, row_block: int = 256) -> np.ndarray:
    """lse_i = log sum_v exp(X_i . W_v) for every row, the logits formed one
    block of rows at a time (float64, host BLAS)."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    N = X.shape[0]
    lse = np.empty(N)
    for r0 in range(0, N, row_block):
        Z = X[r0:r0 + row_block] @ W.T
        m = Z.max(axis=1)
        lse[r0:r0 + row_block] = m + np.log(np.exp(Z - m[:, None]).sum(axis=1))
    return lse


def loss_from_lse(X: np.ndarray, W: np.ndarray, targets: np.ndarray, lse: np.ndarray,
                  ignore_index: int = -100, reduction: str = "mean", z_loss: float = 0.0) -> float:
    """The reduced loss given every row's lse: row loss (lse - x_t) + z lse^2
    for valid rows, x_t = X_i . W_{t_i}; summed, and divided by the valid
    count for "mean"."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    t = np.asarray(targets, dtype=np.int64)
    n_valid, _ = n_valid_and_scale(t, ignore_index, reduction, W.shape[0])
    vr = np.nonzero(t != ignore_index)[0]
    x_t = np.einsum("ij,ij->i", X[vr], W[t[vr]])
    total = float(np.sum((lse[vr] - x_t) + z_loss * lse[vr] * lse[vr]))
    return total / max(n_valid, 1) if reduction == "mean" else total


def grad_input_rows(X: np.ndarray, W: np.ndarray, targets: np.ndarray, rows: np.ndarray,
                    ignore_index: int = -100, reduction: str = "mean", z_loss: float = 0.0) -> np.ndarray:
    """grad_inputs[rows] = G[rows] @ W, each row's logits gradient from its own
    full logits row (the scale uses the valid count of all targets)."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    t = np.asarray(targets, dtype=np.int64)
    _, scale = n_valid_and_scale(t, ignore_index, reduction, W.shape[0])
    _, _, G = ce_rows(X[rows] @ W.T, t[rows], ignore_index, z_loss, scale)
    return G @ W


def grad_weight_rows(X: np.ndarray, W: np.ndarray, targets: np.ndarray, lse: np.ndarray,
                     vocab: np.ndarray, ignore_index: int = -100, reduction: str = "mean",
                     z_loss: float = 0.0) -> np.ndarray:
    """grad_weight[vocab] = G[:, vocab]^T @ X (fp32 accumulation, unrounded):
    the logits gradient's columns ``vocab``, by definition
    G[i, v] = scale ((1 + 2 z lse_i) exp(X_i . W_v - lse_i) - [v == t_i]) for
    valid rows and 0 for ignored rows, need only those columns of the logits
    and every row's lse."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    t = np.asarray(targets, dtype=np.int64)
    vocab = np.asarray(vocab, dtype=np.int64)
    _, scale = n_valid_and_scale(t, ignore_index, reduction, W.shape[0])
    valid = t != ignore_index
    Zc = X @ W[vocab].T                                   # [N, len(vocab)]
    G = (scale * (1.0 + 2.0 * z_loss * lse))[:, None] * np.exp(Zc - lse[:, None])
    G -= scale * (valid[:, None] & (t[:, None] == vocab[None, :]))
    G[~valid] = 0.0
    return G.T @ X
