"""CPU oracle for next-token cross-entropy — test infrastructure only.

This package is the plain, slow, float64 statement of what the CUDA path
computes.  It is used only by ``tests/``, by ``__graft_entry__.smoke()`` and by
the CPU-baseline leg of ``bench.py``; the product path never imports it, and it
imports nothing from the product package.  It shares no kernels, helpers,
constants or pre/post-processing with the CUDA path: the only code both sides
use is the seeded input generator in ``gh_synth``, which holds none of the
method's arithmetic.

Sources (the Greyhound functional API page, ``greyhound.nn.functional``):

* ``cross_entropy`` — per-row loss ``logsumexp(x) - x[target]`` with an
  optional z-loss on the log-sum-exp, ``ignore_index`` masking, and ``mean``
  (divide by the number of valid tokens) or ``sum`` reduction; the gradient with
  respect to the logits is produced in the same pass.
* ``chunked_linear_loss`` / ``chunked_linear_cross_entropy`` — logits
  ``inputs @ weight.T`` evaluated in row chunks; per chunk the logits gradient
  G gives ``grad_inputs[chunk] = G @ weight`` and ``grad_weight += G.T @
  inputs[chunk]``, accumulated in fp32 (cast once) or in the weight dtype
  (rounded between chunks).
* nuvec ``FastOp::CrossEntropy`` / ``CrossEntropyVjp`` — the row loss
  definition and its logits gradient.

Readings where the API documentation is silent:
z-loss is ``z * lse**2`` per valid token, added before the reduction; ``mean``
with no valid token returns 0 with zero gradients; ``mean`` across chunks
divides by the global valid-token count; a target equal to ``ignore_index`` is
ignored even when it lies in [0, V); other targets outside [0, V) are an error.

Every function here is pinned by ``tests/test_oracle_*.py`` against closed
forms, invariants, finite differences, a materialised brute force and
``torch.nn.functional.cross_entropy`` (the PyTorch routine the z-free,
unchunked case reduces to).
"""
from .ce import (bf16_round, cross_entropy, ce_rows, ce_vjp, n_valid_and_scale,
                 selective_log_softmax)
from .linear_ce import (grad_input_rows, grad_weight_rows, linear_cross_entropy,
                        linear_cross_entropy_materialised, loss_from_lse, row_lse)

__all__ = [
    "bf16_round",
    "cross_entropy",
    "ce_rows",
    "ce_vjp",
    "n_valid_and_scale",
    "selective_log_softmax",
    "linear_cross_entropy",
    "linear_cross_entropy_materialised",
    "row_lse",
    "loss_from_lse",
    "grad_input_rows",
    "grad_weight_rows",
]
