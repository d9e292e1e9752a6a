"""Seeded synthetic inputs for next-token cross-entropy workloads.

This module only draws and rounds input data: logits, hidden states, LM-head
weights and target ids.  It holds none of the cross-entropy arithmetic, so the
CPU oracle (``oracle/``) and the CUDA path can both consume the same arrays
without sharing any of the method's code.

Conventions
-----------
* Every draw comes from ``numpy.random.SeedSequence(seed)``.  Large tensors are
  cut into fixed row blocks, each block drawing from its own spawned child
  sequence, so the values do not depend on how many threads fill them.
* bf16 tensors are returned as ``uint16`` bit patterns, rounded from float32
  with round-to-nearest-even.  ``bf16_to_f32`` widens them exactly.
* Targets are int64 class ids.  "p% ignore_index" means exactly
  ``floor(p/100 * n)`` positions, chosen without replacement.
* The draw order inside one workload is fixed: values, then targets, then the
  ignore mask, then (large-vocab stress only) the spikes.

Shapes and value distributions follow the workloads of the Greyhound functional
API page (``cross_entropy`` takes contiguous ``[B, V]`` logits and ``[B]``
targets; ``chunked_linear_cross_entropy`` takes ``[BT, D]`` inputs and a
``[V, D]`` weight), the GPT-2 vocabulary of 50257 (lucid ``CausalLMOutput``
example) and the N(0, 0.02) initialisation of forge ``Gpt2::init_random``.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

IGNORE_INDEX = -100
_ROW_BLOCK_ELEMS = 1 << 22  # ~4M values per independently seeded block


# ---------------------------------------------------------------------------
# bf16 bit handling (input rounding only)
# ---------------------------------------------------------------------------

_ROUND_BLOCK = 1 << 20  # values per block of the bf16 rounding


def _round_block(u: np.ndarray, out: np.ndarray) -> None:
    # (u + 0x7FFF + lsb) >> 16 with lsb = bit 16 of u: nearest, ties to even.
    # Finite float32 patterns are at most 0xFF7FFFFF, so the sum fits 32 bits.
    t = (u >> 16) & np.uint32(1)
    t += u
    t += np.uint32(0x7FFF)
    t >>= 16
    out[...] = t


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest, ties to even); return uint16 bits.

    Works through the array in blocks (threads over blocks), so no temporary
    larger than a block is ever allocated."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).reshape(-1)
    out = np.empty(u.shape, dtype=np.uint16)
    starts = range(0, u.size, _ROUND_BLOCK)

    def work(i0: int) -> None:
        _round_block(u[i0:i0 + _ROUND_BLOCK], out[i0:i0 + _ROUND_BLOCK])

    if u.size <= _ROUND_BLOCK:
        for i0 in starts:
            work(i0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, starts))
    return out.reshape(x.shape)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly (block by block)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    flat = b.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint32)
    starts = range(0, flat.size, _ROUND_BLOCK)

    def work(i0: int) -> None:
        o = out[i0:i0 + _ROUND_BLOCK]
        o[...] = flat[i0:i0 + _ROUND_BLOCK]
        o <<= 16

    if flat.size <= _ROUND_BLOCK:
        for i0 in starts:
            work(i0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, starts))
    return out.view(np.float32).reshape(b.shape)


# ---------------------------------------------------------------------------
# block-parallel seeded fills
# ---------------------------------------------------------------------------

def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _fill_rows(seq: np.random.SeedSequence, rows: int, cols: int, draw) -> np.ndarray:
    """Fill a float32 [rows, cols] array block by block.

    ``draw(rng, n)`` returns ``n`` float32 values.  Block b covers a fixed row
    range and uses ``seq.spawn``'s b-th child, so the result is independent of
    the thread count.
    """
    out = np.empty((rows, cols), dtype=np.float32)
    if rows == 0 or cols == 0:
        return out
    rows_per_block = max(1, _ROW_BLOCK_ELEMS // max(cols, 1))
    nblocks = (rows + rows_per_block - 1) // rows_per_block
    children = seq.spawn(nblocks)

    def work(b: int) -> None:
        r0 = b * rows_per_block
        r1 = min(rows, r0 + rows_per_block)
        rng = np.random.default_rng(children[b])
        out[r0:r1] = draw(rng, (r1 - r0) * cols).reshape(r1 - r0, cols)

    if nblocks == 1:
        work(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nblocks)))
    return out


def _normal(sigma: float):
    def draw(rng, n):
        v = rng.standard_normal(n, dtype=np.float32)
        if sigma != 1.0:
            v *= np.float32(sigma)
        return v
    return draw


def _student_t(df: float, scale: float):
    # t = Z / sqrt(G / df) with G ~ chi-square(df) = 2 * Gamma(df / 2)
    def draw(rng, n):
        z = rng.standard_normal(n, dtype=np.float32)
        g = rng.standard_gamma(df / 2.0, n, dtype=np.float32)
        return (np.float32(scale) * z / np.sqrt(np.float32(2.0 / df) * g)).astype(np.float32)
    return draw


def _targets(rng: np.random.Generator, n: int, V: int, ignore_frac: float,
             ignore_index: int) -> np.ndarray:
    t = rng.integers(0, V, size=n, dtype=np.int64)
    k = int(np.floor(ignore_frac * n + 1e-9))
    if k > 0:
        idx = rng.choice(n, size=k, replace=False)
        t[idx] = ignore_index
    return t


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class CEInputs:
    """One standalone cross-entropy problem.

    ``logits`` is float32 [B, V] for dtype "f32" and uint16 bf16 bits [B, V]
    for dtype "bf16".  ``values_f32()`` gives the exact float32 values.
    """
    name: str
    dtype: str
    logits: np.ndarray
    targets: np.ndarray
    ignore_index: int
    reduction: str
    z_loss: float

    @property
    def B(self) -> int:
        return self.logits.shape[0]

    @property
    def V(self) -> int:
        return self.logits.shape[1]

    def values_f32(self, rows=slice(None)) -> np.ndarray:
        if self.dtype == "f32":
            return self.logits[rows]
        return bf16_to_f32(self.logits[rows])


@dataclasses.dataclass
class LinearCEInputs:
    """One chunked linear cross-entropy problem (bf16 inputs and weight)."""
    name: str
    inputs: np.ndarray   # uint16 bf16 bits [N, D]
    weight: np.ndarray   # uint16 bf16 bits [V, D]
    targets: np.ndarray  # int64 [N]
    chunk: int
    accum: str           # "fp32" | "weight"
    ignore_index: int
    reduction: str
    z_loss: float

    @property
    def N(self) -> int:
        return self.inputs.shape[0]

    @property
    def D(self) -> int:
        return self.inputs.shape[1]

    @property
    def V(self) -> int:
        return self.weight.shape[0]


def ce_normal(B: int, V: int, sigma: float, dtype: str = "bf16", ignore_frac: float = 0.0,
              reduction: str = "mean", z_loss: float = 0.0, seed: int = 0,
              ignore_index: int = IGNORE_INDEX, name: Optional[str] = None) -> CEInputs:
    """Logits ~ N(0, sigma^2), targets uniform in [0, V), a fraction ignored."""
    seq = np.random.SeedSequence(seed)
    s_vals, s_tgt = seq.spawn(2)
    x = _fill_rows(s_vals, B, V, _normal(sigma))
    t = _targets(np.random.default_rng(s_tgt), B, V, ignore_frac, ignore_index)
    logits = x if dtype == "f32" else f32_to_bf16(x)
    return CEInputs(name or f"ce_normal_{B}x{V}", dtype, logits, t, ignore_index, reduction, z_loss)


def ce_student_t_spiked(B: int, V: int, df: float = 3.0, scale: float = 4.0,
                        spike_frac: float = 0.10, spike: float = 30.0, dtype: str = "bf16",
                        reduction: str = "sum", z_loss: float = 1e-4, seed: int = 0,
                        ignore_index: int = IGNORE_INDEX, name: Optional[str] = None) -> CEInputs:
    """Heavy-tailed logits with +``spike`` added at one column of some rows.

    ``floor(spike_frac * B)`` rows, chosen without replacement, get the spike;
    the first half of them (in draw order) at the row's target column, the
    rest at a uniformly drawn column different from the target.
    """
    seq = np.random.SeedSequence(seed)
    s_vals, s_tgt, s_spk = seq.spawn(3)
    x = _fill_rows(s_vals, B, V, _student_t(df, scale))
    t = _targets(np.random.default_rng(s_tgt), B, V, 0.0, ignore_index)
    rng = np.random.default_rng(s_spk)
    k = int(np.floor(spike_frac * B + 1e-9))
    rows = rng.choice(B, size=k, replace=False)
    half = k // 2 + (k % 2)
    for j, r in enumerate(rows):
        if j < half:
            c = int(t[r])
        else:
            c = int(rng.integers(0, V - 1)) if V > 1 else 0
            if V > 1 and c >= t[r]:
                c += 1
        x[r, c] = np.float32(x[r, c] + np.float32(spike))
    logits = x if dtype == "f32" else f32_to_bf16(x)
    return CEInputs(name or f"ce_student_t_{B}x{V}", dtype, logits, t, ignore_index, reduction, z_loss)


def linear_ce_normal(N: int, D: int, V: int, chunk: int, ignore_frac: float = 0.0,
                     x_sigma: float = 1.0, w_sigma: float = 0.02, accum: str = "fp32",
                     reduction: str = "mean", z_loss: float = 0.0, seed: int = 0,
                     ignore_index: int = IGNORE_INDEX, name: Optional[str] = None) -> LinearCEInputs:
    """inputs ~ N(0, x_sigma^2) [N, D], weight ~ N(0, w_sigma^2) [V, D], bf16."""
    seq = np.random.SeedSequence(seed)
    s_x, s_w, s_t = seq.spawn(3)
    X = f32_to_bf16(_fill_rows(s_x, N, D, _normal(x_sigma)))
    W = f32_to_bf16(_fill_rows(s_w, V, D, _normal(w_sigma)))
    t = _targets(np.random.default_rng(s_t), N, V, ignore_frac, ignore_index)
    return LinearCEInputs(name or f"linear_ce_{N}x{D}x{V}", X, W, t, chunk, accum,
                          ignore_index, reduction, z_loss)


# The five named workloads: sizes, distributions and options exactly as
# stated for the GPT-2 / Llama-3-8B LM-head shapes.

def ce_small(z_loss: float = 0.0, seed: int = 0) -> CEInputs:
    """fp32 [64, 1024] ~ N(0, 2^2), 10% ignored, mean."""
    return ce_normal(64, 1024, 2.0, dtype="f32", ignore_frac=0.10, reduction="mean",
                     z_loss=z_loss, seed=seed, name="ce_small_fp32_64x1024")


def ce_gpt2(seed: int = 0) -> CEInputs:
    """bf16 [8192, 50257] ~ N(0, 3^2), 2% ignored, mean, z-loss 1e-4."""
    return ce_normal(8192, 50257, 3.0, dtype="bf16", ignore_frac=0.02, reduction="mean",
                     z_loss=1e-4, seed=seed, name="ce_gpt2_bf16_8192x50257")


def linear_ce_gpt2(seed: int = 0) -> LinearCEInputs:
    """GPT-2 small tied head: [8192, 768] x [50257, 768], chunk 2048, fp32 accum."""
    return linear_ce_normal(8192, 768, 50257, 2048, ignore_frac=0.0, accum="fp32",
                            reduction="mean", z_loss=0.0, seed=seed,
                            name="linear_ce_gpt2_8192x768x50257")


def linear_ce_llama3_8b(seed: int = 0) -> LinearCEInputs:
    """Llama-3-8B head: [16384, 4096] x [128256, 4096], 5% ignored, chunk 4096, z 1e-4."""
    return linear_ce_normal(16384, 4096, 128256, 4096, ignore_frac=0.05, accum="fp32",
                            reduction="mean", z_loss=1e-4, seed=seed,
                            name="linear_ce_llama3_8b_16384x4096x128256")


def ce_large_vocab(seed: int = 0) -> CEInputs:
    """bf16 [4096, 262144], 4 * Student-t(3), 10% rows spiked +30, sum, z 1e-4."""
    return ce_student_t_spiked(4096, 262144, df=3.0, scale=4.0, spike_frac=0.10, spike=30.0,
                               dtype="bf16", reduction="sum", z_loss=1e-4, seed=seed,
                               name="ce_large_vocab_bf16_4096x262144")
