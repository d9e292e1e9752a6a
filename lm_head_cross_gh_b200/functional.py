"""Greyhound-style functional API (the names and signatures of
``greyhound.nn.functional``) over the C ABI, with PyTorch autograd.

Every loss is computed by the library's kernels in the forward call, together
with its gradients (they come out of the same passes); ``backward`` returns
them, multiplied on the device by the upstream gradient.  PyTorch only holds
the tensors: there is no other implementation behind these functions.

* ``cross_entropy(logits, target, ignore_index, reduction, z_loss_multiplier)``
* ``chunked_linear_cross_entropy(inputs, weight, target, ignore_index, reduction,
  z_loss_multiplier, grad_weight_accum_dtype)``
* ``chunked_linear_loss(inputs, weight, loss_and_grad_fn, *loss_args, chunk_size,
  grad_weight_accum_dtype, **loss_kwargs)``
* ``autograd_loss_and_logits_grad(loss_fn)``: adapts a PyTorch scalar loss to
  the ``(loss, grad_logits)`` contract of ``chunked_linear_loss``
* ``selective_log_softmax(logits, index)`` (forward only)

Data parallel (one process per GPU, a batch split over the ranks of a
``torch.distributed`` group):

* ``data_parallel_cross_entropy`` and ``data_parallel_chunked_linear_cross_entropy``
  return the whole batch's loss on every rank and, in backward, this rank's share
  of its gradients: the valid-token counts are summed over the ranks first (one
  int64 all-reduce), every shard divides by that total, the shards' losses are
  summed (one scalar all-reduce) and so are the weight gradients (fp32
  accumulators summed in fp32 and rounded once, for fp32 accumulation).
"""
from __future__ import annotations

import torch

from . import (gh_ce_fwd, gh_ce_fwd_bwd, gh_chunked_linear_loss, gh_linear_ce, gh_selective_log_softmax)

_PKG = __name__.rpartition(".")[0]

__all__ = ["cross_entropy", "chunked_linear_cross_entropy", "chunked_linear_loss",
           "autograd_loss_and_logits_grad", "selective_log_softmax", "data_parallel_cross_entropy",
           "data_parallel_chunked_linear_cross_entropy"]


def _scaled(grad, g):
    """grad * g for the scalar upstream gradient g.

    The product is always formed on the device: testing ``g == 1`` first would
    read g back to the host, which stalls the stream on every backward and is
    not allowed while a CUDA graph is being captured."""
    if grad is None:
        return None
    return grad * g.to(grad.dtype)


class _CrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, logits, target, ignore_index, reduction, z):
        V = logits.shape[-1]
        x = logits.reshape(-1, V).contiguous()
        t = target.reshape(-1).contiguous()
        ctx.shape = logits.shape
        if ctx.needs_input_grad[0]:
            loss, grad = gh_ce_fwd_bwd(x, t, ignore_index, reduction, z)
            ctx.save_for_backward(grad)
        else:
            loss, _ = gh_ce_fwd(x, t, ignore_index, reduction, z)
        return loss

    @staticmethod
    def backward(ctx, g):
        (grad,) = ctx.saved_tensors
        return _scaled(grad, g).view(ctx.shape), None, None, None, None


def cross_entropy(logits, target, ignore_index: int = -100, reduction: str = "mean",
                  z_loss_multiplier: float = 0.0):
    """Cross-entropy of ``logits`` [..., V] (float32 or bfloat16, CUDA) against
    ``target`` [...] (int64) with ``ignore_index``, ``"mean"``/``"sum"`` reduction
    and the z-loss ``z_loss_multiplier * lse**2``.  Returns a float32 scalar; its
    backward gives the logits gradient computed in the forward pass."""
    return _CrossEntropy.apply(logits, target, ignore_index, reduction, float(z_loss_multiplier))


class _LinearCE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, inputs, weight, target, ignore_index, reduction, z, accum):
        loss, dX, dW = gh_linear_ce(inputs.contiguous(), weight.contiguous(), target.contiguous(), ignore_index,
                                    reduction, z, 0, accum)
        ctx.save_for_backward(dX, dW)
        return loss

    @staticmethod
    def backward(ctx, g):
        dX, dW = ctx.saved_tensors
        return (_scaled(dX, g) if ctx.needs_input_grad[0] else None,
                _scaled(dW, g) if ctx.needs_input_grad[1] else None, None, None, None, None, None)


def chunked_linear_cross_entropy(inputs, weight, target, ignore_index: int = -100, reduction: str = "mean",
                                 z_loss_multiplier: float = 0.0, grad_weight_accum_dtype: str = "fp32"):
    """Cross-entropy of ``inputs @ weight.T`` (bf16 [BT, D] and [V, D], CUDA)
    computed in row chunks without materialising the logits; the backward gives
    grad_inputs and grad_weight (accumulated in fp32 or in the weight dtype)."""
    return _LinearCE.apply(inputs, weight, target, ignore_index, reduction, float(z_loss_multiplier),
                           grad_weight_accum_dtype)


class _ChunkedLoss(torch.autograd.Function):
    @staticmethod
    def forward(ctx, inputs, weight, loss_and_grad_fn, chunk, accum, args, kwargs):
        loss, dX, dW = gh_chunked_linear_loss(inputs.contiguous(), weight.contiguous(), loss_and_grad_fn, *args,
                                              chunk=chunk, accum=accum, **kwargs)
        ctx.save_for_backward(dX, dW)
        return loss

    @staticmethod
    def backward(ctx, g):
        dX, dW = ctx.saved_tensors
        return (_scaled(dX, g) if ctx.needs_input_grad[0] else None,
                _scaled(dW, g) if ctx.needs_input_grad[1] else None, None, None, None, None, None)


def chunked_linear_loss(inputs, weight, loss_and_grad_fn, *loss_args, chunk_size=None,
                        grad_weight_accum_dtype: str = "fp32", **loss_kwargs):
    """``inputs @ weight.T`` in row chunks followed by the caller's
    ``loss_and_grad_fn(logits_chunk, *chunk_args, **chunk_kwargs) -> (loss,
    grad_logits)``; tensor arguments whose leading dimension is BT are sliced to
    the chunk's rows.  Returns the sum of the chunk losses."""
    return _ChunkedLoss.apply(inputs, weight, loss_and_grad_fn, int(chunk_size or 0), grad_weight_accum_dtype,
                              loss_args, loss_kwargs)


def autograd_loss_and_logits_grad(loss_fn):
    """Adapt a PyTorch scalar loss ``loss_fn(logits, *args, **kwargs)`` to the
    ``(loss, grad_logits)`` contract: the loss is evaluated on an fp32 copy of
    the chunk logits and differentiated by autograd; the gradient comes back in
    the logits dtype."""
    def loss_and_grad(logits, *args, **kwargs):
        with torch.enable_grad():
            x = logits.detach().float().requires_grad_(True)
            loss = loss_fn(x, *args, **kwargs)
            (g,) = torch.autograd.grad(loss, x)
        return loss.detach(), g.to(logits.dtype)
    return loss_and_grad


def selective_log_softmax(logits, index):
    """``log_softmax(logits)`` gathered at ``index`` (forward only): float32 [...]."""
    return gh_selective_log_softmax(logits.contiguous(), index.contiguous())


def _ops(ops):
    """The library's entry points (``ops`` stands in for them in host-only tests
    of the collective steps)."""
    if ops is not None:
        return ops
    import importlib
    return importlib.import_module(_PKG)


def _all_reduce_sum(t, group):
    import torch.distributed as dist
    dist.all_reduce(t.view(-1), op=dist.ReduceOp.SUM, group=group)
    return t


class _DPCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, logits, target, ignore_index, reduction, z, group, ops):
        V = logits.shape[-1]
        x = logits.reshape(-1, V).contiguous()
        t = target.reshape(-1).contiguous()
        n = _all_reduce_sum(ops.gh_count_valid(t, V, ignore_index), group)
        loss, grad = ops.gh_ce_fwd_bwd_shard(x, t, n, ignore_index, reduction, z)
        loss = _all_reduce_sum(loss, group)
        ctx.shape = logits.shape
        ctx.save_for_backward(grad)
        return loss

    @staticmethod
    def backward(ctx, g):
        (grad,) = ctx.saved_tensors
        return _scaled(grad, g).view(ctx.shape), None, None, None, None, None, None


def data_parallel_cross_entropy(logits, target, ignore_index: int = -100, reduction: str = "mean",
                                z_loss_multiplier: float = 0.0, group=None, ops=None):
    """``cross_entropy`` of the whole batch whose shard ``logits`` / ``target``
    this rank holds (the mean divides by the valid count over all ranks)."""
    return _DPCrossEntropy.apply(logits, target, ignore_index, reduction, float(z_loss_multiplier), group,
                                 _ops(ops))


class _DPLinearCE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, inputs, weight, target, ignore_index, reduction, z, accum, group, ops, slices, comm_sms):
        import torch.distributed as dist
        t = target.contiguous()
        n = _all_reduce_sum(ops.gh_count_valid(t, weight.shape[0], ignore_index), group)
        if accum == "fp32":
            # every shard's fp32 accumulator is summed in fp32 and the batch's sum
            # is rounded to the weight dtype once; the sum of each range of
            # weight rows starts as soon as the last chunk has computed it, while
            # the other ranges are still being computed
            V, D = weight.shape
            dW32 = torch.empty((V, D), dtype=torch.float32, device=weight.device)
            works = []

            def on_slice(v0, v1):
                works.append(dist.all_reduce(dW32[v0:v1], op=dist.ReduceOp.SUM, group=group, async_op=True))

            max_sms = 0
            if weight.is_cuda and comm_sms > 0:
                max_sms = max(2, torch.cuda.get_device_properties(weight.device).multi_processor_count - comm_sms)
            loss, dX, _ = ops.gh_linear_ce_shard_f32(inputs.contiguous(), weight.contiguous(), t, n, ignore_index,
                                                     reduction, z, 0, grad_weight_f32=dW32, on_slice=on_slice,
                                                     dw_slices=max(1, int(slices)), max_sms=max_sms)
            for w in works:
                w.wait()
            dW = ops.gh_cast_f32_to_bf16(dW32)
        else:
            # "weight": each shard rounds between its chunks; the shards' sums are
            # added in the weight dtype
            loss, dX, dW = ops.gh_linear_ce_shard(inputs.contiguous(), weight.contiguous(), t, n, ignore_index,
                                                  reduction, z, 0, accum)
            dW = _all_reduce_sum(dW, group)
        loss = _all_reduce_sum(loss, group)
        ctx.save_for_backward(dX, dW)
        return loss

    @staticmethod
    def backward(ctx, g):
        dX, dW = ctx.saved_tensors
        return (_scaled(dX, g) if ctx.needs_input_grad[0] else None,
                _scaled(dW, g) if ctx.needs_input_grad[1] else None, None, None, None, None, None, None, None,
                None, None)


def data_parallel_chunked_linear_cross_entropy(inputs, weight, target, ignore_index: int = -100,
                                               reduction: str = "mean", z_loss_multiplier: float = 0.0,
                                               grad_weight_accum_dtype: str = "fp32", group=None, ops=None,
                                               overlap_slices: int = 4, comm_sms: int = 16):
    """``chunked_linear_cross_entropy`` of the whole batch whose rows ``inputs`` /
    ``target`` this rank holds, with the weight replicated: the weight gradient
    is summed over the ranks, in fp32 and rounded once for
    ``grad_weight_accum_dtype="fp32"``, in the weight dtype for ``"weight"``.

    For fp32 accumulation the last chunk's weight-gradient contraction runs in
    ``overlap_slices`` ranges of weight rows on all but ``comm_sms`` SMs, and
    each range's all-reduce is issued (asynchronously) as soon as it is
    enqueued, so the communication of the first ranges overlaps the
    computation of the rest."""
    return _DPLinearCE.apply(inputs, weight, target, ignore_index, reduction, float(z_loss_multiplier),
                             grad_weight_accum_dtype, group, _ops(ops), int(overlap_slices), int(comm_sms))
