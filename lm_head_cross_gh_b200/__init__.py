"""B200-native next-token cross-entropy: Python binding of ``libgh.so``.

The functions here only marshal arguments into the C ABI declared in
``include/gh.h``; every step of the computation runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
CPU or PyTorch fallback: if ``libgh.so`` is missing or a call fails, an
exception is raised.

* ``gh_ce_fwd_bwd`` — Greyhound ``cross_entropy``: loss and logits gradient of
  materialised ``[B, V]`` logits in one call.
* ``gh_linear_ce`` — Greyhound ``chunked_linear_cross_entropy``: loss,
  ``grad_inputs`` and ``grad_weight`` of ``inputs @ weight.T`` computed chunk
  by chunk, without the full logits.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgh.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "gh.h")

GH_OK = 0
GH_ERR_INVALID_ARG = 1
GH_ERR_UNSUPPORTED = 2
GH_ERR_ALLOC = 3
GH_ERR_CUDA = 4
GH_ERR_TIMEOUT = 5
GH_ERR_TARGET_RANGE = 6

GH_REDUCTION = {"mean": 0, "sum": 1}
GH_ACCUM = {"fp32": 0, "weight": 1}
GH_F32, GH_BF16 = 0, 1


class GhError(RuntimeError):
    """A libgh call returned a status other than GH_OK."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None

# gh_chunk_loss_fn(ctx, row0, rows, logits, ld, V, loss_accum, stream) -> gh_status_t
CHUNK_LOSS_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                 ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p)
DW_SLICE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p)


def lib() -> ctypes.CDLL:
    """The loaded ``libgh.so`` with argument types set (loads on first use)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m lm_head_cross_gh_b200._build` "
            "(nvcc, sm_100a).  There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    c_void_p, c_int64, c_int, c_float = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    L.gh_ce_fwd_bwd.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_int, c_int64, c_int, c_float,
                                c_void_p, c_void_p, c_void_p]
    L.gh_ce_fwd_bwd.restype = c_int
    L.gh_ce_fwd_bwd_noalloc.argtypes = list(L.gh_ce_fwd_bwd.argtypes)
    L.gh_ce_fwd_bwd_noalloc.restype = c_int
    L.gh_count_valid.argtypes = [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p]
    L.gh_count_valid.restype = c_int
    L.gh_ce_fwd_bwd_shard.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_int, c_int64, c_int, c_float,
                                      c_void_p, c_void_p, c_void_p, c_void_p]
    L.gh_ce_fwd_bwd_shard.restype = c_int
    L.gh_linear_ce_shard.argtypes = [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int64, c_int,
                                     c_int64, c_int, c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
    L.gh_linear_ce_shard.restype = c_int
    L.gh_linear_ce_shard_f32.argtypes = [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int64,
                                         c_int64, c_int, c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
    L.gh_linear_ce_shard_f32.restype = c_int
    L.gh_linear_ce_shard_f32_sliced.argtypes = list(L.gh_linear_ce_shard_f32.argtypes[:-1]) + [
        c_int64, c_int, DW_SLICE_FN, c_void_p, c_void_p]
    L.gh_linear_ce_shard_f32_sliced.restype = c_int
    L.gh_cast_f32_to_bf16.argtypes = [c_void_p, c_void_p, c_int64, c_void_p]
    L.gh_cast_f32_to_bf16.restype = c_int
    L.gh_ce_fwd.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_int, c_int64, c_int, c_float,
                            c_void_p, c_void_p, c_void_p]
    L.gh_ce_fwd.restype = c_int
    L.gh_chunked_linear_loss.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int64, c_int,
                                         CHUNK_LOSS_FN, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
    L.gh_chunked_linear_loss.restype = c_int
    L.gh_ce_vjp.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_int, c_int64, c_void_p, c_void_p, c_void_p,
                            c_void_p]
    L.gh_ce_vjp.restype = c_int
    L.gh_selective_log_softmax.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_int, c_void_p, c_void_p]
    L.gh_selective_log_softmax.restype = c_int
    L.gh_linear_ce.argtypes = [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int64, c_int,
                               c_int64, c_int, c_float, c_void_p, c_void_p, c_void_p, c_void_p]
    L.gh_linear_ce.restype = c_int
    L.gh_get_device_status.argtypes = [c_void_p]
    L.gh_get_device_status.restype = c_int
    L.gh_status_string.argtypes = [c_int]
    L.gh_status_string.restype = ctypes.c_char_p
    L.gh_version.argtypes = []
    L.gh_version.restype = ctypes.c_char_p
    L.gh_profile_enable.argtypes = [c_int]
    L.gh_profile_enable.restype = c_int
    L.gh_profile_read.argtypes = [c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_int64)]
    L.gh_profile_read.restype = c_int
    L.gh_launch_count.argtypes = []
    L.gh_launch_count.restype = c_int64
    L.gh_debug_set.argtypes = [c_int, c_int64]
    L.gh_debug_set.restype = c_int
    L.gh_exp2_eval.argtypes = [c_void_p, c_void_p, c_int64, c_int, c_void_p]
    L.gh_exp2_eval.restype = c_int
    _lib = L
    return L


def header_symbols() -> list:
    """Names of the functions ``include/gh.h`` declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"\btypedef\b[^;]*;", "", text, flags=re.S)  # enums and the callback type
    return sorted(set(re.findall(r"\b(gh_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().gh_status_string(int(status)).decode()


def gh_status_string(status: int) -> str:
    return status_string(status)


def gh_version() -> str:
    return lib().gh_version().decode()


def _check(status: int, where: str) -> None:
    if status != GH_OK:
        raise GhError(status, where)


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _need(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def gh_ce_fwd_bwd(logits, targets, ignore_index: int = -100, reduction: str = "mean",
                  z_loss: float = 0.0, *, grad=None, loss=None, stream=None):
    """Cross-entropy loss and logits gradient (one call into ``gh_ce_fwd_bwd``).

    ``logits``: CUDA tensor [B, V], float32 or bfloat16, contiguous.
    ``targets``: CUDA int64 [B].  ``grad`` (optional output, same shape and
    dtype; may be ``logits`` itself for the in-place form) and ``loss``
    (optional float32 scalar output) are allocated when not given.
    Returns ``(loss, grad)``; both are valid on ``stream`` when the call returns.
    """
    import torch
    _need(logits.dim() == 2 and logits.is_cuda and logits.is_contiguous(), "logits: contiguous CUDA [B, V]")
    _need(logits.dtype in (torch.float32, torch.bfloat16), "logits dtype must be float32 or bfloat16")
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (logits.shape[0],), "targets: contiguous CUDA int64 [B]")
    _need(reduction in GH_REDUCTION, "reduction must be 'mean' or 'sum'")
    if grad is None:
        grad = torch.empty_like(logits)
    _need(grad.shape == logits.shape and grad.dtype == logits.dtype and grad.is_contiguous(), "grad mismatch")
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=logits.device)
    _need(loss.dtype == torch.float32 and loss.numel() == 1, "loss must be a float32 scalar")
    B, V = logits.shape
    dtype = GH_F32 if logits.dtype == torch.float32 else GH_BF16
    st = lib().gh_ce_fwd_bwd(_ptr(logits), _ptr(targets), B, V, dtype, int(ignore_index),
                             GH_REDUCTION[reduction], float(z_loss), _ptr(loss), _ptr(grad),
                             _stream_handle(stream))
    _check(st, "gh_ce_fwd_bwd")
    return loss, grad


GH_NOALLOC_MAX_ROWS = 65536


def gh_ce_fwd_bwd_noalloc(logits, targets, ignore_index: int = -100, reduction: str = "mean",
                          z_loss: float = 0.0, *, grad, loss, stream=None):
    """``gh_ce_fwd_bwd`` without any device allocation inside the library.

    For callers that cannot allocate during a step (their device memory is
    owned by another allocator, or allocator calls are forbidden there).  The
    caller passes every output (``grad`` and the float32 scalar ``loss``);
    the library's scratch is a fixed device array shared by all calls, so
    calls that overlap on the GPU race.  ``B`` <= 65536.
    """
    import torch
    _need(logits.dim() == 2 and logits.is_cuda and logits.is_contiguous(), "logits: contiguous CUDA [B, V]")
    _need(logits.dtype in (torch.float32, torch.bfloat16), "logits dtype must be float32 or bfloat16")
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (logits.shape[0],), "targets: contiguous CUDA int64 [B]")
    _need(reduction in GH_REDUCTION, "reduction must be 'mean' or 'sum'")
    _need(grad.shape == logits.shape and grad.dtype == logits.dtype and grad.is_contiguous(), "grad mismatch")
    _need(loss.dtype == torch.float32 and loss.numel() == 1 and loss.is_cuda, "loss must be a CUDA float32 scalar")
    B, V = logits.shape
    dtype = GH_F32 if logits.dtype == torch.float32 else GH_BF16
    st = lib().gh_ce_fwd_bwd_noalloc(_ptr(logits), _ptr(targets), B, V, dtype, int(ignore_index),
                                     GH_REDUCTION[reduction], float(z_loss), _ptr(loss), _ptr(grad),
                                     _stream_handle(stream))
    _check(st, "gh_ce_fwd_bwd_noalloc")
    return loss, grad


def gh_count_valid(targets, V: int, ignore_index: int = -100, *, count=None, stream=None):
    """Number of targets that are not ``ignore_index`` (CUDA int64 scalar tensor)."""
    import torch
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous(), "targets: CUDA int64")
    if count is None:
        count = torch.empty((), dtype=torch.int64, device=targets.device)
    _need(count.dtype == torch.int64 and count.numel() == 1 and count.is_cuda, "count: CUDA int64 scalar")
    _check(lib().gh_count_valid(_ptr(targets), targets.numel(), int(V), int(ignore_index), _ptr(count),
                                _stream_handle(stream)), "gh_count_valid")
    return count


def gh_ce_fwd_bwd_shard(logits, targets, n_valid_total, ignore_index: int = -100, reduction: str = "mean",
                        z_loss: float = 0.0, *, grad=None, loss=None, stream=None):
    """``gh_ce_fwd_bwd`` for one shard of a data-parallel batch: the mean divides
    by ``n_valid_total`` (CUDA int64 scalar: the valid count of all shards)."""
    import torch
    _need(logits.dim() == 2 and logits.is_cuda and logits.is_contiguous(), "logits: contiguous CUDA [B, V]")
    _need(logits.dtype in (torch.float32, torch.bfloat16), "logits dtype must be float32 or bfloat16")
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (logits.shape[0],), "targets: contiguous CUDA int64 [B]")
    _need(n_valid_total.dtype == torch.int64 and n_valid_total.numel() == 1 and n_valid_total.is_cuda,
          "n_valid_total: CUDA int64 scalar")
    _need(reduction in GH_REDUCTION, "reduction must be 'mean' or 'sum'")
    if grad is None:
        grad = torch.empty_like(logits)
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=logits.device)
    B, V = logits.shape
    dtype = GH_F32 if logits.dtype == torch.float32 else GH_BF16
    st = lib().gh_ce_fwd_bwd_shard(_ptr(logits), _ptr(targets), B, V, dtype, int(ignore_index),
                                   GH_REDUCTION[reduction], float(z_loss), _ptr(n_valid_total), _ptr(loss),
                                   _ptr(grad), _stream_handle(stream))
    _check(st, "gh_ce_fwd_bwd_shard")
    return loss, grad


def gh_linear_ce_shard(inputs, weight, targets, n_valid_total, ignore_index: int = -100, reduction: str = "mean",
                       z_loss: float = 0.0, chunk: int = 0, accum: str = "fp32", *, grad_inputs=None,
                       grad_weight=None, loss=None, stream=None):
    """``gh_linear_ce`` for one shard of a data-parallel batch (mean over
    ``n_valid_total``, a CUDA int64 scalar)."""
    import torch
    _need(inputs.dim() == 2 and weight.dim() == 2 and inputs.shape[1] == weight.shape[1], "shapes")
    _need(inputs.dtype == torch.bfloat16 and weight.dtype == torch.bfloat16, "inputs/weight must be bfloat16")
    _need(inputs.is_cuda and weight.is_cuda and inputs.is_contiguous() and weight.is_contiguous(), "layout")
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (inputs.shape[0],), "targets: contiguous CUDA int64 [N]")
    _need(n_valid_total.dtype == torch.int64 and n_valid_total.numel() == 1 and n_valid_total.is_cuda,
          "n_valid_total: CUDA int64 scalar")
    _need(reduction in GH_REDUCTION and accum in GH_ACCUM, "reduction / accum")
    N, D = inputs.shape
    V = weight.shape[0]
    if grad_inputs is None:
        grad_inputs = torch.empty_like(inputs)
    if grad_weight is None:
        grad_weight = torch.empty_like(weight)
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=inputs.device)
    st = lib().gh_linear_ce_shard(_ptr(inputs), _ptr(weight), _ptr(targets), N, D, V, int(chunk), GH_ACCUM[accum],
                                  int(ignore_index), GH_REDUCTION[reduction], float(z_loss), _ptr(n_valid_total),
                                  _ptr(loss), _ptr(grad_inputs), _ptr(grad_weight), _stream_handle(stream))
    _check(st, "gh_linear_ce_shard")
    return loss, grad_inputs, grad_weight


def gh_linear_ce_shard_f32(inputs, weight, targets, n_valid_total, ignore_index: int = -100,
                           reduction: str = "mean", z_loss: float = 0.0, chunk: int = 0, *, grad_inputs=None,
                           grad_weight_f32=None, loss=None, stream=None, on_slice=None, dw_slices: int = 1,
                           max_sms: int = 0):
    """``gh_linear_ce_shard`` with fp32 accumulation whose weight gradient comes
    back as the shard's unrounded fp32 sum (float32 [V, D]), for an fp32
    cross-rank sum followed by one rounding (``gh_cast_f32_to_bf16``).

    With ``on_slice`` (``gh_linear_ce_shard_f32_sliced``) the last chunk's
    weight-gradient launch is cut into ``dw_slices`` ranges of weight rows on
    at most ``max_sms`` SMs (0: all), and ``on_slice(v0, v1)`` is called, with
    the library's stream current, after each range is enqueued: rows v0..v1-1
    of the fp32 gradient are final behind the work enqueued so far."""
    import torch
    _need(inputs.dim() == 2 and weight.dim() == 2 and inputs.shape[1] == weight.shape[1], "shapes")
    _need(inputs.dtype == torch.bfloat16 and weight.dtype == torch.bfloat16, "inputs/weight must be bfloat16")
    _need(inputs.is_cuda and weight.is_cuda and inputs.is_contiguous() and weight.is_contiguous(), "layout")
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (inputs.shape[0],), "targets: contiguous CUDA int64 [N]")
    _need(n_valid_total.dtype == torch.int64 and n_valid_total.numel() == 1 and n_valid_total.is_cuda,
          "n_valid_total: CUDA int64 scalar")
    _need(reduction in GH_REDUCTION, "reduction")
    N, D = inputs.shape
    V = weight.shape[0]
    if grad_inputs is None:
        grad_inputs = torch.empty_like(inputs)
    if grad_weight_f32 is None:
        grad_weight_f32 = torch.empty((V, D), dtype=torch.float32, device=weight.device)
    _need(grad_weight_f32.dtype == torch.float32 and grad_weight_f32.shape == (V, D)
          and grad_weight_f32.is_contiguous(), "grad_weight_f32: contiguous float32 [V, D]")
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=inputs.device)
    args = (_ptr(inputs), _ptr(weight), _ptr(targets), N, D, V, int(chunk), int(ignore_index),
            GH_REDUCTION[reduction], float(z_loss), _ptr(n_valid_total), _ptr(loss), _ptr(grad_inputs),
            _ptr(grad_weight_f32))
    if on_slice is None:
        st = lib().gh_linear_ce_shard_f32(*args, _stream_handle(stream))
        _check(st, "gh_linear_ce_shard_f32")
        return loss, grad_inputs, grad_weight_f32
    _need(int(dw_slices) >= 1, "dw_slices >= 1")
    dev = inputs.device
    errors = []

    def callback(ctx, v0, v1, stream_ptr):
        try:
            strm = (torch.cuda.ExternalStream(stream_ptr, device=dev) if stream_ptr
                    else torch.cuda.default_stream(dev))
            with torch.cuda.stream(strm):
                on_slice(int(v0), int(v1))
            return GH_OK
        except BaseException as e:  # reported after the call returns
            errors.append(e)
            return GH_ERR_INVALID_ARG

    fn = DW_SLICE_FN(callback)
    st = lib().gh_linear_ce_shard_f32_sliced(*args, int(dw_slices), int(max_sms), fn, None,
                                             _stream_handle(stream))
    if errors:
        raise errors[0]
    _check(st, "gh_linear_ce_shard_f32_sliced")
    return loss, grad_inputs, grad_weight_f32


def gh_cast_f32_to_bf16(src, out=None, stream=None):
    """bf16 copy of a float32 CUDA tensor, rounded to nearest even by the library."""
    import torch
    _need(src.dtype == torch.float32 and src.is_cuda and src.is_contiguous(), "src: contiguous CUDA float32")
    if out is None:
        out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    _need(out.dtype == torch.bfloat16 and out.numel() == src.numel() and out.is_contiguous(), "out")
    _check(lib().gh_cast_f32_to_bf16(_ptr(src), _ptr(out), src.numel(), _stream_handle(stream)),
           "gh_cast_f32_to_bf16")
    return out


def gh_ce_fwd(logits, targets, ignore_index: int = -100, reduction: str = "mean", z_loss: float = 0.0, *,
              loss=None, row_loss=None, stream=None):
    """Cross-entropy loss without the gradient (one call into ``gh_ce_fwd``).

    ``logits`` CUDA [B, V] float32 or bfloat16, ``targets`` CUDA int64 [B].
    ``row_loss`` (optional float32 [B] output) receives each row's loss
    (0 for ignored rows), the unreduced form.  Returns ``(loss, row_loss)``;
    ``row_loss`` is None unless it was given.
    """
    import torch
    _need(logits.dim() == 2 and logits.is_cuda and logits.is_contiguous(), "logits: contiguous CUDA [B, V]")
    _need(logits.dtype in (torch.float32, torch.bfloat16), "logits dtype must be float32 or bfloat16")
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (logits.shape[0],), "targets: contiguous CUDA int64 [B]")
    _need(reduction in GH_REDUCTION, "reduction must be 'mean' or 'sum'")
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=logits.device)
    _need(loss.dtype == torch.float32 and loss.numel() == 1, "loss must be a float32 scalar")
    if row_loss is not None:
        _need(row_loss.dtype == torch.float32 and row_loss.is_cuda and row_loss.is_contiguous()
              and row_loss.shape == (logits.shape[0],), "row_loss: contiguous CUDA float32 [B]")
    B, V = logits.shape
    dtype = GH_F32 if logits.dtype == torch.float32 else GH_BF16
    st = lib().gh_ce_fwd(_ptr(logits), _ptr(targets), B, V, dtype, int(ignore_index), GH_REDUCTION[reduction],
                         float(z_loss), _ptr(loss), _ptr(row_loss), _stream_handle(stream))
    _check(st, "gh_ce_fwd")
    return loss, row_loss


class _DeviceView:
    """A CUDA array interface over memory the library owns during a callback."""

    def __init__(self, ptr, shape, strides, typestr):
        self.__cuda_array_interface__ = {"version": 3, "data": (ptr, False), "shape": tuple(shape),
                                         "strides": tuple(strides), "typestr": typestr, "stream": None}


def gh_chunked_linear_loss(inputs, weight, loss_and_grad_fn, *loss_args, chunk: int = 0, accum: str = "fp32",
                           grad_inputs=None, grad_weight=None, loss=None, stream=None, **loss_kwargs):
    """Chunked linear projection with a caller-provided loss (``gh_chunked_linear_loss``).

    For each row chunk the library computes ``logits = inputs[c] @ weight.T``
    (bf16) and this wrapper calls ``loss_and_grad_fn(logits_chunk, *args,
    **kwargs)`` on the library's stream; tensor arguments whose leading
    dimension is N are sliced to the chunk's rows.  The function returns
    ``(loss, grad_logits)``: a scalar and a tensor shaped like the chunk.  The
    gradient is written over the chunk logits, the loss added to the total.
    Returns ``(loss, grad_inputs, grad_weight)``; the loss is the sum over chunks.
    """
    import torch
    _need(inputs.dim() == 2 and weight.dim() == 2 and inputs.shape[1] == weight.shape[1], "shapes")
    _need(inputs.dtype == torch.bfloat16 and weight.dtype == torch.bfloat16, "inputs/weight must be bfloat16")
    _need(inputs.is_cuda and weight.is_cuda and inputs.is_contiguous() and weight.is_contiguous(), "layout")
    _need(accum in GH_ACCUM, "accum must be 'fp32' or 'weight'")
    N, D = inputs.shape
    V = weight.shape[0]
    dev = inputs.device
    if grad_inputs is None:
        grad_inputs = torch.empty_like(inputs)
    if grad_weight is None:
        grad_weight = torch.empty_like(weight)
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=dev)
    _need(loss.dtype == torch.float32 and loss.numel() == 1, "loss must be a float32 scalar")
    errors = []

    def cut(v, r0, n):
        return v[r0:r0 + n] if isinstance(v, torch.Tensor) and v.dim() >= 1 and v.shape[0] == N else v

    def callback(ctx, row0, rows, logits_ptr, ld, v, loss_ptr, stream_ptr):
        try:
            strm = (torch.cuda.ExternalStream(stream_ptr, device=dev) if stream_ptr
                    else torch.cuda.default_stream(dev))
            with torch.cuda.stream(strm):
                logits = torch.as_tensor(_DeviceView(logits_ptr, (rows, v), (ld * 2, 2), "<i2"),
                                         device=dev).view(torch.bfloat16)
                acc = torch.as_tensor(_DeviceView(loss_ptr, (1,), (4,), "<f4"), device=dev)
                args = [cut(a, row0, rows) for a in loss_args]
                kwargs = {k: cut(a, row0, rows) for k, a in loss_kwargs.items()}
                chunk_loss, grad_logits = loss_and_grad_fn(logits, *args, **kwargs)
                if tuple(grad_logits.shape) != (rows, v):
                    raise ValueError(f"grad_logits shape {tuple(grad_logits.shape)} != {(rows, v)}")
                logits.copy_(grad_logits)
                acc.add_(torch.as_tensor(chunk_loss, device=dev).reshape(1).to(torch.float32))
            return GH_OK
        except BaseException as e:  # reported after the call returns
            errors.append(e)
            return GH_ERR_INVALID_ARG

    fn = CHUNK_LOSS_FN(callback)
    st = lib().gh_chunked_linear_loss(_ptr(inputs), _ptr(weight), N, D, V, int(chunk), GH_ACCUM[accum], fn, None,
                                      _ptr(loss), _ptr(grad_inputs), _ptr(grad_weight), _stream_handle(stream))
    if errors:
        raise errors[0]
    _check(st, "gh_chunked_linear_loss")
    return loss, grad_inputs, grad_weight


def gh_ce_vjp(logits, targets, row_loss, g, ignore_index: int = -100, *, grad=None, stream=None):
    """Logits gradient of the per-row cross-entropy for upstream gradients ``g``
    (one call into ``gh_ce_vjp``): ``grad[r] = g[r] * (softmax(logits[r]) - onehot(targets[r]))``.

    ``row_loss`` is the forward's z-free row loss ``lse - x_t`` (``gh_ce_fwd``
    with ``z_loss=0``), ``g`` float32 [B]; both CUDA.  ``grad`` (optional
    output, may be ``logits`` itself) is allocated when not given.  Returns ``grad``.
    """
    import torch
    _need(logits.dim() == 2 and logits.is_cuda and logits.is_contiguous(), "logits: contiguous CUDA [B, V]")
    _need(logits.dtype in (torch.float32, torch.bfloat16), "logits dtype must be float32 or bfloat16")
    B, V = logits.shape
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (B,), "targets: contiguous CUDA int64 [B]")
    for name, v in (("row_loss", row_loss), ("g", g)):
        _need(v.dtype == torch.float32 and v.is_cuda and v.is_contiguous() and v.shape == (B,),
              f"{name}: contiguous CUDA float32 [B]")
    if grad is None:
        grad = torch.empty_like(logits)
    _need(grad.shape == logits.shape and grad.dtype == logits.dtype and grad.is_contiguous(), "grad mismatch")
    dtype = GH_F32 if logits.dtype == torch.float32 else GH_BF16
    st = lib().gh_ce_vjp(_ptr(logits), _ptr(targets), B, V, dtype, int(ignore_index), _ptr(row_loss), _ptr(g),
                         _ptr(grad), _stream_handle(stream))
    _check(st, "gh_ce_vjp")
    return grad


def gh_selective_log_softmax(logits, index, *, out=None, stream=None):
    """``log_softmax(logits)[..., index]`` per row without the full log-probabilities
    (one call into ``gh_selective_log_softmax``).

    ``logits`` CUDA [..., V] float32 or bfloat16, contiguous; ``index`` CUDA
    int64 [...] (the leading shape of ``logits``).  Returns float32 [...]; an
    index outside [0, V) gives NaN in its row and sets GH_ERR_TARGET_RANGE in
    the device status.
    """
    import torch
    _need(logits.dim() >= 1 and logits.is_cuda and logits.is_contiguous(), "logits: contiguous CUDA [..., V]")
    _need(logits.dtype in (torch.float32, torch.bfloat16), "logits dtype must be float32 or bfloat16")
    _need(index.dtype == torch.int64 and index.is_cuda and index.is_contiguous()
          and tuple(index.shape) == tuple(logits.shape[:-1]), "index: contiguous CUDA int64 [...]")
    if out is None:
        out = torch.empty(index.shape, dtype=torch.float32, device=logits.device)
    _need(out.dtype == torch.float32 and out.is_contiguous() and tuple(out.shape) == tuple(index.shape),
          "out: contiguous float32 [...]")
    V = logits.shape[-1]
    rows = index.numel()
    dtype = GH_F32 if logits.dtype == torch.float32 else GH_BF16
    st = lib().gh_selective_log_softmax(_ptr(logits), _ptr(index), rows, V, dtype, _ptr(out),
                                        _stream_handle(stream))
    _check(st, "gh_selective_log_softmax")
    return out


def gh_linear_ce(inputs, weight, targets, ignore_index: int = -100, reduction: str = "mean",
                 z_loss: float = 0.0, chunk: int = 0, accum: str = "fp32", *, grad_inputs=None,
                 grad_weight=None, loss=None, stream=None):
    """Chunked linear cross-entropy (one call into ``gh_linear_ce``).

    ``inputs`` bf16 [N, D], ``weight`` bf16 [V, D], ``targets`` int64 [N], all
    contiguous CUDA tensors.  ``chunk`` rows per logits chunk (<= 0: default),
    ``accum`` "fp32" or "weight".  Returns ``(loss, grad_inputs, grad_weight)``.
    """
    import torch
    _need(inputs.dim() == 2 and weight.dim() == 2 and inputs.shape[1] == weight.shape[1], "shapes")
    _need(inputs.dtype == torch.bfloat16 and weight.dtype == torch.bfloat16, "inputs/weight must be bfloat16")
    _need(inputs.is_cuda and weight.is_cuda and inputs.is_contiguous() and weight.is_contiguous(), "layout")
    _need(targets.dtype == torch.int64 and targets.is_cuda and targets.is_contiguous()
          and targets.shape == (inputs.shape[0],), "targets: contiguous CUDA int64 [N]")
    _need(reduction in GH_REDUCTION and accum in GH_ACCUM, "reduction / accum")
    if grad_inputs is None:
        grad_inputs = torch.empty_like(inputs)
    if grad_weight is None:
        grad_weight = torch.empty_like(weight)
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=inputs.device)
    N, D = inputs.shape
    V = weight.shape[0]
    st = lib().gh_linear_ce(_ptr(inputs), _ptr(weight), _ptr(targets), N, D, V, int(chunk), GH_ACCUM[accum],
                            int(ignore_index), GH_REDUCTION[reduction], float(z_loss), _ptr(loss),
                            _ptr(grad_inputs), _ptr(grad_weight), _stream_handle(stream))
    _check(st, "gh_linear_ce")
    return loss, grad_inputs, grad_weight


GH_KERNEL = {"ce_row": 0, "logits_gemm": 1, "chunk_ce": 2, "dx_gemm": 3, "dw_gemm": 4, "ce_vjp": 5}


def gh_profile_enable(enable: bool = True) -> None:
    """Start (discarding earlier records) or stop recording per-kernel CUDA events."""
    _check(lib().gh_profile_enable(1 if enable else 0), "gh_profile_enable")


GH_DEBUG = {"wait_limit_ns": 0, "withhold_ring_piece": 1, "withhold_gemm_stage": 2}


def gh_debug_set(knob: str, value: int) -> None:
    """Failure-path test knobs (off by default): the device wait limit in ns
    (``wait_limit_ns``; <= 0 restores the default), or one copy the next ring
    or GEMM launch leaves out (``withhold_ring_piece``, ``withhold_gemm_stage``;
    -1 none)."""
    _check(lib().gh_debug_set(GH_DEBUG[knob], int(value)), "gh_debug_set")


def gh_exp2_eval(y, method: str, out=None, stream=None):
    """2^y of a float32 CUDA tensor by one of the kernels' two routes:
    ``"mufu"`` (ex2.approx) or ``"fma"`` (the FMA-pipe polynomial, y <= 0)."""
    import torch
    _need(y.dtype == torch.float32 and y.is_cuda and y.is_contiguous(), "y: contiguous CUDA float32")
    if out is None:
        out = torch.empty_like(y)
    _need(out.dtype == torch.float32 and out.numel() == y.numel() and out.is_contiguous(), "out")
    m = {"mufu": 0, "fma": 1}[method]
    _check(lib().gh_exp2_eval(_ptr(y), _ptr(out), y.numel(), m, _stream_handle(stream)), "gh_exp2_eval")
    return out


def gh_profile_read(kind: str):
    """(summed milliseconds, launches) recorded for one kernel kind."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int64(0)
    _check(lib().gh_profile_read(GH_KERNEL[kind], ctypes.byref(ms), ctypes.byref(n)), "gh_profile_read")
    return ms.value, n.value


def gh_launch_count() -> int:
    """Kernels launched by libgh in this process so far."""
    return int(lib().gh_launch_count())


def gh_get_device_status(stream=None) -> int:
    """Synchronise ``stream``; return and clear the device status word."""
    return int(lib().gh_get_device_status(_stream_handle(stream)))


__all__ = [
    "GhError", "lib", "header_symbols", "status_string", "gh_status_string", "gh_version",
    "gh_ce_fwd_bwd", "gh_ce_fwd_bwd_noalloc", "GH_NOALLOC_MAX_ROWS", "gh_ce_fwd", "gh_selective_log_softmax",
    "gh_ce_vjp", "gh_linear_ce", "gh_chunked_linear_loss", "CHUNK_LOSS_FN",
    "gh_count_valid", "gh_ce_fwd_bwd_shard", "gh_linear_ce_shard", "gh_linear_ce_shard_f32",
    "gh_cast_f32_to_bf16", "gh_exp2_eval",
    "gh_get_device_status", "gh_profile_enable", "gh_profile_read", "gh_debug_set", "GH_DEBUG",
    "gh_launch_count", "GH_KERNEL",
    "GH_OK", "GH_ERR_INVALID_ARG", "GH_ERR_UNSUPPORTED", "GH_ERR_ALLOC", "GH_ERR_CUDA",
    "GH_ERR_TIMEOUT", "GH_ERR_TARGET_RANGE", "GH_REDUCTION", "GH_ACCUM", "GH_F32", "GH_BF16",
]
