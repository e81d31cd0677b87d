"""Python binding of the C ABI in include/fa.h (argument marshalling only).

The ``fa_*`` functions mirror the C entry points one to one: they take torch
tensors that already live on the GPU, check dtype/shape/contiguity, and pass raw
pointers, sizes and the current CUDA stream to libfa_b200.so. Every arithmetic
step runs in the library's kernels; there is no CPU or PyTorch fallback.

``forward``, ``backward`` and ``attention`` are conveniences on top: they allocate
outputs (and the backward workspace) with torch and call the entry points;
``attention`` is differentiable through ``FlashAttentionFunction``.

Operation (see include/fa.h): O = softmax(scale * Q K^T [causal mask]) V and
LSE = natural-log log-sum-exp per query row, for [B, H, N, d] tensors, d in
{64, 128}; backward gives dQ, dK, dV of the loss <dO, O>.
"""
from __future__ import annotations

import contextlib
import functools
import math

import torch

from ._lib import FAError, check, lib

__all__ = [
    "FAError", "fa_forward", "fa_backward", "fa_backward_workspace_size",
    "fa_backward_preprocess", "fa_backward_main", "fa_backward_dq_convert",
    "fa_backward_noalloc", "fa_forward_f16", "fa_backward_f16", "fa_forward_masked",
    "fa_backward_masked", "fa_forward_dropout", "fa_backward_dropout", "fa_forward_f32",
    "fa_backward_f32", "fa_get_status", "fa_watchdog_selftest", "fa_version", "fa_dropout_rate",
    "fa_launch_plan",
    "forward", "backward", "attention", "FlashAttentionFunction",
]


def _one_device(*args):
    """A context that makes current the one CUDA device of a call's tensors (and
    stream): the library launches on the current device, and a stream left as None
    is that device's current stream. Arguments on two different GPUs raise."""
    devs = set()
    for a in args:
        dev = getattr(a, "device", None)
        if isinstance(dev, torch.device) and dev.type == "cuda" and dev.index is not None:
            devs.add(dev)
    if len(devs) > 1:
        raise ValueError("the tensors of one call must be on one GPU, got "
                         + ", ".join(sorted(str(x) for x in devs)))
    return torch.cuda.device(devs.pop()) if devs else contextlib.nullcontext()


def _on_one_device(fn):
    @functools.wraps(fn)
    def call(*args, **kwargs):
        with _one_device(*args, *kwargs.values()):
            return fn(*args, **kwargs)
    return call


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return int(getattr(stream, "cuda_stream", stream))


def _shape(t: torch.Tensor):
    if t.dim() != 4:
        raise ValueError(f"expected a [B, H, N, d] tensor, got shape {tuple(t.shape)}")
    return tuple(int(x) for x in t.shape)


def _need(name: str, t: torch.Tensor, dtype: torch.dtype, shape) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def fa_version() -> str:
    return lib().fa_version().decode()


def fa_backward_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib().fa_backward_workspace_size(B, H, N, d))


@_on_one_device
def fa_forward(Q, K, V, O, LSE, scale: float, causal: bool, stream=None) -> None:
    B, H, N, d = _shape(Q)
    bf = torch.bfloat16
    args = [_need("Q", Q, bf, (B, H, N, d)), _need("K", K, bf, (B, H, N, d)),
            _need("V", V, bf, (B, H, N, d)), _need("O", O, bf, (B, H, N, d)),
            _need("LSE", LSE, torch.float32, (B, H, N))]
    check("fa_forward", lib().fa_forward(*args, B, H, N, d, float(scale), int(bool(causal)),
                                         _stream(stream)))


@_on_one_device
def fa_forward_f16(Q, K, V, O, LSE, scale: float, causal: bool, stream=None) -> None:
    B, H, N, d = _shape(Q)
    h = torch.float16
    args = [_need("Q", Q, h, (B, H, N, d)), _need("K", K, h, (B, H, N, d)),
            _need("V", V, h, (B, H, N, d)), _need("O", O, h, (B, H, N, d)),
            _need("LSE", LSE, torch.float32, (B, H, N))]
    check("fa_forward_f16", lib().fa_forward_f16(*args, B, H, N, d, float(scale),
                                                 int(bool(causal)), _stream(stream)))


def _block_mask(block_mask, N: int):
    """Device pointer of a [ceil(N/128)]^2 uint8/bool CUDA tensor, or None."""
    if block_mask is None:
        return None
    T = (N + 127) // 128
    if not isinstance(block_mask, torch.Tensor) or not block_mask.is_cuda:
        raise ValueError("block_mask must be a CUDA tensor")
    if block_mask.dtype not in (torch.uint8, torch.bool):
        raise TypeError("block_mask must be uint8 or bool")
    if tuple(block_mask.shape) != (T, T) or not block_mask.is_contiguous():
        raise ValueError(f"block_mask must be a contiguous [{T}, {T}] tensor")
    return block_mask.data_ptr()


def _window(window):
    if window is None:
        return -1, -1
    left, right = window
    return int(left), int(right)


@_on_one_device
def fa_forward_masked(Q, K, V, O, LSE, scale: float, causal: bool, window=None,
                      block_mask=None, stream=None) -> None:
    """fa_forward with a sliding window (left, right) (negative = unbounded side)
    and/or a 128 x 128 block mask, both ANDed with causal."""
    B, H, N, d = _shape(Q)
    bf = torch.bfloat16
    args = [_need("Q", Q, bf, (B, H, N, d)), _need("K", K, bf, (B, H, N, d)),
            _need("V", V, bf, (B, H, N, d)), _need("O", O, bf, (B, H, N, d)),
            _need("LSE", LSE, torch.float32, (B, H, N))]
    wl, wr = _window(window)
    check("fa_forward_masked", lib().fa_forward_masked(
        *args, B, H, N, d, float(scale), int(bool(causal)), wl, wr, _block_mask(block_mask, N),
        _stream(stream)))


@_on_one_device
def fa_backward_masked(Q, K, V, O, dO, LSE, dQ, dK, dV, scale: float, causal: bool, workspace,
                       window=None, block_mask=None, stream=None) -> None:
    ptrs, (B, H, N, d), ws, nbytes = _bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace,
                                               torch.bfloat16)
    wl, wr = _window(window)
    check("fa_backward_masked", lib().fa_backward_masked(
        *ptrs, B, H, N, d, float(scale), int(bool(causal)), wl, wr, _block_mask(block_mask, N),
        ws, nbytes, _stream(stream)))


def fa_launch_plan(B: int, H: int, N: int, d: int, causal: bool = False) -> dict:
    """How a plain call of this shape is distributed on the current GPU (launches
    nothing): ``fwd_persistent`` / ``bwd_persistent`` (persistent kernels, CTAs walking
    a list of tiles) and ``bwd_split`` (key tiles run as two CTAs)."""
    import ctypes
    fp, bp, bs = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    check("fa_launch_plan", lib().fa_launch_plan(B, H, N, d, int(causal), ctypes.addressof(fp),
                                                 ctypes.addressof(bp), ctypes.addressof(bs)))
    return {"fwd_persistent": bool(fp.value), "bwd_persistent": bool(bp.value),
            "bwd_split": bs.value}


def fa_dropout_rate(p: float) -> float:
    """The drop probability the dropout calls apply for ``p``: p rounded down to a
    multiple of 1/256. Raises ValueError for a rate they refuse (outside [0, 1), or
    in (0, 1/256), which would round down to no dropout)."""
    r = float(lib().fa_dropout_rate(float(p)))
    if r < 0:
        raise ValueError(f"dropout rate {p} is outside [0, 1) or below 1/256")
    return r


def _dropout(dropout):
    """(p, seed, offset, head_base) from dropout = (p, seed, offset) or (p, seed, offset,
    head_base); head_base (default 0) as for fa_forward_dropout_heads."""
    if dropout is None:
        return 0.0, 0, 0, 0
    p, seed, offset, *rest = dropout
    if len(rest) > 1:
        raise ValueError("dropout is (p, seed, offset) or (p, seed, offset, head_base)")
    head_base = int(rest[0]) if rest else 0
    return float(p), int(seed) & ((1 << 64) - 1), int(offset) & 0xFFFFFFFF, head_base


@_on_one_device
def fa_forward_dropout(Q, K, V, O, LSE, scale: float, causal: bool, dropout, window=None,
                       block_mask=None, stream=None) -> None:
    """fa_forward_masked with dropout=(p, seed, offset) on P (Philox-4x32-10 mask, one
    byte per element; the drop rate is p rounded down to a multiple of 1/256). A fourth
    element, head_base, draws the masks of heads head_base + b*H + h of a larger
    problem (fa_forward_dropout_heads)."""
    B, H, N, d = _shape(Q)
    bf = torch.bfloat16
    args = [_need("Q", Q, bf, (B, H, N, d)), _need("K", K, bf, (B, H, N, d)),
            _need("V", V, bf, (B, H, N, d)), _need("O", O, bf, (B, H, N, d)),
            _need("LSE", LSE, torch.float32, (B, H, N))]
    wl, wr = _window(window)
    p, seed, offset, head_base = _dropout(dropout)
    common = (*args, B, H, N, d, float(scale), int(bool(causal)), wl, wr,
              _block_mask(block_mask, N), p, seed, offset)
    if head_base:
        check("fa_forward_dropout_heads",
              lib().fa_forward_dropout_heads(*common, head_base, _stream(stream)))
    else:
        check("fa_forward_dropout", lib().fa_forward_dropout(*common, _stream(stream)))


@_on_one_device
def fa_backward_dropout(Q, K, V, O, dO, LSE, dQ, dK, dV, scale: float, causal: bool, workspace,
                        dropout, window=None, block_mask=None, stream=None) -> None:
    ptrs, (B, H, N, d), ws, nbytes = _bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace,
                                               torch.bfloat16)
    wl, wr = _window(window)
    p, seed, offset, head_base = _dropout(dropout)
    common = (*ptrs, B, H, N, d, float(scale), int(bool(causal)), wl, wr,
              _block_mask(block_mask, N), p, seed, offset)
    if head_base:
        check("fa_backward_dropout_heads", lib().fa_backward_dropout_heads(
            *common, head_base, ws, nbytes, _stream(stream)))
    else:
        check("fa_backward_dropout", lib().fa_backward_dropout(
            *common, ws, nbytes, _stream(stream)))


@_on_one_device
def fa_forward_f32(Q, K, V, O, LSE, scale: float, causal: bool, stream=None) -> None:
    B, H, N, d = _shape(Q)
    f = torch.float32
    args = [_need("Q", Q, f, (B, H, N, d)), _need("K", K, f, (B, H, N, d)),
            _need("V", V, f, (B, H, N, d)), _need("O", O, f, (B, H, N, d)),
            _need("LSE", LSE, f, (B, H, N))]
    check("fa_forward_f32", lib().fa_forward_f32(*args, B, H, N, d, float(scale),
                                                 int(bool(causal)), _stream(stream)))


def _bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, dtype):
    B, H, N, d = _shape(Q)
    s4 = (B, H, N, d)
    ptrs = [_need("Q", Q, dtype, s4), _need("K", K, dtype, s4), _need("V", V, dtype, s4),
            _need("O", O, dtype, s4), _need("dO", dO, dtype, s4),
            _need("LSE", LSE, torch.float32, (B, H, N)),
            _need("dQ", dQ, dtype, s4), _need("dK", dK, dtype, s4), _need("dV", dV, dtype, s4)]
    if not (isinstance(workspace, torch.Tensor) and workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ptrs, (B, H, N, d), workspace.data_ptr(), workspace.numel() * workspace.element_size()


@_on_one_device
def fa_backward(Q, K, V, O, dO, LSE, dQ, dK, dV, scale: float, causal: bool, workspace,
                stream=None) -> None:
    ptrs, (B, H, N, d), ws, nbytes = _bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace,
                                               torch.bfloat16)
    check("fa_backward", lib().fa_backward(*ptrs, B, H, N, d, float(scale), int(bool(causal)),
                                           ws, nbytes, _stream(stream)))


def _ws(workspace):
    if not (isinstance(workspace, torch.Tensor) and workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


@_on_one_device
def fa_backward_preprocess(O, dO, LSE, scale: float, causal: bool, workspace, stream=None):
    B, H, N, d = _shape(O)
    bf = torch.bfloat16
    ws, nbytes = _ws(workspace)
    check("fa_backward_preprocess", lib().fa_backward_preprocess(
        _need("O", O, bf, (B, H, N, d)), _need("dO", dO, bf, (B, H, N, d)),
        _need("LSE", LSE, torch.float32, (B, H, N)), B, H, N, d, float(scale),
        int(bool(causal)), ws, nbytes, _stream(stream)))


@_on_one_device
def fa_backward_main(Q, K, V, dO, dK, dV, scale: float, causal: bool, workspace, stream=None):
    B, H, N, d = _shape(Q)
    s4, bf = (B, H, N, d), torch.bfloat16
    ws, nbytes = _ws(workspace)
    check("fa_backward_main", lib().fa_backward_main(
        _need("Q", Q, bf, s4), _need("K", K, bf, s4), _need("V", V, bf, s4),
        _need("dO", dO, bf, s4), _need("dK", dK, bf, s4), _need("dV", dV, bf, s4),
        B, H, N, d, float(scale), int(bool(causal)), ws, nbytes, _stream(stream)))


@_on_one_device
def fa_backward_dq_convert(dQ, scale: float, workspace, stream=None):
    B, H, N, d = _shape(dQ)
    ws, nbytes = _ws(workspace)
    check("fa_backward_dq_convert", lib().fa_backward_dq_convert(
        _need("dQ", dQ, torch.bfloat16, (B, H, N, d)), B, H, N, d, float(scale), ws, nbytes,
        _stream(stream)))


@_on_one_device
def fa_backward_noalloc(Q, K, V, O, dO, LSE, dQ, dK, dV, scale: float, causal: bool,
                        stream=None) -> None:
    """fa_backward for callers that cannot allocate device memory: the workspace
    is a fixed 32 MiB array inside the library (one per GPU). Shapes needing more
    raise FAError (FA_ERR_UNSUPPORTED). Calls on one GPU share the array, so they
    must not overlap: keep them on one stream. The first call on a GPU does a
    one-time look-up of the array's address; make it before any stream capture."""
    B, H, N, d = _shape(Q)
    s4, bf = (B, H, N, d), torch.bfloat16
    ptrs = [_need("Q", Q, bf, s4), _need("K", K, bf, s4), _need("V", V, bf, s4),
            _need("O", O, bf, s4), _need("dO", dO, bf, s4),
            _need("LSE", LSE, torch.float32, (B, H, N)),
            _need("dQ", dQ, bf, s4), _need("dK", dK, bf, s4), _need("dV", dV, bf, s4)]
    check("fa_backward_noalloc", lib().fa_backward_noalloc(
        *ptrs, B, H, N, d, float(scale), int(bool(causal)), _stream(stream)))


@_on_one_device
def fa_backward_f16(Q, K, V, O, dO, LSE, dQ, dK, dV, scale: float, causal: bool, workspace,
                    stream=None) -> None:
    ptrs, (B, H, N, d), ws, nbytes = _bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace,
                                               torch.float16)
    check("fa_backward_f16", lib().fa_backward_f16(*ptrs, B, H, N, d, float(scale),
                                                   int(bool(causal)), ws, nbytes,
                                                   _stream(stream)))


@_on_one_device
def fa_backward_f32(Q, K, V, O, dO, LSE, dQ, dK, dV, scale: float, causal: bool, workspace,
                    stream=None) -> None:
    ptrs, (B, H, N, d), ws, nbytes = _bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace,
                                               torch.float32)
    check("fa_backward_f32", lib().fa_backward_f32(*ptrs, B, H, N, d, float(scale),
                                                   int(bool(causal)), ws, nbytes,
                                                   _stream(stream)))


@_on_one_device
def fa_get_status(stream=None) -> int:
    """Synchronises the stream; returns the library status code (0 = ok, 4 = a
    kernel's bounded wait ran out since the last call)."""
    return int(lib().fa_get_status(_stream(stream)))


@_on_one_device
def fa_watchdog_selftest(timeout_ms: int, stream=None) -> None:
    check("fa_watchdog_selftest", lib().fa_watchdog_selftest(int(timeout_ms), _stream(stream)))


# ---------------------------------------------------------------- conveniences


def _default_scale(d: int, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _masked(window, block_mask) -> bool:
    return window is not None or block_mask is not None


def forward(q, k, v, causal: bool = False, scale=None, window=None, block_mask=None,
            dropout=None):
    """(O, LSE) for bf16, f16 or fp32 q, k, v of shape [B, H, N, d] on the GPU.
    ``window`` / ``block_mask`` as for fa_forward_masked and ``dropout`` = (p, seed,
    offset) as for fa_forward_dropout (bf16 only)."""
    B, H, N, d = _shape(q)
    scale = _default_scale(d, scale)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if dropout is not None:
        if q.dtype != torch.bfloat16:
            raise TypeError("dropout is supported for bf16 inputs")
        fa_forward_dropout(q, k, v, o, lse, scale, causal, dropout, window, block_mask)
    elif _masked(window, block_mask):
        if q.dtype != torch.bfloat16:
            raise TypeError("window and block_mask are supported for bf16 inputs")
        fa_forward_masked(q, k, v, o, lse, scale, causal, window, block_mask)
    elif q.dtype == torch.bfloat16:
        fa_forward(q, k, v, o, lse, scale, causal)
    elif q.dtype == torch.float16:
        fa_forward_f16(q, k, v, o, lse, scale, causal)
    elif q.dtype == torch.float32:
        fa_forward_f32(q, k, v, o, lse, scale, causal)
    else:
        raise TypeError(f"unsupported dtype {q.dtype}: bf16, f16 or fp32")
    return o, lse


def workspace_for(q) -> torch.Tensor:
    B, H, N, d = _shape(q)
    n = max(1, fa_backward_workspace_size(B, H, N, d))
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def backward(q, k, v, o, lse, do, causal: bool = False, scale=None, workspace=None,
             window=None, block_mask=None, dropout=None):
    """(dQ, dK, dV) of the loss <dO, O> (same masks and dropout as the forward)."""
    B, H, N, d = _shape(q)
    scale = _default_scale(d, scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = workspace_for(q) if workspace is None else workspace
    if dropout is not None:
        if q.dtype != torch.bfloat16:
            raise TypeError("dropout is supported for bf16 inputs")
        fa_backward_dropout(q, k, v, o, do, lse, dq, dk, dv, scale, causal, ws, dropout, window,
                            block_mask)
    elif _masked(window, block_mask):
        if q.dtype != torch.bfloat16:
            raise TypeError("window and block_mask are supported for bf16 inputs")
        fa_backward_masked(q, k, v, o, do, lse, dq, dk, dv, scale, causal, ws, window,
                           block_mask)
    elif q.dtype == torch.bfloat16:
        fa_backward(q, k, v, o, do, lse, dq, dk, dv, scale, causal, ws)
    elif q.dtype == torch.float16:
        fa_backward_f16(q, k, v, o, do, lse, dq, dk, dv, scale, causal, ws)
    elif q.dtype == torch.float32:
        fa_backward_f32(q, k, v, o, do, lse, dq, dk, dv, scale, causal, ws)
    else:
        raise TypeError(f"unsupported dtype {q.dtype}: bf16, f16 or fp32")
    return dq, dk, dv


class FlashAttentionFunction(torch.autograd.Function):
    """Differentiable exact attention through the library's forward and backward."""

    @staticmethod
    def forward(ctx, q, k, v, causal: bool = False, scale=None, window=None, block_mask=None,
                dropout=None):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse = forward(q, k, v, causal, scale, window, block_mask, dropout)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale, ctx.window, ctx.block_mask = causal, scale, window, block_mask
        ctx.dropout = dropout  # the backward regenerates the same keep mask
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = backward(q, k, v, o, lse, do.contiguous(), ctx.causal, ctx.scale,
                              window=ctx.window, block_mask=ctx.block_mask,
                              dropout=ctx.dropout)
        return dq, dk, dv, None, None, None, None, None


def attention(q, k, v, causal: bool = False, scale=None, window=None, block_mask=None,
              dropout=None):
    """Differentiable attention; ``dropout`` = (p, seed, offset): pass a new offset (or
    seed) per call to draw a new mask."""
    return FlashAttentionFunction.apply(q, k, v, causal, scale, window, block_mask, dropout)
