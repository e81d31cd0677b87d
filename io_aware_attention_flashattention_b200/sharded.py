"""Head-sharded attention over several GPUs (no collective on the data path).

Every (batch, head) of exact attention is an independent problem in both passes, so
one [B, H, N, d] call splits into contiguous ranges of the flattened B*H heads. In
the contiguous [B, H, N, d] layout a head range is one contiguous block of memory,
so a shard is a plain slice: it is copied to its GPU, the library's kernels run
there on that GPU's current stream, and the results are copied back into the
caller's output tensors. Nothing is exchanged between the shards; the copies are
the only traffic.

Two forms:
  * one process, several devices: ``forward_sharded`` / ``backward_sharded`` /
    ``attention_sharded`` take the whole problem on one device and a device list;
  * one process per GPU (torch.distributed): ``rank_heads`` gives each rank its
    head range, each rank runs the plain entry points on its slice, and
    ``gather_heads`` assembles the full output on every rank when the caller wants
    it (an all-gather of outputs, outside the attention computation itself).

Dropout: the keep mask is keyed by the head index, so each shard passes its first
flattened head as head_base (fa_forward_dropout_heads) and draws exactly the masks
the unsharded call draws for its heads.
"""
from __future__ import annotations

import torch

from . import api


def shard_ranges(total: int, parts: int):
    """Split ``range(total)`` into ``parts`` contiguous ranges whose sizes differ by at
    most one (the first ``total % parts`` ranges get the extra item). Returns a list of
    (start, stop); ranges are empty when parts > total."""
    if parts < 1:
        raise ValueError("parts must be >= 1")
    if total < 0:
        raise ValueError("total must be >= 0")
    base, extra = divmod(total, parts)
    out, start = [], 0
    for i in range(parts):
        stop = start + base + (1 if i < extra else 0)
        out.append((start, stop))
        start = stop
    return out


def rank_heads(B: int, H: int, rank: int, world: int):
    """The (start, stop) range of flattened B*H heads that ``rank`` of ``world`` owns."""
    if not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    return shard_ranges(B * H, world)[rank]


def _flat(t: torch.Tensor) -> torch.Tensor:
    """[B, H, N, d] (or [B, H, N]) as [B*H, ...], a view of the contiguous tensor."""
    if not t.is_contiguous():
        raise ValueError("sharded calls take contiguous tensors")
    return t.reshape(t.shape[0] * t.shape[1], *t.shape[2:])


def _devices(devices):
    devs = [torch.device(d) for d in devices]
    if not devs or any(d.type != "cuda" for d in devs):
        raise ValueError("devices must be a non-empty list of CUDA devices")
    return devs


def _piece(t: torch.Tensor, a: int, b: int, dev: torch.device) -> torch.Tensor:
    """Heads [a, b) of a flattened tensor on ``dev`` as a [1, b - a, ...] tensor."""
    return _flat(t)[a:b].to(dev, non_blocking=True).unsqueeze(0)


def _mask_on(block_mask, dev):
    return None if block_mask is None else block_mask.to(dev, non_blocking=True)


def _shard_dropout(dropout, a: int):
    """The dropout tuple for the shard whose first flattened head is ``a``."""
    if dropout is None:
        return None
    p, seed, offset, *rest = dropout
    return (p, seed, offset, (int(rest[0]) if rest else 0) + a)


def forward_sharded(q, k, v, devices, causal: bool = False, scale=None, window=None,
                    block_mask=None, dropout=None):
    """(O, LSE) of the whole problem, computed in head shards on ``devices`` (a list of
    CUDA devices; one may appear more than once). Inputs and outputs live on q's
    device; each shard's inputs are copied to its GPU and its outputs copied back.
    ``dropout`` = (p, seed, offset) as for api.forward draws the unsharded call's
    masks."""
    devs = _devices(devices)
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    for (a, b), dev in zip(shard_ranges(B * H, len(devs)), devs):
        if a == b:
            continue
        with torch.cuda.device(dev):
            qs, ks, vs = (_piece(t, a, b, dev) for t in (q, k, v))
            os_, ls = api.forward(qs, ks, vs, causal, scale, window, _mask_on(block_mask, dev),
                                  _shard_dropout(dropout, a))
            _flat(o)[a:b].copy_(os_[0], non_blocking=True)
            _flat(lse)[a:b].copy_(ls[0], non_blocking=True)
    return o, lse


def backward_sharded(q, k, v, o, lse, do, devices, causal: bool = False, scale=None,
                     window=None, block_mask=None, dropout=None):
    """(dQ, dK, dV) of the loss <dO, O>, computed in head shards on ``devices``, with
    the same masks and dropout as the forward. Each shard's backward workspace is
    allocated on its own GPU."""
    devs = _devices(devices)
    B, H, N, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for (a, b), dev in zip(shard_ranges(B * H, len(devs)), devs):
        if a == b:
            continue
        with torch.cuda.device(dev):
            qs, ks, vs, os_, dos = (_piece(t, a, b, dev) for t in (q, k, v, o, do))
            ls = _piece(lse, a, b, dev)
            g = api.backward(qs, ks, vs, os_, ls, dos, causal, scale, None, window,
                             _mask_on(block_mask, dev), _shard_dropout(dropout, a))
            for dst, src in zip((dq, dk, dv), g):
                _flat(dst)[a:b].copy_(src[0], non_blocking=True)
    return dq, dk, dv


class ShardedAttentionFunction(torch.autograd.Function):
    """Differentiable head-sharded attention."""

    @staticmethod
    def forward(ctx, q, k, v, devices, causal=False, scale=None, window=None, block_mask=None,
                dropout=None):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse = forward_sharded(q, k, v, devices, causal, scale, window, block_mask, dropout)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.args = (devices, causal, scale, window, block_mask, dropout)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        devices, causal, scale, window, block_mask, dropout = ctx.args
        dq, dk, dv = backward_sharded(q, k, v, o, lse, do.contiguous(), devices, causal, scale,
                                      window, block_mask, dropout)
        return dq, dk, dv, None, None, None, None, None, None


def attention_sharded(q, k, v, devices, causal: bool = False, scale=None, window=None,
                      block_mask=None, dropout=None):
    """Differentiable attention whose heads are computed on ``devices``."""
    return ShardedAttentionFunction.apply(q, k, v, devices, causal, scale, window, block_mask,
                                          dropout)


def gather_heads(local: torch.Tensor, B: int, H: int, group=None) -> torch.Tensor:
    """All ranks' head ranges of one output assembled on every rank.

    ``local`` holds this rank's heads (rank_heads order) as [n_local, ...]. Ranges
    differ in length by at most one head, so every rank pads its piece to the longest
    range for one all_gather and the padding is dropped afterwards. Returns the full
    [B, H, ...] tensor."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    ranges = shard_ranges(B * H, world)
    longest = max(b - a for a, b in ranges)
    rest = tuple(local.shape[1:])
    pad = torch.zeros((longest, *rest), dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    pieces = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(pieces, pad, group=group)
    full = torch.cat([p[: b - a] for p, (a, b) in zip(pieces, ranges)], dim=0)
    return full.reshape(B, H, *rest)
