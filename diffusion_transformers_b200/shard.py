"""Head partition of one BinaryAttention forward across ranks (one process per GPU).

Every (b, h) of the attention is an independent problem: the scores, the
softmax and P.V of head h read only Q, K, V of head h and the bias plane
bias[h] ("BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
Transformers", §2 methodology, the learnable bias b_ij added before the
softmax; one [N, N] plane per head is this library's reading of its shape).
So one forward splits across g ranks with no exchange
step: rank r takes heads [h0, h1) = [r*H//g, (r+1)*H//g), holds only its
slices Q, K, V [B, h1-h0, N, d] and bias [h1-h0, N, N] (the dense bias, the
largest tensor of the call, is never replicated; a per-sample bias
[B, H, N, N] is sliced the same way on its head axis), and computes
O[:, h0:h1].
O stays sharded where the next layer consumes it; gather_heads() puts it back
together on every rank for callers that want it whole. The backward splits the
same way: a rank's dV, ds, dt and dbias are those of its heads.

Host logic only: the kernels see an ordinary call with H = h1 - h0.
"""
from __future__ import annotations

import numpy as np


def head_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of `rank` among `world` ranks: contiguous, sizes differ
    by at most one, every head on exactly one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if H < world:
        raise ValueError(f"{H} heads cannot be split over {world} ranks")
    return rank * H // world, (rank + 1) * H // world


def slice_heads(x, h0: int, h1: int, axis: int):
    """Contiguous copy of heads [h0, h1) of x along `axis` (numpy array or
    torch tensor; None stays None): Q, K, V and O carry heads on axis 1, the
    bias on axis 0."""
    if x is None:
        return None
    idx = [slice(None)] * x.ndim
    idx[axis] = slice(h0, h1)
    part = x[tuple(idx)]
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(part)
    return part.contiguous()


def shard_inputs(inp: dict, world: int, rank: int) -> dict:
    """This rank's part of a make_inputs() dictionary: Q, K, V sliced on the
    head axis, the bias on its head axis (the first of a shared [H, N, N]
    bias, the second of a per-sample [B, H, N, N] one), H replaced by the
    slice's size."""
    h0, h1 = head_range(inp["H"], world, rank)
    out = dict(inp)
    for key in ("q", "k", "v"):
        out[key] = slice_heads(inp[key], h0, h1, 1)
    bias = inp.get("bias")
    out["bias"] = slice_heads(bias, h0, h1, 1 if bias is not None and bias.ndim == 4 else 0)
    out["H"] = h1 - h0
    out["heads"] = (h0, h1)
    return out


def gather_heads(o_local, H: int, world: int, rank: int, group=None):
    """O [B, H, N, d] on every rank from each rank's O[:, h0:h1] (torch tensors,
    any torch.distributed backend). Slices of unequal size are padded to the
    largest for the all_gather and trimmed after it."""
    import torch
    import torch.distributed as dist

    h0, h1 = head_range(H, world, rank)
    if o_local.shape[1] != h1 - h0:
        raise ValueError(f"rank {rank} holds {o_local.shape[1]} heads, expected {h1 - h0}")
    hmax = max(head_range(H, world, r)[1] - head_range(H, world, r)[0] for r in range(world))
    pad = o_local.new_zeros((o_local.shape[0], hmax) + tuple(o_local.shape[2:]))
    pad[:, : h1 - h0] = o_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    pieces = []
    for r in range(world):
        a, b = head_range(H, world, r)
        pieces.append(parts[r][:, : b - a])
    return torch.cat(pieces, dim=1)
