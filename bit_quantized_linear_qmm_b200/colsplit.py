"""Column-parallel split of a quantized linear layer over ranks (one process per GPU).

Each rank holds a contiguous block of the layer's output features, computes its
part of y = x W^T + b with the library (x is replicated), and the full y is
assembled with one all-gather -- the only exchange, needed only when the
consumer wants all of y.  Nothing else crosses ranks: the split needs no
collective on the data path.

The block of a rank depends on the weight format, because the formats lay out
output features differently:

- MLX affine codes [N, K*b/32], scales / biases [N, K/g], int8 weights [N, K],
  per-group int8 [N, K] with scales [K/g, N]: output n is row n, so a rank takes
  rows n0..n1 (and the matching columns of the group-major per-group scales).
- packed int4 [K/2, N]: output n is column n: a rank takes columns n0..n1.
- BitLinear [N/4, K]: byte row r holds outputs r + j N/4 (j = 0..3): a rank
  takes packed rows r0..r1, which are the outputs {r + j N/4}; its local layer
  has N_local = 4 (r1 - r0) and local output i + j N_local is global
  r0 + i + j N/4.

Blocks are balanced to within one alignment unit; `align` keeps every block a
multiple of what the kernels need (16 columns for packed int4, 4 outputs for
BitLinear through its packed rows).
"""
from __future__ import annotations

import numpy as np


def block(n: int, world: int, rank: int, align: int = 1) -> tuple[int, int]:
    """[start, stop) of rank's share of n units, in multiples of `align` (the last rank takes the rest)."""
    if not (0 <= rank < world) or n <= 0 or align <= 0:
        raise ValueError("bad split")
    units = -(-n // align)
    u0 = units * rank // world
    u1 = units * (rank + 1) // world
    return min(n, u0 * align), min(n, u1 * align)


def output_index(fmt: str, n: int, world: int, rank: int) -> np.ndarray:
    """Global output features of rank's share, in the order its local layer produces them."""
    if fmt == "bitlinear":
        R = n // 4
        r0, r1 = block(R, world, rank)
        rows = np.arange(r0, r1)
        return np.concatenate([rows + j * R for j in range(4)])
    align = 16 if fmt == "w4a8" else 1
    n0, n1 = block(n, world, rank, align)
    return np.arange(n0, n1)


def shard(fmt: str, weights: dict, n: int, world: int, rank: int) -> dict:
    """Rank's part of a layer's weight tensors (numpy or torch; slicing only).

    weights keys per format: affine: codes [N, .], scales [N, G], biases [N, G];
    w8a8: w [N, K], scale_w [N]; w4a8: packed [K/2, N], scale_w [N];
    pergroup: w [N, K], scale_w [G, N]; bitlinear: packed [N/4, K]; every format: bias [N] or None.
    """
    out = {}
    if fmt == "bitlinear":
        r0, r1 = block(n // 4, world, rank)
        out["packed"] = weights["packed"][r0:r1]
    else:
        n0, n1 = block(n, world, rank, 16 if fmt == "w4a8" else 1)
        for key, t in weights.items():
            if key == "bias" or t is None:
                continue
            if fmt == "w4a8" and key == "packed":
                out[key] = t[:, n0:n1]
            elif fmt == "pergroup" and key == "scale_w":
                out[key] = t[:, n0:n1]
            else:
                out[key] = t[n0:n1]
    bias = weights.get("bias")
    out["bias"] = None if bias is None else bias[output_index(fmt, n, world, rank)]
    return out


def assemble(fmt: str, parts: list, n: int) -> np.ndarray:
    """Full y [M, N] from every rank's local y (in rank order), as an all-gather delivers them."""
    world = len(parts)
    M = parts[0].shape[0]
    y = np.empty((M, n), dtype=parts[0].dtype)
    for rank, part in enumerate(parts):
        y[:, output_index(fmt, n, world, rank)] = part
    return y


def assemble_torch(fmt: str, parts: list, n: int):
    """assemble() for torch tensors on one device (the result of torch.distributed.all_gather)."""
    import torch
    world = len(parts)
    y = torch.empty((parts[0].shape[0], n), dtype=parts[0].dtype, device=parts[0].device)
    for rank, part in enumerate(parts):
        idx = torch.as_tensor(output_index(fmt, n, world, rank), device=part.device)
        y[:, idx] = part
    return y


def gather_y(y_local, fmt: str, n: int, group=None):
    """All-gathers every rank's local y (torch, [M, n_local]) and assembles the full y [M, n] in
    global output order.  Shares differ by at most one alignment unit, so each is padded to the
    largest before the collective (which needs equal sizes) and trimmed after it."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    sizes = [len(output_index(fmt, n, world, r)) for r in range(world)]
    width = max(sizes)
    M = y_local.shape[0]
    pad = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
    pad[:, : y_local.shape[1]] = y_local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad, group=group)
    return assemble_torch(fmt, [b[:, :s] for b, s in zip(bufs, sizes)], n)
