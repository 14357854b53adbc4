"""Column split of the op across GPUs: one process per GPU, no data exchanged.

Output column j of the fused op depends on column j of x2, scale, bias and
sharedInput, and on the whole of x1, groupList, rowIndex, pertokenScale and
logit -- nothing else.  So P GPUs can each compute a block of output columns
on their own: every GPU holds the row-side inputs (x1 and the routing, the same
on all GPUs) and only its own columns of the weights, and writes only its own
columns of the output.  In deterministic mode each column block is summed in
the same fixed order as the whole op, so the stitched blocks are bitwise equal
to a single-GPU call.

Blocks are whole 256-column tiles (the library's n granule), dealt as evenly
as the tile count allows: with 28 tiles (n = 7168) over 8 GPUs, ranks 0-3 get
4 tiles and ranks 4-7 get 3.  A rank left with no tile (more GPUs than tiles)
gets an empty block and makes no call.

A block can be run in place inside full-width tensors: pass pointers advanced
to its first column and the full widths as the problem's strides
(``problem_strides``), or give each GPU compact copies of its columns (strides
left at 0).
"""
from __future__ import annotations

from typing import Tuple

N_GRANULE = 256   # columns per output tile: every block is a multiple of it


def column_block(n: int, world: int, rank: int, granule: int = N_GRANULE) -> Tuple[int, int]:
    """Columns [c0, c1) that rank `rank` of `world` owns for an n-column op."""
    if n % granule:
        raise ValueError(f"n = {n} is not a multiple of {granule}")
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    tiles = n // granule
    q, r = divmod(tiles, world)
    t0 = rank * q + min(rank, r)
    t1 = t0 + q + (1 if rank < r else 0)
    return t0 * granule, t1 * granule


def column_blocks(n: int, world: int, granule: int = N_GRANULE):
    """Every rank's block, in rank order; consecutive and covering [0, n)."""
    return [column_block(n, world, r, granule) for r in range(world)]


def problem_strides(n_full: int, weight: str = "int8") -> dict:
    """Keyword strides for ``make_problem`` when a block runs in place inside
    tensors that are n_full columns wide (x2, scale/bias, out, sharedInput)."""
    del weight   # ld_x2 counts columns for int8, int4 and transposed int8 alike
    return dict(ld_x2=n_full, ld_sb=n_full, ld_out=n_full, ld_shared=n_full)


def block_offsets(c0: int, k: int, weight: str = "int8", transpose_x2: bool = False) -> dict:
    """Byte offsets of column c0 inside full-width tensors: x2 in its layout, f32
    scale/bias/out, bf16 sharedInput (bf16 scale: use ``scale_bf16``)."""
    if weight == "int8":
        x2 = c0 * k if transpose_x2 else c0
    else:
        x2 = c0 // 8 * 4
    return dict(x2=x2, scale=4 * c0, scale_bf16=2 * c0, bias=4 * c0, out=4 * c0, shared=2 * c0)


def slice_columns(p, c0: int, c1: int):
    """A copy of host problem `p` (the fields of ``synth.Problem``) restricted to
    columns [c0, c1): compact copies of x2, scale, bias and sharedInput columns;
    the row-side inputs are shared with `p`."""
    import copy

    import numpy as np
    q = copy.copy(p)
    q.n = c1 - c0
    if p.weight == "int8":
        q.x2 = np.ascontiguousarray(p.x2[:, c0:c1, :] if getattr(p, "transpose_x2", False) else p.x2[:, :, c0:c1])
    else:
        q.x2 = np.ascontiguousarray(p.x2[:, :, c0 // 8:c1 // 8])
    for name in ("scale", "bias", "shared"):
        a = getattr(p, name, None)
        setattr(q, name, None if a is None else np.ascontiguousarray(a[:, c0:c1]))
    return q
