"""CPU oracle of the expert-parallel AlltoAllv + quantised grouped matmul + shared-expert
matmul (page "aclnnAlltoAllvQuantGroupedMatMul", function description and the list of
shape variables).

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only ``tests/``, the smoke entry
and the benchmark's CPU leg may use it.  It shares no code with the CUDA library.

What each card computes (page 2, in the readings this project takes where the page's
formulas are not legible):
  1. AlltoAllv: card r receives from every card s the rows s addressed to r's experts;
     s's send buffer holds them in (destination card, local expert) order.
  2. Permute: the received rows are put in expert order, and inside one expert in
     source-card order; the order inside a chunk is kept.  This buffer is
     permuteOut, and its per-expert counts are the grouped matmul's group list.
  3. Grouped matmul over the card's own experts: each permuted row times its
     expert's weight, dequantised by the quant mode (below).
  4. The shared expert's matmul of the card's own BS token rows, beside it.
Dequantisation, in the modes page 2 supports:
  pertensor: y = (acc * weight scale) * activation scale, acc the exact sum of E4M3
             products, the activation scale that of the row's source card;
  mx:        y = sum over 32-blocks of 2^(sfa-127) 2^(sfb-127) times the block's exact
             E4M3 x E2M1 product sum (the MxA8W4 oracle).
The matmuls reuse the pinned single-card oracle (``finalize`` / ``finalize_mx``) with
identity routing, unit logits and no bias, so each output row is its source row's
product; the permute is written out here with plain loops over cards and experts.
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np

from . import finalize, finalize_mx


def dispatch(send_rows: Sequence[np.ndarray], send_counts: Sequence[np.ndarray], e: int):
    """Steps 1-2 for every card.  ``send_rows[s]`` is card s's send buffer (any row
    width), ``send_counts[s]`` its world*e chunk counts.  Returns a list over cards r
    of ``(permuted rows, group_counts [e])``."""
    world = len(send_rows)
    result = []
    for r in range(world):
        pieces: List[np.ndarray] = []
        group_counts = np.zeros(e, np.int64)
        for j in range(e):
            for s in range(world):
                counts = np.asarray(send_counts[s], np.int64)
                start = int(counts[: r * e + j].sum())      # rows before chunk (r, j) in s's buffer
                cnt = int(counts[r * e + j])
                pieces.append(np.asarray(send_rows[s])[start:start + cnt])
                group_counts[j] += cnt
        width = np.asarray(send_rows[0]).shape[1:]
        rows = np.concatenate(pieces) if pieces else np.zeros((0,) + width, np.asarray(send_rows[0]).dtype)
        result.append((rows, group_counts))
    return result


def source_cards(send_counts: Sequence[np.ndarray], e: int) -> List[np.ndarray]:
    """For every card r, the source card of each of its permuted rows."""
    world = len(send_counts)
    tags = [np.full((int(np.sum(send_counts[s])), 1), s, np.int64) for s in range(world)]
    return [rows[:, 0] for rows, _ in dispatch(tags, send_counts, e)]


def grouped_matmul(mode: str, x, x_scale_rows, group_counts, w, w_scale, want32: bool = False):
    """Step 3 on one card: ``x`` [A, h1] permuted E4M3 codes, ``x_scale_rows`` the
    per-row activation scale (pertensor: f32 [A]) or E8M0 [A, h1/32] (mx); ``w`` and
    ``w_scale`` in the card's layout.  Returns (out64, sabs, out32) of shape [A, n1]."""
    a = int(np.sum(group_counts))
    if mode == "pertensor":
        e, _, n1 = w.shape
        scale = np.full((e, n1), np.float32(np.asarray(w_scale).reshape(-1)[0]), np.float32)
        return finalize(x, w, np.asarray(group_counts, np.int64), 1, weight="fp8", scale=scale,
                        pertoken_scale=np.asarray(x_scale_rows, np.float32).reshape(-1), output_bs=a,
                        row_index=np.arange(a, dtype=np.int64), want32=want32)
    return finalize_mx(x, x_scale_rows, w, w_scale, np.asarray(group_counts, np.int64), 1, output_bs=a,
                       row_index=np.arange(a, dtype=np.int64), want32=want32)


def shared_matmul(mode: str, mm_x, mm_x_scale, mm_w, mm_w_scale, want32: bool = False):
    """Step 4: the shared expert's matmul of [BS, h2] by its weight (one group)."""
    bs = mm_x.shape[0]
    gl = np.array([bs], np.int64)
    if mode == "pertensor":
        n2 = mm_w.shape[1]
        scale = np.full((1, n2), np.float32(np.asarray(mm_w_scale).reshape(-1)[0]), np.float32)
        pts = np.full(bs, np.float32(np.asarray(mm_x_scale).reshape(-1)[0]), np.float32)
        return finalize(mm_x, mm_w[None], gl, 1, weight="fp8", scale=scale, pertoken_scale=pts, output_bs=bs,
                        row_index=np.arange(bs, dtype=np.int64), want32=want32)
    return finalize_mx(mm_x, mm_x_scale, mm_w[None], mm_w_scale[None], gl, 1, output_bs=bs,
                       row_index=np.arange(bs, dtype=np.int64), want32=want32)


def reference(problem, want32: bool = False):
    """All four steps for every card of a ``synth.ep.EpProblem``.  Returns a list over
    cards of dicts: ``permute_out``, ``permute_scale`` (mx: E8M0 rows; pertensor: the
    per-row f32 source-card scale), ``group_counts``, ``gmm`` and ``mm`` as
    (out64, sabs, out32) tuples (``mm`` None without a shared expert)."""
    p = problem
    cards = p.cards
    counts = [c.send_counts for c in cards]
    xs = dispatch([c.x for c in cards], counts, p.e)
    if p.mode == "mx":
        scales = [rows for rows, _ in dispatch([c.x_scale for c in cards], counts, p.e)]
    else:
        src = source_cards(counts, p.e)
        scales = [np.array([cards[s].x_scale[0] for s in src[r]], np.float32) for r in range(p.world)]
    out = []
    for r, c in enumerate(cards):
        x, gc = xs[r]
        gmm = grouped_matmul(p.mode, x, scales[r], gc, c.w, c.w_scale, want32) if x.shape[0] > 0 else None
        mm = (shared_matmul(p.mode, c.mm_x, c.mm_x_scale, c.mm_w, c.mm_w_scale, want32)
              if c.mm_x is not None else None)
        out.append({"permute_out": x, "permute_scale": scales[r], "group_counts": gc, "gmm": gmm, "mm": mm})
    return out
