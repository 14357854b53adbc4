"""Seeded synthetic inputs for the expert-parallel AlltoAllv + quantised grouped matmul
+ shared-expert matmul of page "aclnnAlltoAllvQuantGroupedMatMul".

Recipe (random draws and data layout only, none of the operation's arithmetic):
- ``world`` cards, ``e`` experts per card; expert g lives on card g // e as that
  card's local expert g % e (page 2: each card computes only its own experts).
- Every card has ``tokens`` tokens (BS); each picks ``topk`` distinct experts out of
  world * e by the routing recipe of the single-card workloads (Gumbel-top-k over a
  popularity vector).  A (token, slot) pair becomes one row of the card's send
  buffer, which holds the token's activation row; the rows are ordered by
  destination card, then the destination's local expert, then token.  So BSK =
  tokens * topk and ``send_counts[d * e + j]`` counts the rows for card d's expert j.
- ``recv_counts`` of card r at ``s * e + j`` is card s's ``send_counts[r * e + j]``.
- Quant modes (page 2 names pertensor and mx as the supported ones):
  ``pertensor``: activations and weights are FLOAT8 E4M3FN codes with one f32
  scale per tensor (per card for the activations, per card for the routed weights,
  one for the shared expert's weights);
  ``mx``: activations are E4M3 codes with one E8M0 scale byte per 32 elements of a
  row, routed and shared weights are FP4 E2M1 pairs stored (experts, n, k/2) with
  one E8M0 scale byte per 32 k.
- The shared expert multiplies the card's BS token rows (``mm_x``, H2 wide) by its
  (H2, N2) weight.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from .inputs import SEED_BASE, e4m3_codes_normal, make_routing

EP_SEED_OFFSET = 100


@dataclass
class EpCard:
    """One card's inputs.  Arrays are host numpy arrays in the op's layouts."""
    rank: int
    x: np.ndarray                       # E4M3 codes [BSK, h1], send order
    x_scale: Optional[np.ndarray]       # pertensor: f32 [1]; mx: E8M0 [BSK, h1/32]
    send_counts: np.ndarray             # int64 [world * e]
    recv_counts: np.ndarray             # int64 [world * e]
    w: np.ndarray                       # pertensor: E4M3 [e, h1, n1]; mx: E2M1 pairs [e, n1, h1/2]
    w_scale: np.ndarray                 # pertensor: f32 [1]; mx: E8M0 [e, n1, h1/32]
    mm_x: Optional[np.ndarray]          # E4M3 [BS, h2]
    mm_x_scale: Optional[np.ndarray]    # pertensor: f32 [1]; mx: E8M0 [BS, h2/32]
    mm_w: Optional[np.ndarray]          # pertensor: E4M3 [h2, n2]; mx: E2M1 pairs [n2, h2/2]
    mm_w_scale: Optional[np.ndarray]    # pertensor: f32 [1]; mx: E8M0 [n2, h2/32]
    tokens_of_rows: np.ndarray = field(default=None)   # int64 [BSK]: the token each send row carries


@dataclass
class EpProblem:
    mode: str
    world: int
    e: int
    tokens: int
    topk: int
    h1: int
    n1: int
    h2: int
    n2: int
    cards: List[EpCard]


def make_ep_problem(world: int, e: int, tokens: int, topk: int, h1: int, n1: int, h2: int = 0, n2: int = 0,
                    mode: str = "mx", routing: str = "uniform", routing_param: float = 0.0,
                    seed: Optional[int] = None) -> EpProblem:
    if mode not in ("pertensor", "mx"):
        raise ValueError(mode)
    rng = np.random.default_rng(SEED_BASE + EP_SEED_OFFSET if seed is None else seed)
    E = world * e
    topk = min(topk, E)
    sends = []
    for c in range(world):
        experts, _ = make_routing(rng, tokens, topk, E, routing, routing_param)
        tok = np.repeat(np.arange(tokens, dtype=np.int64), topk)
        dest = experts.reshape(-1)                     # global expert = card * e + local expert
        order = np.lexsort((tok, dest))                # by destination card and expert, then token
        counts = np.bincount(dest, minlength=E).astype(np.int64)
        act = e4m3_codes_normal(rng, (tokens, h1), 2.0)
        rows = tok[order]
        x = act[rows]
        if mode == "mx":
            tok_sf = rng.integers(120, 128, size=(tokens, h1 // 32), dtype=np.uint8)
            x_scale = tok_sf[rows]
        else:
            x_scale = np.array([rng.uniform(1e-3, 1e-2)], np.float32)
        sends.append((x, x_scale, counts, rows))
    cards = []
    for r in range(world):
        recv = np.array([sends[s][2][r * e + j] for s in range(world) for j in range(e)], np.int64)
        if mode == "mx":
            w = rng.integers(0, 256, size=(e, n1, h1 // 2), dtype=np.uint8)
            w_scale = rng.integers(118, 128, size=(e, n1, h1 // 32), dtype=np.uint8)
        else:
            w = e4m3_codes_normal(rng, (e, h1, n1), 0.5)
            w_scale = np.array([rng.uniform(1e-3, 1e-2)], np.float32)
        mm_x = mm_x_scale = mm_w = mm_w_scale = None
        if h2 > 0 and n2 > 0:
            mm_x = e4m3_codes_normal(rng, (tokens, h2), 2.0)
            if mode == "mx":
                mm_x_scale = rng.integers(120, 128, size=(tokens, h2 // 32), dtype=np.uint8)
                mm_w = rng.integers(0, 256, size=(n2, h2 // 2), dtype=np.uint8)
                mm_w_scale = rng.integers(118, 128, size=(n2, h2 // 32), dtype=np.uint8)
            else:
                mm_x_scale = np.array([rng.uniform(1e-3, 1e-2)], np.float32)
                mm_w = e4m3_codes_normal(rng, (h2, n2), 0.5)
                mm_w_scale = np.array([rng.uniform(1e-3, 1e-2)], np.float32)
        x, x_scale, counts, rows = sends[r]
        cards.append(EpCard(rank=r, x=x, x_scale=x_scale, send_counts=counts, recv_counts=recv, w=w,
                            w_scale=w_scale, mm_x=mm_x, mm_x_scale=mm_x_scale, mm_w=mm_w, mm_w_scale=mm_w_scale,
                            tokens_of_rows=rows))
    return EpProblem(mode=mode, world=world, e=e, tokens=tokens, topk=topk, h1=h1, n1=n1, h2=h2, n2=n2, cards=cards)
