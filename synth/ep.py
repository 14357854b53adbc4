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
from typing import List, Optional, Sequence

import numpy as np

from .inputs import SEED_BASE, e4m3_codes_normal, make_routing

EP_SEED_OFFSET = 100


@dataclass
class EpCard:
    """One card's inputs.  Arrays are host numpy arrays in the op's layouts."""
    rank: int
    x: Optional[np.ndarray]             # E4M3 codes [BSK, h1], send order
    x_scale: Optional[np.ndarray]       # pertensor: f32 [1]; mx: E8M0 [BSK, h1/32]
    send_counts: np.ndarray             # int64 [world * e]
    recv_counts: np.ndarray             # int64 [world * e]
    w: Optional[np.ndarray]             # pertensor: E4M3 [e, h1, n1]; mx: E2M1 pairs [e, n1, h1/2]
    w_scale: Optional[np.ndarray]       # pertensor: f32 [1]; mx: E8M0 [e, n1, h1/32]
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
                    seed: Optional[int] = None, ranks: Optional[Sequence[int]] = None) -> EpProblem:
    """Every card's counts; the activations and weights of the cards in ``ranks``
    (default all; a card left out has them as None).  One generator draws every
    card's routing, then card c's data comes from a generator of its own, so a card's
    data is the same whichever cards are drawn."""
    if mode not in ("pertensor", "mx"):
        raise ValueError(mode)
    base = SEED_BASE + EP_SEED_OFFSET if seed is None else seed
    rng = np.random.default_rng(base)
    E = world * e
    topk = min(topk, E)
    layouts = []
    for c in range(world):
        experts, _ = make_routing(rng, tokens, topk, E, routing, routing_param)
        tok = np.repeat(np.arange(tokens, dtype=np.int64), topk)
        dest = experts.reshape(-1)                     # global expert = card * e + local expert
        order = np.lexsort((tok, dest))                # by destination card and expert, then token
        counts = np.bincount(dest, minlength=E).astype(np.int64)
        layouts.append((counts, tok[order]))
    wanted = set(range(world) if ranks is None else ranks)
    cards = []
    for r in range(world):
        counts, rows = layouts[r]
        recv = np.array([layouts[s][0][r * e + j] for s in range(world) for j in range(e)], np.int64)
        card = EpCard(rank=r, x=None, x_scale=None, send_counts=counts, recv_counts=recv, w=None, w_scale=None,
                      mm_x=None, mm_x_scale=None, mm_w=None, mm_w_scale=None, tokens_of_rows=rows)
        if r in wanted:
            g = np.random.default_rng([base, r + 1])
            act = e4m3_codes_normal(g, (tokens, h1), 2.0)
            card.x = act[rows]
            if mode == "mx":
                card.x_scale = g.integers(120, 128, size=(tokens, h1 // 32), dtype=np.uint8)[rows]
                card.w = g.integers(0, 256, size=(e, n1, h1 // 2), dtype=np.uint8)
                card.w_scale = g.integers(118, 128, size=(e, n1, h1 // 32), dtype=np.uint8)
            else:
                card.x_scale = np.array([g.uniform(1e-3, 1e-2)], np.float32)
                card.w = e4m3_codes_normal(g, (e, h1, n1), 0.5)
                card.w_scale = np.array([g.uniform(1e-3, 1e-2)], np.float32)
            if h2 > 0 and n2 > 0:
                card.mm_x = e4m3_codes_normal(g, (tokens, h2), 2.0)
                if mode == "mx":
                    card.mm_x_scale = g.integers(120, 128, size=(tokens, h2 // 32), dtype=np.uint8)
                    card.mm_w = g.integers(0, 256, size=(n2, h2 // 2), dtype=np.uint8)
                    card.mm_w_scale = g.integers(118, 128, size=(n2, h2 // 32), dtype=np.uint8)
                else:
                    card.mm_x_scale = np.array([g.uniform(1e-3, 1e-2)], np.float32)
                    card.mm_w = e4m3_codes_normal(g, (h2, n2), 0.5)
                    card.mm_w_scale = np.array([g.uniform(1e-3, 1e-2)], np.float32)
        cards.append(card)
    return EpProblem(mode=mode, world=world, e=e, tokens=tokens, topk=topk, h1=h1, n1=n1, h2=h2, n2=n2, cards=cards)


# The benchmark's expert-parallel workload, per card: page 2's limits (e <= 32 per card,
# topK in [2, 8], H2 <= 12288) with the single-card workloads' hidden size as H1 and
# H2 and a 4096-wide first projection (two 2048-wide halves) as N1 and N2.
EP_BENCH = dict(e=32, tokens=4096, topk=8, h1=7168, n1=4096, h2=7168, n2=4096)
