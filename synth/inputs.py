"""Seeded synthetic workloads of the shapes the GroupedMatmulFinalizeRouting pages use.

Shapes and limits follow the aclnnGroupedMatmulFinalizeRoutingWeightNzV2 page
(parameter constraints: m up to 16*1024*8, k = 2048, n = 7168, e in [1, 256]).
Value distributions and routing are the five workloads of this project
(tiny, mid prefill, decode, large prefill, W4A8 with the per-token prologue).

Routing recipe shared by every workload: each token picks ``topk`` distinct
experts; the (token, slot) pairs are stably sorted by expert, then by token.
That order is the row order of ``x1``; ``row_index[i]`` is the token of row i;
``logit[i]`` is that slot's routing weight; ``counts[g]`` is the number of rows
of expert g.  Sampling ``topk`` distinct experts in proportion to a popularity
vector p uses the Gumbel-top-k form of successive sampling without replacement:
the ``topk`` largest keys ``log p_j + G_j`` with G_j standard Gumbel.

Nothing here performs the op's arithmetic: int4 weights are drawn directly as
random 32-bit words (each nibble then is uniform over the 16 int4 values), and
bf16 tensors are plain random normals rounded to bf16 by torch.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

SEED_BASE = 20261202


@dataclass(frozen=True)
class Spec:
    index: int            # workload number; its seed is SEED_BASE + index
    tokens: int
    topk: int
    e: int
    k: int
    n: int
    routing: str          # 'top_normal' | 'zipf' | 'uniform' | 'dirichlet'
    routing_param: float
    group_list_type: int  # 0 = cumulative ends, 1 = per-group counts
    weight: str           # 'int8' | 'int4' | 'fp8' (x1 and x2 FLOAT8 E4M3FN) | 'mxfp4' (MxA8W4)
    bias: bool
    shared: bool
    shared_offset: int
    prologue: bool        # activations arrive as bf16 and go through per-token quant
    description: str


CONFIGS = {
    "tiny": Spec(1, 32, 2, 4, 256, 512, "top_normal", 0.0, 1, "int8", False, False, 0, False,
                 "tokens=32 topK=2 m=64 e=4 k=256 n=512; top-2 of normal logits, softmax weights"),
    "mid_prefill": Spec(2, 1024, 8, 32, 2048, 7168, "zipf", 1.1, 0, "int8", False, False, 0, False,
                        "tokens=1024 topK=8 m=8192 e=32 k=2048 n=7168; Zipf(1.1) expert popularity"),
    "decode": Spec(3, 16, 8, 256, 2048, 7168, "uniform", 0.0, 1, "int8", True, False, 0, False,
                   "tokens=16 topK=8 m=128 e=256 k=2048 n=7168; uniform experts, bias"),
    "large_prefill": Spec(4, 16384, 8, 256, 2048, 7168, "dirichlet", 0.3, 0, "int8", False, True, 0, False,
                          "tokens=16384 topK=8 m=131072 e=256 k=2048 n=7168; Dirichlet(0.3) popularity, "
                          "bf16 sharedInput at offset 0"),
    "w4a8_prologue": Spec(5, 4096, 8, 128, 2048, 7168, "uniform", 0.0, 0, "int4", True, False, 0, True,
                          "tokens=4096 topK=8 m=32768 e=128 k=2048 n=7168; int4 weights packed 8 per int32, "
                          "bf16 activations quantised per token, bias"),
    # page 1's Atlas 350 per-token / per-channel mode (x1 and x2 FLOAT8 E4M3FN) on the
    # large prefill's shapes and routing
    "fp8_prefill": Spec(6, 16384, 8, 256, 2048, 7168, "dirichlet", 0.3, 0, "fp8", False, True, 0, False,
                        "tokens=16384 topK=8 m=131072 e=256 k=2048 n=7168; x1 and x2 FLOAT8 E4M3FN, "
                        "Dirichlet(0.3) popularity, bf16 sharedInput at offset 0"),
    # page 1's Atlas 350 MxA8W4 mode on the W4A8 workload's shapes: bf16 activations
    # through the per-32-group FP8 cast, FP4 E2M1 weights (e, n, k) with E8M0 block scales
    "w4a8_mx": Spec(7, 4096, 8, 128, 2048, 7168, "uniform", 0.0, 0, "mxfp4", True, False, 0, True,
                    "tokens=4096 topK=8 m=32768 e=128 k=2048 n=7168; MxA8W4: bf16 activations cast to E4M3 "
                    "with E8M0 scales per 32, FP4 E2M1 weights (e, n, k) with E8M0 scales per 32, bias"),
}


@dataclass
class Problem:
    """One seeded instance.  Arrays are host numpy arrays in the op's layouts."""
    name: str
    tokens: int
    topk: int
    m: int
    e: int
    k: int
    n: int
    output_bs: int
    group_list_type: int
    weight: str
    x1: Optional[np.ndarray]          # int8 [m, k]   (None when the prologue makes it)
    x_bf16: Optional[np.ndarray]      # uint16 bf16 bits [m, k] (prologue workloads only)
    x2: np.ndarray                    # int8 / E4M3 bytes [e, k, n] or int32 [e, k, n/8]
    scale: np.ndarray                 # f32 [e, n]
    pertoken_scale: Optional[np.ndarray]  # f32 [m]  (None when the prologue makes it)
    group_list: np.ndarray            # int64 [e]
    counts: np.ndarray                # int64 [e]
    logit: np.ndarray                 # f32 [m]
    row_index: np.ndarray             # int64 [m]
    bias: Optional[np.ndarray]        # f32 [e, n]
    shared: Optional[np.ndarray]      # uint16 bf16 bits [shared_bs, n]
    shared_offset: int
    extra: dict = field(default_factory=dict)

    @property
    def shared_bs(self) -> int:
        return 0 if self.shared is None else int(self.shared.shape[0])


def _softmax_rows(v: np.ndarray) -> np.ndarray:
    z = v - v.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=1, keepdims=True)


def _gumbel_topk(rng: np.random.Generator, logp: np.ndarray, tokens: int, topk: int) -> np.ndarray:
    g = rng.gumbel(size=(tokens, logp.shape[0]))
    keys = logp[None, :] + g
    part = np.argpartition(-keys, topk - 1, axis=1)[:, :topk]
    return part


def make_routing(rng: np.random.Generator, tokens: int, topk: int, e: int, kind: str, param: float):
    """Return (experts [tokens, topk] distinct per row, weights f32 [tokens, topk])."""
    if kind == "top_normal":
        lg = rng.standard_normal((tokens, e))
        experts = np.argsort(-lg, axis=1, kind="stable")[:, :topk]
        weights = _softmax_rows(np.take_along_axis(lg, experts, axis=1))
        return experts.astype(np.int64), weights.astype(np.float32)
    if kind == "zipf":
        p = np.arange(1, e + 1, dtype=np.float64) ** (-param)
    elif kind == "uniform":
        p = np.ones(e, dtype=np.float64)
    elif kind == "dirichlet":
        p = rng.dirichlet(np.full(e, param))
        p = np.maximum(p, 1e-300)
    else:
        raise ValueError(kind)
    p = p / p.sum()
    experts = _gumbel_topk(rng, np.log(p), tokens, topk)
    weights = _softmax_rows(rng.standard_normal((tokens, topk)))
    return experts.astype(np.int64), weights.astype(np.float32)


def _layout(experts: np.ndarray, weights: np.ndarray, e: int):
    tokens, topk = experts.shape
    tok = np.repeat(np.arange(tokens, dtype=np.int64), topk)
    exp = experts.reshape(-1)
    w = weights.reshape(-1)
    order = np.lexsort((tok, exp))           # primary key expert, then token
    row_index = tok[order]
    logit = w[order].astype(np.float32)
    counts = np.bincount(exp, minlength=e).astype(np.int64)
    return row_index, logit, counts


def bf16_bits_normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    import torch
    v = (rng.standard_normal(shape, dtype=np.float32) * np.float32(std))
    return torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def e4m3_codes_normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    """FLOAT8 E4M3FN codes (uint8) of normal(0, std) draws, converted by torch's
    float8_e4m3fn cast (round to nearest even) in chunks of the leading axis."""
    import torch
    out = np.empty(shape, np.uint8)
    lead = out.reshape(shape[0], -1)
    for i in range(shape[0]):
        v = rng.standard_normal(lead.shape[1], dtype=np.float32) * np.float32(std)
        lead[i] = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return out


def make_problem(name: str, *, tokens: Optional[int] = None, e: Optional[int] = None,
                 k: Optional[int] = None, n: Optional[int] = None, seed: Optional[int] = None,
                 group_list_type: Optional[int] = None, weights_only_experts: Optional[np.ndarray] = None,
                 ) -> Problem:
    """Build workload ``name``; keyword overrides shrink it for tests (same recipe)."""
    spec = CONFIGS[name]
    tokens = spec.tokens if tokens is None else tokens
    e = spec.e if e is None else e
    k = spec.k if k is None else k
    n = spec.n if n is None else n
    gtype = spec.group_list_type if group_list_type is None else group_list_type
    topk = min(spec.topk, e)
    rng = np.random.default_rng(SEED_BASE + spec.index if seed is None else seed)

    experts, weights = make_routing(rng, tokens, topk, e, spec.routing, spec.routing_param)
    row_index, logit, counts = _layout(experts, weights, e)
    m = tokens * topk
    group_list = np.cumsum(counts).astype(np.int64) if gtype == 0 else counts.copy()

    if spec.prologue:
        x1 = None
        x_bf16 = bf16_bits_normal(rng, (m, k))
        pts = None
    elif spec.weight == "fp8":
        x1 = e4m3_codes_normal(rng, (m, k), 4.0)
        x_bf16 = None
        pts = rng.uniform(1e-3, 1e-2, size=m).astype(np.float32)
    else:
        x1 = rng.integers(-127, 128, size=(m, k), dtype=np.int8)
        x_bf16 = None
        pts = rng.uniform(1e-3, 1e-2, size=m).astype(np.float32)
    if spec.weight == "int8":
        x2 = rng.integers(-127, 128, size=(e, k, n), dtype=np.int8)
    elif spec.weight == "fp8":
        x2 = e4m3_codes_normal(rng, (e, k, n), 0.5)
    elif spec.weight == "mxfp4":
        x2 = rng.integers(0, 256, size=(e, n, k // 2), dtype=np.uint8)     # every nibble uniform over the 16 codes
    else:
        x2 = rng.integers(0, 2 ** 32, size=(e, k, n // 8), dtype=np.uint32).view(np.int32)
    if spec.weight == "mxfp4":      # E8M0 weight scales per 32 k: 2^-9 .. 2^0
        scale = rng.integers(118, 128, size=(e, n, k // 32), dtype=np.uint8)
    else:
        scale = rng.uniform(1e-3, 1e-2, size=(e, n)).astype(np.float32)
    bias = rng.normal(0.0, 0.01, size=(e, n)).astype(np.float32) if spec.bias else None
    shared = bf16_bits_normal(rng, (tokens, n)) if spec.shared else None
    pr = Problem(name=name, tokens=tokens, topk=topk, m=m, e=e, k=k, n=n, output_bs=tokens,
                 group_list_type=gtype, weight=spec.weight, x1=x1, x_bf16=x_bf16, x2=x2,
                 scale=scale, pertoken_scale=pts, group_list=group_list, counts=counts,
                 logit=logit, row_index=row_index, bias=bias, shared=shared,
                 shared_offset=spec.shared_offset)
    if spec.weight == "mxfp4":
        pr.transpose_x2 = True      # the MX weights are (e, n, k), as page 1 requires in that mode
    return pr


def sample_rows(rng_seed: int, limit: int, count: int) -> np.ndarray:
    """A sorted seeded sample of distinct row ids in [0, limit)."""
    rng = np.random.default_rng(rng_seed)
    count = min(count, limit)
    return np.sort(rng.choice(limit, size=count, replace=False)).astype(np.int64)

