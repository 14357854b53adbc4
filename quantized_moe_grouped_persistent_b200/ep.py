"""Expert-parallel AlltoAllv + quantised grouped matmul + shared-expert matmul on B200.

Page "aclnnAlltoAllvQuantGroupedMatMul", function description: the routed experts
are spread over the epWorldSize cards of an EP domain, e per card; each card first
exchanges token rows with every other card, permutes what it received into expert
order and runs the quantised grouped matmul over its own experts, while the shared
expert's quantised matmul runs beside it.  The quant modes are the two the page
supports: ``pertensor`` (E4M3 activations and weights, one f32 scale per tensor)
and ``mx`` (E4M3 activations with E8M0 scales per 32 elements, FP4 E2M1 weights
stored (e, n, k/2) with E8M0 scales per 32 k: the library's MxA8W4 mode).

How it maps onto this library (marshalling only; no arithmetic in Python):
  - ``qgmm_ep_plan`` (C ABI, host) turns the send and receive counts into the offset
    of every (card, expert) chunk in the send buffer and in the permuted receive
    buffer.
  - The exchange posts one send and one receive per non-empty (peer, expert) chunk
    in a single batched group of torch.distributed point-to-point operations (NCCL
    over NVLink on GPUs, gloo on the CPU), each receive landing straight at its
    permuted offset: the permute costs no pass of its own.  The chunks a card
    addresses to itself move in one library kernel (``qgmm_ep_permute_rows``) per
    buffer.  The activation scales travel the same
    way (mx: the E8M0 rows; pertensor: the source card's scale, one f32 per row).
  - The grouped matmul is ``qgmm_finalize`` over the permuted rows with the
    per-expert counts as a type-1 group list, identity routing and unit logits, so
    each output row is its permuted row's dequantised product (f32).
  - The shared expert's matmul is ``qgmm_finalize`` with one group, launched first
    on a side stream so that it runs while the exchange is in flight.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (QGMM_GROUP_COUNTS, QGMM_W_FP8_E4M3, QGMM_W_MXFP4, QgmmError, QGMM_ERR_SHAPE, ep_permute_rows, ep_plan,
               finalize, finalize_profiled, finalize_workspace, make_problem)

MODES = ("pertensor", "mx")


def _dev(a, device):
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return a.to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def _counts_to(device, counts) -> torch.Tensor:
    """Host counts -> a device int64 tensor, through pinned memory without a host wait."""
    host = torch.tensor(np.asarray(counts, np.int64).reshape(-1), dtype=torch.int64)
    if device.type != "cuda":
        return host
    return host.pin_memory().to(device, non_blocking=True)


def _scalar(v) -> float:
    """A per-tensor scale given as a number, a 1-element array or a 1-element tensor."""
    if isinstance(v, torch.Tensor):
        v = v.detach().cpu().numpy()
    return float(np.asarray(v, np.float64).reshape(-1)[0])


class Exchange:
    """The AlltoAllv with the permute folded into where each chunk lands.

    ``local(src, dst, src_rows, dst_rows, counts)`` moves the card's own chunks; the
    default is the library's one-kernel device copy (device tensors only)."""

    def __init__(self, world: int, rank: int, e: int, group=None, local=None):
        self.world, self.rank, self.e, self.group = world, rank, e, group
        self.local = ep_permute_rows if local is None else local

    def check_counts(self, send_counts, recv_counts, device) -> None:
        """Every card's receive counts must be its peers' send counts (page 2: the
        cards' A sum to their BSK).  One all-gather of the counts; raises on a mismatch."""
        import torch.distributed as dist
        mine = torch.tensor(np.concatenate([send_counts, recv_counts]).astype(np.int64), device=device)
        every = [torch.empty_like(mine) for _ in range(self.world)]
        dist.all_gather(every, mine, group=self.group)
        c = np.stack([t.cpu().numpy() for t in every])
        n = self.world * self.e
        sends, recvs = c[:, :n], c[:, n:]
        for r in range(self.world):
            for s in range(self.world):
                if not np.array_equal(recvs[r, s * self.e:(s + 1) * self.e], sends[s, r * self.e:(r + 1) * self.e]):
                    raise QgmmError(QGMM_ERR_SHAPE, f"ep exchange: card {r} expects other counts from card {s}")

    def run(self, pairs, plan, send_counts, recv_counts) -> None:
        """``pairs``: (send buffer, permuted receive buffer) tensors, rows first, all
        with the same chunking.  Posts every transfer, then waits for all of them."""
        import torch.distributed as dist
        e, so, ro = self.e, plan["send_offsets"], plan["recv_offsets"]
        own = slice(self.rank * e, (self.rank + 1) * e)   # the chunks this card keeps
        if not np.array_equal(np.asarray(send_counts)[own], np.asarray(recv_counts)[own]):
            raise QgmmError(QGMM_ERR_SHAPE, "ep exchange: own send and receive counts differ")
        if int(np.asarray(send_counts)[own].sum()) > 0:
            for src, dst in pairs:
                self.local(src, dst, so[own], ro[own], np.asarray(send_counts)[own])
        ops = []
        for peer in range(self.world):
            if peer == self.rank:
                continue
            for j in range(e):
                c = peer * e + j
                sc, rc = int(send_counts[c]), int(recv_counts[c])
                for b, (src, dst) in enumerate(pairs):
                    tag = b * e + j
                    if sc:
                        ops.append(dist.P2POp(dist.isend, src[int(so[c]):int(so[c]) + sc], peer, self.group, tag))
                    if rc:
                        rs = int(ro[c])
                        ops.append(dist.P2POp(dist.irecv, dst[rs:rs + rc], peer, self.group, tag))
        if ops:
            for w in dist.batch_isend_irecv(ops):
                w.wait()


class EpGroupedMatmul:
    """One card's AlltoAllv + grouped matmul + shared-expert matmul, weights resident.

    ``w``/``w_scale``: pertensor -- E4M3 codes [e, h1, n1] and one f32 scale;
    mx -- E2M1 pairs [e, n1, h1/2] and E8M0 bytes [e, n1, h1/32].  The shared
    expert (optional): pertensor -- E4M3 [h2, n2] and one f32 scale; mx -- E2M1
    pairs [n2, h2/2] and E8M0 [n2, h2/32].
    """

    def __init__(self, mode: str, world: int, rank: int, e: int, w, w_scale, mm_w=None, mm_w_scale=None,
                 device="cuda", group=None):
        if mode not in MODES:
            raise ValueError(mode)
        self.mode, self.world, self.rank, self.e = mode, world, rank, e
        self.device = torch.device(device)
        self.exchange = Exchange(world, rank, e, group)
        self.w = _dev(w, self.device)
        if mode == "pertensor":
            _, self.h1, self.n1 = w.shape
            self.w_scale = torch.full((e, self.n1), _scalar(w_scale), dtype=torch.float32, device=self.device)
        else:
            _, self.n1, half = w.shape
            self.h1 = 2 * half
            self.w_scale = _dev(w_scale, self.device)
        self.mm_w = None
        if mm_w is not None:
            if mode == "pertensor":
                self.h2, self.n2 = mm_w.shape
                self.mm_w = _dev(mm_w, self.device).reshape(1, self.h2, self.n2)
                self.mm_w_scale = torch.full((1, self.n2), _scalar(mm_w_scale), dtype=torch.float32,
                                             device=self.device)
            else:
                self.n2, half = mm_w.shape
                self.h2 = 2 * half
                self.mm_w = _dev(mm_w, self.device).reshape(1, self.n2, half)
                self.mm_w_scale = _dev(mm_w_scale, self.device).reshape(1, self.n2, self.h2 // 32)
        self._ws = {}
        self._side = None

    # -- the library calls -------------------------------------------------------------
    def _problem(self, m, k, n, e):
        wt = QGMM_W_FP8_E4M3 if self.mode == "pertensor" else QGMM_W_MXFP4
        return make_problem(m, k, n, e, m, weight_type=wt, group_list_type=QGMM_GROUP_COUNTS,
                            transpose_x2=self.mode == "mx")

    def _workspace(self, prob, key):
        nbytes = finalize_workspace(prob)
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            self._ws[key] = ws
        return ws

    def _matmul(self, key, x, x_scale, group_list, w, w_scale, k, n, e, out, stream, events=None):
        prob = self._problem(int(x.shape[0]), k, n, e)
        ws = self._workspace(prob, key)
        if events is None:
            finalize(prob, x, w, w_scale, x_scale, group_list, None, None, None, None, out, ws, stream=stream)
        else:         # the caller's two CUDA events, recorded around the grouped GEMM's launch
            finalize_profiled(prob, x, w, w_scale, x_scale, group_list, None, None, None, None, out, ws, events[0],
                              events[1], stream=stream)

    # -- the three parts of one call ---------------------------------------------------
    def shared(self, mm_x, mm_x_scale):
        """Launch the shared expert's matmul on the side stream (after the current
        stream's prior work) and return its output [BS, n2]; ``join()`` makes the
        current stream wait for it."""
        dev = self.device
        cur = torch.cuda.current_stream(dev)
        mm_x = _dev(mm_x, dev)
        bs = int(mm_x.shape[0])
        if self.mode == "pertensor":
            mm_scale = torch.full((bs,), _scalar(mm_x_scale), dtype=torch.float32, device=dev)
        else:
            mm_scale = _dev(mm_x_scale, dev)
        mm_gl = _counts_to(dev, [bs])
        mm_y = torch.empty((bs, self.n2), dtype=torch.float32, device=dev)
        if self._side is None:
            self._side = torch.cuda.Stream(dev)
        self._side.wait_stream(cur)
        self._matmul("mm", mm_x, mm_scale, mm_gl, self.mm_w, self.mm_w_scale, self.h2, self.n2, 1, mm_y, self._side)
        for t in (mm_x, mm_scale, mm_gl, mm_y):     # allocated on the current stream, used on the side one
            t.record_stream(self._side)
        return mm_y

    def join(self) -> None:
        if self._side is not None:
            torch.cuda.current_stream(self.device).wait_stream(self._side)

    def dispatch(self, x, x_scale, send_counts, recv_counts, check_counts: bool = True):
        """AlltoAllv + permute.  ``x``: this card's send buffer, E4M3 codes [BSK, h1]
        in (destination card, expert) order; ``x_scale``: pertensor -- one f32 (a
        number or a 1-element array); mx -- E8M0 [BSK, h1/32].  Returns
        ``(permute_out [A, h1], permute_scale, plan)``; ``permute_scale`` is f32 [A]
        (each row's source-card scale) or E8M0 [A, h1/32]."""
        dev = self.device
        send_counts = np.asarray(send_counts, np.int64).reshape(-1)
        recv_counts = np.asarray(recv_counts, np.int64).reshape(-1)
        plan = ep_plan(self.world, self.e, send_counts, recv_counts)
        if check_counts and self.world > 1:
            self.exchange.check_counts(send_counts, recv_counts, dev)
        x = _dev(x, dev)
        if x.shape[0] != plan["bsk"] or x.shape[1] != self.h1:
            raise QgmmError(QGMM_ERR_SHAPE, "ep: x must be [sum(send_counts), h1]")
        a = plan["a"]
        permute_out = torch.empty((a, self.h1), dtype=torch.uint8, device=dev)
        if self.mode == "pertensor":
            send_scale = torch.full((plan["bsk"], 1), _scalar(x_scale), dtype=torch.float32, device=dev)
            permute_scale = torch.empty((a, 1), dtype=torch.float32, device=dev)
        else:
            send_scale = _dev(x_scale, dev)
            permute_scale = torch.empty((a, self.h1 // 32), dtype=torch.uint8, device=dev)
        self.exchange.run([(x, permute_out), (send_scale, permute_scale)], plan, send_counts, recv_counts)
        return permute_out, (permute_scale.reshape(-1) if self.mode == "pertensor" else permute_scale), plan

    def grouped(self, permute_out, permute_scale, group_counts, events=None):
        """The grouped matmul over this card's experts: f32 [A, n1] (None when A = 0).
        ``events``: two CUDA events to record around the grouped GEMM kernel."""
        dev = self.device
        a = int(permute_out.shape[0])
        if a == 0:
            return None
        gl = _counts_to(dev, group_counts)
        gmm_y = torch.empty((a, self.n1), dtype=torch.float32, device=dev)
        self._matmul("gmm", permute_out, permute_scale, gl, self.w, self.w_scale, self.h1, self.n1, self.e, gmm_y,
                     torch.cuda.current_stream(dev), events)
        return gmm_y

    def forward(self, x, x_scale, send_counts, recv_counts, mm_x=None, mm_x_scale=None,
                check_counts: bool = True, events=None) -> dict:
        """One call: the shared expert's matmul starts on the side stream, then the
        exchange, then the grouped matmul; the current stream then waits for both.
        Returns ``gmm_y`` f32 [A, n1] (None if A = 0), ``mm_y`` f32 [BS, n2] (None
        without a shared expert), ``permute_out``, ``permute_scale``, ``group_counts``."""
        mm_y = self.shared(mm_x, mm_x_scale) if mm_x is not None and self.mm_w is not None else None
        permute_out, permute_scale, plan = self.dispatch(x, x_scale, send_counts, recv_counts, check_counts)
        gmm_y = self.grouped(permute_out, permute_scale, plan["group_counts"], events)
        if mm_y is not None:
            self.join()
        return {"gmm_y": gmm_y, "mm_y": mm_y, "permute_out": permute_out, "permute_scale": permute_scale,
                "group_counts": plan["group_counts"]}
