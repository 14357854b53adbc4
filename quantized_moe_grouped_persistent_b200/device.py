"""Device-resident operands for one problem instance, and calls through the C ABI.

Marshalling only: host arrays are copied into torch device tensors, and the
operation itself runs in libqgmm.so's kernels.
"""
from __future__ import annotations

import copy
from typing import Optional

import numpy as np
import torch

from . import (QGMM_IDX_INT32, QGMM_IDX_INT64, QGMM_SCALE_BF16, QGMM_SCALE_F32, QGMM_W_FP8_E4M3,
               QGMM_W_INT4_PACKED_INT32, QGMM_W_INT8, QGMM_W_MXFP4, debug_accum_mx, per_token_quant_mxfp8,
               debug_accum, device_status, finalize, finalize_workspace, make_problem, per_token_quant)


def to_device(a: Optional[np.ndarray], device) -> Optional[torch.Tensor]:
    if a is None:
        return None
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


class DeviceProblem:
    """Operands of one instance on ``device``; ``p`` has the fields of ``synth.Problem``."""

    def __init__(self, p, device="cuda", expected_m_per_expert: int = 0, with_optional: bool = True):
        self.p = p
        self.device = torch.device(device)
        self.m, self.k, self.n, self.e = p.m, p.k, p.n, p.e
        self.output_bs = p.output_bs
        self.weight_type = {"int8": QGMM_W_INT8, "int4": QGMM_W_INT4_PACKED_INT32,
                            "fp8": QGMM_W_FP8_E4M3, "mxfp4": QGMM_W_MXFP4}[p.weight]
        self.mx = p.weight == "mxfp4"
        self.group_list_type = p.group_list_type
        self.expected_m_per_expert = expected_m_per_expert
        dev = self.device
        self.prologue = p.x1 is None
        if self.prologue and self.mx:     # the per-32-group FP8 cast: E4M3 codes and E8M0 scales
            self.x_bf16 = to_device(p.x_bf16, dev)
            self.x1 = torch.empty((p.m, p.k), dtype=torch.uint8, device=dev)
            self.pts = torch.empty((p.m, p.k // 32), dtype=torch.uint8, device=dev)
        elif self.prologue:
            self.x_bf16 = to_device(p.x_bf16, dev)
            self.x1 = torch.empty((p.m, p.k), dtype=torch.int8, device=dev)
            self.pts = torch.empty(p.m, dtype=torch.float32, device=dev)
        else:
            self.x_bf16 = None
            self.x1 = to_device(p.x1, dev)
            self.pts = to_device(p.pertoken_scale, dev)
        self.x2 = to_device(p.x2, dev)
        self.transpose_x2 = bool(getattr(p, "transpose_x2", False))   # int8 x2 stored (e, n, k)
        self.group_list = to_device(p.group_list.astype(np.int64), dev)
        self.scale = to_device(p.scale, dev) if with_optional else None
        # a uint16 scale array holds bf16 bits
        self.scale_type = QGMM_SCALE_BF16 if p.scale is not None and p.scale.dtype == np.uint16 else QGMM_SCALE_F32
        self.logit = to_device(p.logit, dev) if with_optional else None
        self.row_index = to_device(p.row_index, dev)
        self.row_index_type = QGMM_IDX_INT32 if p.row_index.dtype == np.int32 else QGMM_IDX_INT64
        self.bias = to_device(p.bias, dev) if with_optional else None
        self.shared = to_device(p.shared, dev)
        self.shared_bs = 0 if p.shared is None else p.shared.shape[0]
        self.shared_offset = p.shared_offset
        self.out = torch.empty((p.output_bs, p.n), dtype=torch.float32, device=dev)
        self._ws = {}

    def io_copy(self) -> "DeviceProblem":
        """Same problem with its own per-call buffers (activations, scales, routing,
        sharedInput, output, workspace) and the same resident weights, scale and bias,
        so that two calls can be in flight at once."""
        c = copy.copy(self)
        for name in ("x_bf16", "x1", "pts", "group_list", "logit", "row_index", "shared", "out"):
            t = getattr(self, name)
            setattr(c, name, None if t is None else torch.empty_like(t))
        c._ws = {}
        return c

    def problem(self, deterministic: bool = False):
        return make_problem(self.m, self.k, self.n, self.e, self.output_bs, weight_type=self.weight_type,
                            group_list_type=self.group_list_type, row_index_type=self.row_index_type,
                            shared_bs=self.shared_bs, shared_offset=self.shared_offset,
                            deterministic=deterministic, expected_m_per_expert=self.expected_m_per_expert,
                            scale_type=self.scale_type, transpose_x2=self.transpose_x2)

    def workspace(self, deterministic: bool = False) -> torch.Tensor:
        key = bool(deterministic)
        if key not in self._ws:
            nbytes = finalize_workspace(self.problem(deterministic))
            self._ws[key] = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws[key]

    def quantize(self, stream=None):
        if self.prologue and self.mx:
            per_token_quant_mxfp8(self.x_bf16, self.x1, self.pts, stream=stream)
        elif self.prologue:
            per_token_quant(self.x_bf16, self.x1, self.pts, stream=stream)

    def run(self, deterministic: bool = False, stream=None, out: Optional[torch.Tensor] = None,
            quantize: bool = True) -> torch.Tensor:
        if quantize:
            self.quantize(stream)
        out = self.out if out is None else out
        finalize(self.problem(deterministic), self.x1, self.x2, self.scale, self.pts, self.group_list, self.logit,
                 self.row_index, self.bias, self.shared, out, self.workspace(deterministic), stream=stream)
        return out

    def accum(self, stream=None) -> torch.Tensor:
        if self.mx:   # block-scaled f32 accumulators
            acc = torch.zeros((self.m, self.n), dtype=torch.float32, device=self.device)
            debug_accum_mx(self.problem(False), self.x1, self.pts, self.x2, self.scale, self.group_list, acc,
                           self.workspace(False), stream=stream)
            return acc
        acc = torch.zeros((self.m, self.n), dtype=torch.int32, device=self.device)
        debug_accum(self.problem(False), self.x1, self.x2, self.group_list, acc, self.workspace(False),
                    stream=stream)
        return acc

    def status(self, deterministic: bool = False, stream=None) -> int:
        return device_status(self.workspace(deterministic), stream=stream)
