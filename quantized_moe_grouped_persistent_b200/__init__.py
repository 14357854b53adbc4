"""B200 (sm_100a) fused int8 GroupedMatmul + MoeFinalizeRouting.

A thin ctypes binding over ``libqgmm.so`` (C ABI in ``include/qgmm.h``).  It
only marshals arguments: torch tensors are passed as device pointers together
with the current CUDA stream; every step of the operation runs in the
library's kernels.  There is no fallback: if the library is missing or the
device is not a B200, the calls raise.

Entry points mirror the C ABI:
    finalize_workspace(problem) -> bytes
    finalize(problem, x1, x2, ..., out, workspace)
    per_token_quant(x_bf16, x1_out, scale_out)
    debug_accum(problem, x1, x2, group_list, acc_out, workspace)
    device_status(workspace) -> QGMM_DEV_* flags
    ep_plan(world, e, send_counts, recv_counts) -> offsets of the expert-parallel dispatch
    ep_permute_rows(src, dst, src_rows, dst_rows, counts) -> a card's own chunks, one kernel
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqgmm.so")

QGMM_OK = 0
QGMM_ERR_NULL_PTR = 1
QGMM_ERR_SHAPE = 2
QGMM_ERR_DTYPE = 3
QGMM_ERR_WORKSPACE_TOO_SMALL = 4
QGMM_ERR_UNSUPPORTED = 5
QGMM_ERR_CUDA = 6
QGMM_ERR_DEVICE_INPUT = 7
QGMM_ERR_ALIGNMENT = 8
QGMM_ERR_SCRATCH_LIMIT = 9
QGMM_STATIC_SCRATCH_BYTES = 16 << 20

QGMM_W_INT8 = 0
QGMM_W_INT4_PACKED_INT32 = 1
QGMM_W_FP8_E4M3 = 2
QGMM_W_MXFP4 = 3
QGMM_IDX_INT64 = 0
QGMM_IDX_INT32 = 1
QGMM_GROUP_CUMSUM = 0
QGMM_GROUP_COUNTS = 1
QGMM_SCALE_F32 = 0
QGMM_SCALE_BF16 = 1

QGMM_DEV_GROUP_NEGATIVE = 1 << 0
QGMM_DEV_GROUP_NOT_MONOTONE = 1 << 1
QGMM_DEV_GROUP_TOTAL_GT_M = 1 << 2
QGMM_DEV_ROW_INDEX_RANGE = 1 << 3
QGMM_DEV_TIMEOUT = 1 << 4

EXPORTS = ("qgmm_finalize_workspace", "qgmm_finalize_launches", "qgmm_plan", "qgmm_finalize", "qgmm_finalize_profiled",
           "qgmm_per_token_quant", "qgmm_per_token_quant_mxfp8", "qgmm_debug_accum", "qgmm_debug_accum_mx",
           "qgmm_device_status",
           "qgmm_finalize_static_scratch", "qgmm_ep_plan", "qgmm_ep_permute_rows", "qgmm_status_string")


class QgmmProblem(C.Structure):
    """Mirror of ``qgmm_problem`` (same field order, natural C alignment)."""
    _fields_ = [
        ("m", C.c_int64), ("k", C.c_int64), ("n", C.c_int64), ("e", C.c_int64), ("output_bs", C.c_int64),
        ("weight_type", C.c_int32), ("group_list_type", C.c_int32), ("row_index_type", C.c_int32),
        ("shared_bs", C.c_int64), ("shared_offset", C.c_int64),
        ("deterministic", C.c_int32),
        ("expected_m_per_expert", C.c_int64),
        ("scale_type", C.c_int32),
        ("transpose_x2", C.c_int32),
        ("ld_x2", C.c_int64), ("ld_sb", C.c_int64), ("ld_out", C.c_int64), ("ld_shared", C.c_int64),
    ]


class QgmmPlanInfo(C.Structure):
    """Mirror of ``qgmm_plan_info``."""
    _fields_ = [(name, C.c_int32) for name in ("tile_rows", "pair", "tail_mode", "slab_ntiles", "grid",
                                               "gemm_launches")]


class QgmmError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = status_string(code) if _lib is not None else str(code)
        super().__init__(f"{what}: {msg} (status {code})")
        self.code = code


_lib = None


def lib():
    """Load libqgmm.so (built in-tree by ``build.py``); raise if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqgmm.so not built at {LIB_PATH}; run quantized_moe_grouped_persistent_b200/build.py")
        L = C.CDLL(LIB_PATH)
        P, I64, U = C.c_void_p, C.c_int64, C.c_size_t
        L.qgmm_finalize_workspace.argtypes = [C.POINTER(QgmmProblem), C.POINTER(C.c_size_t)]
        L.qgmm_finalize_launches.argtypes = [C.POINTER(QgmmProblem), C.POINTER(C.c_int32)]
        L.qgmm_plan.argtypes = [C.POINTER(QgmmProblem), C.c_int32, C.POINTER(QgmmPlanInfo)]
        L.qgmm_finalize.argtypes = [C.POINTER(QgmmProblem), P, P, P, P, P, P, P, P, P, P, P, U, P]
        L.qgmm_finalize_profiled.argtypes = [C.POINTER(QgmmProblem), P, P, P, P, P, P, P, P, P, P, P, U, P, P, P]
        L.qgmm_per_token_quant.argtypes = [P, I64, I64, P, P, P]
        L.qgmm_per_token_quant_mxfp8.argtypes = [P, I64, I64, P, P, P]
        L.qgmm_debug_accum.argtypes = [C.POINTER(QgmmProblem), P, P, P, P, P, U, P]
        L.qgmm_debug_accum_mx.argtypes = [C.POINTER(QgmmProblem), P, P, P, P, P, P, P, U, P]
        L.qgmm_device_status.argtypes = [P, C.POINTER(C.c_uint32), P]
        L.qgmm_finalize_static_scratch.argtypes = [C.POINTER(QgmmProblem), P, P, P, P, P, P, P, P, P, P, P]
        L.qgmm_ep_plan.argtypes = [C.c_int32, C.c_int32, P, P, P, P, P, P]
        L.qgmm_ep_permute_rows.argtypes = [P, P, I64, C.c_int32, P, P, P, P]
        L.qgmm_status_string.argtypes = [C.c_int]
        L.qgmm_status_string.restype = C.c_char_p
        for name in EXPORTS[:-1]:
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().qgmm_status_string(code).decode()


def make_problem(m: int, k: int, n: int, e: int, output_bs: int, *, weight_type: int = QGMM_W_INT8,
                 group_list_type: int = QGMM_GROUP_CUMSUM, row_index_type: int = QGMM_IDX_INT64,
                 shared_bs: int = 0, shared_offset: int = 0, deterministic: bool = False,
                 expected_m_per_expert: int = 0, scale_type: int = QGMM_SCALE_F32,
                 transpose_x2: bool = False, ld_x2: int = 0, ld_sb: int = 0, ld_out: int = 0,
                 ld_shared: int = 0) -> QgmmProblem:
    return QgmmProblem(m, k, n, e, output_bs, weight_type, group_list_type, row_index_type, shared_bs,
                       shared_offset, int(bool(deterministic)), expected_m_per_expert, scale_type,
                       int(bool(transpose_x2)), ld_x2, ld_sb, ld_out, ld_shared)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != QGMM_OK:
        raise QgmmError(rc, what)


def finalize_workspace(problem: QgmmProblem) -> int:
    out = C.c_size_t(0)
    _check(lib().qgmm_finalize_workspace(C.byref(problem), C.byref(out)), "qgmm_finalize_workspace")
    return out.value


def finalize_launches(problem: QgmmProblem) -> int:
    """Number of kernels one ``finalize`` call with ``problem`` launches on the current device."""
    out = C.c_int32(0)
    _check(lib().qgmm_finalize_launches(C.byref(problem), C.byref(out)), "qgmm_finalize_launches")
    return out.value


def plan(problem: QgmmProblem, sms: int) -> dict:
    """The grouped GEMM's plan for ``problem`` on a device with ``sms`` SMs (no device needed)."""
    info = QgmmPlanInfo()
    _check(lib().qgmm_plan(C.byref(problem), int(sms), C.byref(info)), "qgmm_plan")
    return {name: getattr(info, name) for name, _ in QgmmPlanInfo._fields_}


def finalize(problem: QgmmProblem, x1, x2, scale, pertoken_scale, group_list, logit, row_index, bias,
             shared_input, out, workspace, ws_bytes: Optional[int] = None, stream=None) -> None:
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().qgmm_finalize(C.byref(problem), _ptr(x1), _ptr(x2), _ptr(scale), _ptr(pertoken_scale),
                             _ptr(group_list), _ptr(logit), _ptr(row_index), _ptr(bias), _ptr(shared_input),
                             _ptr(out), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "qgmm_finalize")


def finalize_profiled(problem: QgmmProblem, x1, x2, scale, pertoken_scale, group_list, logit, row_index, bias,
                      shared_input, out, workspace, begin_event, end_event, ws_bytes: Optional[int] = None,
                      stream=None) -> None:
    """``finalize`` that also records ``begin_event``/``end_event`` (torch.cuda.Event) around the GEMM launch.

    torch creates an event's handle on its first ``record()``; record each event once before passing it.
    """
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().qgmm_finalize_profiled(C.byref(problem), _ptr(x1), _ptr(x2), _ptr(scale), _ptr(pertoken_scale),
                                      _ptr(group_list), _ptr(logit), _ptr(row_index), _ptr(bias),
                                      _ptr(shared_input), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream),
                                      begin_event.cuda_event, end_event.cuda_event)
    _check(rc, "qgmm_finalize_profiled")


def per_token_quant(x_bf16, x1_out, scale_out, rows: Optional[int] = None, k: Optional[int] = None,
                    stream=None) -> None:
    if rows is None:
        rows, k = x_bf16.shape
    rc = lib().qgmm_per_token_quant(_ptr(x_bf16), rows, k, _ptr(x1_out), _ptr(scale_out), _stream(stream))
    _check(rc, "qgmm_per_token_quant")


def per_token_quant_mxfp8(x_bf16, q_out, sf_out, rows: Optional[int] = None, k: Optional[int] = None,
                          stream=None) -> None:
    """Per-32-group FP8 cast: E4M3 codes into ``q_out`` [rows, k], E8M0 scale codes into ``sf_out`` [rows, k/32]."""
    if rows is None:
        rows, k = x_bf16.shape
    rc = lib().qgmm_per_token_quant_mxfp8(_ptr(x_bf16), rows, k, _ptr(q_out), _ptr(sf_out), _stream(stream))
    _check(rc, "qgmm_per_token_quant_mxfp8")


def debug_accum(problem: QgmmProblem, x1, x2, group_list, acc_out, workspace, ws_bytes: Optional[int] = None,
                stream=None) -> None:
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().qgmm_debug_accum(C.byref(problem), _ptr(x1), _ptr(x2), _ptr(group_list), _ptr(acc_out),
                                _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "qgmm_debug_accum")


def debug_accum_mx(problem: QgmmProblem, x1, sfa, x2, sfb, group_list, acc_out, workspace,
                   ws_bytes: Optional[int] = None, stream=None) -> None:
    """MxA8W4 block-scaled f32 accumulators into ``acc_out`` (f32 [m, n])."""
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().qgmm_debug_accum_mx(C.byref(problem), _ptr(x1), _ptr(sfa), _ptr(x2), _ptr(sfb), _ptr(group_list),
                                   _ptr(acc_out), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "qgmm_debug_accum_mx")


def device_status(workspace, stream=None) -> int:
    """Synchronise the stream and return the QGMM_DEV_* bits of the last call on ``workspace``."""
    flags = C.c_uint32(0)
    rc = lib().qgmm_device_status(_ptr(workspace), C.byref(flags), _stream(stream))
    if rc not in (QGMM_OK, QGMM_ERR_DEVICE_INPUT):
        raise QgmmError(rc, "qgmm_device_status")
    return flags.value


def finalize_static_scratch(problem: QgmmProblem, x1, x2, scale, pertoken_scale, group_list, logit, row_index,
                            bias, shared_input, out, stream=None) -> None:
    """``finalize`` without a workspace argument, for callers that cannot allocate device memory.

    The library uses its own 16 MiB device array as scratch (see ``qgmm_finalize_static_scratch`` in
    ``include/qgmm.h``): problems whose workspace would exceed it raise with ``QGMM_ERR_SCRATCH_LIMIT``,
    the first call on a device looks up the array's address, and calls that overlap on one GPU race.
    """
    rc = lib().qgmm_finalize_static_scratch(C.byref(problem), _ptr(x1), _ptr(x2), _ptr(scale),
                                            _ptr(pertoken_scale), _ptr(group_list), _ptr(logit), _ptr(row_index),
                                            _ptr(bias), _ptr(shared_input), _ptr(out), _stream(stream))
    _check(rc, "qgmm_finalize_static_scratch")


def ep_plan(world: int, e: int, send_counts, recv_counts) -> dict:
    """Offsets of one card's expert-parallel dispatch (``qgmm_ep_plan``, a host call).

    ``send_counts`` / ``recv_counts`` are ``world * e`` row counts, chunk (card, expert)
    at ``card * e + expert``.  Returns ``send_offsets`` and ``recv_offsets`` (int64
    numpy arrays of the same shape; receive offsets are rows of the permuted,
    expert-major buffer), ``group_counts`` (rows per local expert) and ``bsk`` / ``a``.
    """
    import numpy as np
    sc = np.ascontiguousarray(np.asarray(send_counts, dtype=np.int64).reshape(-1))
    rc_ = np.ascontiguousarray(np.asarray(recv_counts, dtype=np.int64).reshape(-1))
    if sc.size != world * e or rc_.size != world * e:
        raise QgmmError(QGMM_ERR_SHAPE, "qgmm_ep_plan")
    so = np.zeros(world * e, np.int64)
    ro = np.zeros(world * e, np.int64)
    gc = np.zeros(max(e, 1), np.int64)
    tot = np.zeros(2, np.int64)
    ptr = lambda a: a.ctypes.data_as(C.c_void_p)
    _check(lib().qgmm_ep_plan(int(world), int(e), ptr(sc), ptr(rc_), ptr(so), ptr(ro), ptr(gc), ptr(tot)),
           "qgmm_ep_plan")
    return {"send_offsets": so, "recv_offsets": ro, "group_counts": gc[:e], "bsk": int(tot[0]), "a": int(tot[1])}


QGMM_EP_MAX_CHUNKS = 32


def ep_permute_rows(src, dst, src_rows, dst_rows, counts, stream=None) -> None:
    """Copy row chunks of device tensor ``src`` into ``dst`` (same row width), chunk c
    taking ``counts[c]`` rows from ``src_rows[c]`` to ``dst_rows[c]``, in one kernel
    (``qgmm_ep_permute_rows``).  The tables are host sequences of at most
    QGMM_EP_MAX_CHUNKS entries."""
    import numpy as np
    if not (src.is_cuda and dst.is_cuda):
        raise QgmmError(QGMM_ERR_UNSUPPORTED, "qgmm_ep_permute_rows: device tensors only")
    row_bytes = src.stride(0) * src.element_size()
    if dst.stride(0) * dst.element_size() != row_bytes or not src.is_contiguous() or not dst.is_contiguous():
        raise QgmmError(QGMM_ERR_SHAPE, "qgmm_ep_permute_rows")
    tabs = [np.ascontiguousarray(np.asarray(a, np.int64).reshape(-1)) for a in (src_rows, dst_rows, counts)]
    n = tabs[2].size
    if tabs[0].size != n or tabs[1].size != n:
        raise QgmmError(QGMM_ERR_SHAPE, "qgmm_ep_permute_rows")
    ptr = lambda a: a.ctypes.data_as(C.c_void_p)
    _check(lib().qgmm_ep_permute_rows(_ptr(src), _ptr(dst), row_bytes, n, ptr(tabs[0]), ptr(tabs[1]), ptr(tabs[2]),
                                      _stream(stream)), "qgmm_ep_permute_rows")
