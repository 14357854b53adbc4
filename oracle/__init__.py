"""CPU oracle for the fused int8 GroupedMatmul + MoeFinalizeRouting op.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference leg may import this package.  It shares
no code with the CUDA library and never imports it.

The arithmetic lives in ``qgmm_oracle.c`` (plain C, IEEE float, no FMA
contraction); this module only marshals numpy arrays.  Function-by-function
citations are in the C file's header.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import numpy as np

from .build import build as _build

QO_OK = 0
QO_ERR_NEGATIVE_COUNT = 1
QO_ERR_NOT_MONOTONE = 2
QO_ERR_TOTAL_GT_M = 3
QO_ERR_BAD_ROW_INDEX = 4
QO_ERR_ACC_OVERFLOW = 5
QO_ERR_ARG = 6


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what}: code {code}")
        self.code = code


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = C.CDLL(path)
        P, I64, I32 = C.c_void_p, C.c_int64, C.c_int
        L.qo_group_offsets.argtypes = [P, I64, I32, I64, P]
        L.qo_accum.argtypes = [P, P, I32, I64, I64, I64, I64, P, I32, P, I64, P, I32]
        L.qo_finalize.argtypes = [P, P, I32, I64, I64, I64, I64, P, I32, P, P, P, P, P, I32,
                                  P, I64, I64, I64, P, I64, P, P, P, I32]
        L.qo_per_token_quant.argtypes = [P, I64, I64, P, P]
        L.qo_bf16_to_f32.argtypes = [P, I64, P]
        L.qo_per_token_quant_mxfp8.argtypes = [P, I64, I64, P, P]
        L.qo_accum_f8.argtypes = [P, P, I64, I64, I64, I64, P, I32, P, I64, P, P, I32]
        L.qo_accum_f8.restype = C.c_int
        L.qo_accum_mx.argtypes = [P, P, P, P, I64, I64, I64, I64, P, I32, P, I64, P, P, I32]
        L.qo_accum_mx.restype = C.c_int
        L.qo_finalize_mx.argtypes = [P, P, P, P, I64, I64, I64, I64, P, I32, P, P, P, I32, P, I64, I64, I64,
                                     P, I64, P, P, P, I32]
        L.qo_finalize_mx.restype = C.c_int
        L.qo_e2m1_decode.argtypes = [C.c_uint8]
        L.qo_e2m1_decode.restype = C.c_double
        L.qo_e8m0_decode.argtypes = [C.c_uint8]
        L.qo_e8m0_decode.restype = C.c_double
        for f in (L.qo_group_offsets, L.qo_accum, L.qo_finalize, L.qo_per_token_quant, L.qo_bf16_to_f32,
                  L.qo_per_token_quant_mxfp8):
            f.restype = C.c_int
        L.qo_e4m3_encode.argtypes = [C.c_float]
        L.qo_e4m3_encode.restype = C.c_uint8
        L.qo_e4m3_decode.argtypes = [C.c_uint8]
        L.qo_e4m3_decode.restype = C.c_float
        _lib = L
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else C.c_void_p(a.ctypes.data)


def _c(a: Optional[np.ndarray], dtype) -> Optional[np.ndarray]:
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def group_offsets(group_list: np.ndarray, group_list_type: int, m: int) -> np.ndarray:
    gl = _c(group_list, np.int64)
    off = np.zeros(gl.shape[0] + 1, np.int64)
    rc = lib().qo_group_offsets(_ptr(gl), gl.shape[0], group_list_type, m, _ptr(off))
    if rc:
        raise OracleError(rc, "group_offsets")
    return off


def _weights(x2: np.ndarray, weight: str, transpose_x2: bool = False):
    """The C oracle's weight layout, (e, k, n) int8 / E4M3 bytes or (e, k, n/8) int32.
    A transposed x2 (page 1, full-quant scenario: (e, n, k)) is swapped back to it."""
    if weight == "int8":
        return _c(np.swapaxes(x2, 1, 2) if transpose_x2 else x2, np.int8), 0
    if weight == "fp8":
        return _c(np.swapaxes(x2, 1, 2) if transpose_x2 else x2, np.uint8), 2
    if transpose_x2:
        raise ValueError("transposed x2 is int8 only")
    return _c(x2, np.int32), 1


def accum(x1, x2, group_list, group_list_type: int, weight: str = "int8",
          rows: Optional[np.ndarray] = None, threads: Optional[int] = None,
          transpose_x2: bool = False) -> np.ndarray:
    """Exact int32 accumulators ``x1[i] @ W[g(i)]`` for source rows ``rows`` (default all).
    FP8 (E4M3 bytes): use ``accum_f8``."""
    if weight == "fp8":
        return accum_f8(x1, x2, group_list, group_list_type, rows=rows, threads=threads,
                        transpose_x2=transpose_x2)[0]
    x1 = _c(x1, np.int8)
    w, wt = _weights(x2, weight, transpose_x2)
    m, k = x1.shape
    e = w.shape[0]
    n = w.shape[2] * (8 if wt else 1)
    r = _c(rows, np.int64)
    nrows = m if r is None else r.shape[0]
    out = np.zeros((nrows, n), np.int32)
    rc = lib().qo_accum(_ptr(x1), _ptr(w), wt, m, k, n, e, _ptr(_c(group_list, np.int64)),
                        group_list_type, _ptr(r), nrows, _ptr(out), threads or default_threads())
    if rc:
        raise OracleError(rc, "accum")
    return out


def accum_f8(x1, x2, group_list, group_list_type: int, rows: Optional[np.ndarray] = None,
             threads: Optional[int] = None, transpose_x2: bool = False):
    """E4M3 operands (uint8 codes): exact double accumulators and the sums of
    |products| for source rows ``rows`` (default all)."""
    x1 = _c(x1, np.uint8)
    w, _ = _weights(x2, "fp8", transpose_x2)
    m, k = x1.shape
    e, n = w.shape[0], w.shape[2]
    r = _c(rows, np.int64)
    nrows = m if r is None else r.shape[0]
    acc = np.zeros((nrows, n), np.float64)
    mag = np.zeros((nrows, n), np.float64)
    rc = lib().qo_accum_f8(_ptr(x1), _ptr(w), m, k, n, e, _ptr(_c(group_list, np.int64)), group_list_type,
                           _ptr(r), nrows, _ptr(acc), _ptr(mag), threads or default_threads())
    if rc:
        raise OracleError(rc, "accum_f8")
    return acc, mag


def finalize(x1, x2, group_list, group_list_type: int, *, weight: str = "int8",
             scale=None, pertoken_scale=None, logit=None, bias=None, row_index=None,
             shared=None, shared_offset: int = 0, output_bs: Optional[int] = None,
             dest_rows: Optional[np.ndarray] = None, want64: bool = True, want32: bool = True,
             threads: Optional[int] = None, transpose_x2: bool = False):
    """The op's output rows ``dest_rows`` (default all ``output_bs`` rows).

    ``scale`` is f32, or uint16 holding bf16 bits (widened exactly by the C oracle).

    Returns ``(out64, sabs64, out32)``: double value; per element the magnitude
    that bounds rounding error, |sharedInput| + sum over contributions of
    (|acc*scale*pts| + |bias|) * |logit|; and the f32 value in the fixed
    summation order (None if not asked).
    """
    if scale is not None and scale.dtype == np.uint16:
        scale = bf16_to_f32(scale)
    x1 = _c(x1, np.uint8 if weight == "fp8" else np.int8)
    w, wt = _weights(x2, weight, transpose_x2)
    m, k = x1.shape
    e = w.shape[0]
    n = w.shape[2] * (8 if wt == 1 else 1)
    if output_bs is None:
        output_bs = m
    ri = None
    rit = 0
    if row_index is not None:
        if row_index.dtype == np.int32:
            ri, rit = _c(row_index, np.int32), 1
        else:
            ri, rit = _c(row_index, np.int64), 0
    sh = _c(shared, np.uint16)
    shared_bs = 0 if sh is None else sh.shape[0]
    d = _c(dest_rows, np.int64)
    nd = output_bs if d is None else d.shape[0]
    out64 = np.zeros((nd, n), np.float64) if want64 else None
    sabs = np.zeros((nd, n), np.float64) if want64 else None
    out32 = np.zeros((nd, n), np.float32) if want32 else None
    rc = lib().qo_finalize(_ptr(x1), _ptr(w), wt, m, k, n, e, _ptr(_c(group_list, np.int64)),
                           group_list_type, _ptr(_c(scale, np.float32)),
                           _ptr(_c(pertoken_scale, np.float32)), _ptr(_c(logit, np.float32)),
                           _ptr(_c(bias, np.float32)), _ptr(ri), rit, _ptr(sh), shared_bs,
                           shared_offset, output_bs, _ptr(d), nd, _ptr(out64), _ptr(sabs),
                           _ptr(out32), threads or default_threads())
    if rc:
        raise OracleError(rc, "finalize")
    return out64, sabs, out32


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bits (uint16, any shape) -> f32 values, exactly."""
    b = _c(bits, np.uint16)
    out = np.zeros(b.shape, np.float32)
    rc = lib().qo_bf16_to_f32(_ptr(b), b.size, _ptr(out))
    if rc:
        raise OracleError(rc, "bf16_to_f32")
    return out


def per_token_quant(x_bf16: np.ndarray):
    """bf16 bits [rows, k] -> (int8 [rows, k], f32 pts [rows])."""
    x = _c(x_bf16, np.uint16)
    rows, k = x.shape
    q = np.zeros((rows, k), np.int8)
    pts = np.zeros(rows, np.float32)
    rc = lib().qo_per_token_quant(_ptr(x), rows, k, _ptr(q), _ptr(pts))
    if rc:
        raise OracleError(rc, "per_token_quant")
    return q, pts


def problem_finalize(p, *, x1=None, pertoken_scale=None, dest_rows=None, want64=True,
                     want32=True, threads=None):
    """Run ``finalize`` on a ``synth.Problem`` (x1/pts override for prologue workloads)."""
    return finalize(p.x1 if x1 is None else x1, p.x2, p.group_list, p.group_list_type,
                    weight=p.weight, scale=p.scale,
                    pertoken_scale=p.pertoken_scale if pertoken_scale is None else pertoken_scale,
                    logit=p.logit, bias=p.bias, row_index=p.row_index, shared=p.shared,
                    shared_offset=p.shared_offset, output_bs=p.output_bs, dest_rows=dest_rows,
                    want64=want64, want32=want32, threads=threads,
                    transpose_x2=bool(getattr(p, "transpose_x2", False)))


def e4m3_encode(v: float) -> int:
    """FLOAT8 E4M3FN code of an f32 value: round to nearest even, saturating at 448."""
    return int(lib().qo_e4m3_encode(float(v)))


def e4m3_decode(code: int) -> float:
    """The value of an E4M3FN code (NaN for 0x7F / 0xFF)."""
    return float(lib().qo_e4m3_decode(int(code)))


def per_token_quant_mxfp8(x_bf16: np.ndarray):
    """bf16 bits [rows, k] (k % 32 == 0) -> (E4M3 codes uint8 [rows, k], E8M0 scale
    codes uint8 [rows, k / 32]); x ~= decode(q) * 2^(sf - 127) per group of 32."""
    x = _c(x_bf16, np.uint16)
    rows, k = x.shape
    q = np.zeros((rows, k), np.uint8)
    sf = np.zeros((rows, k // 32), np.uint8)
    rc = lib().qo_per_token_quant_mxfp8(_ptr(x), rows, k, _ptr(q), _ptr(sf))
    if rc:
        raise OracleError(rc, "per_token_quant_mxfp8")
    return q, sf


def e2m1_decode(nibble: int) -> float:
    """The value of an FP4 E2M1 code (low 4 bits)."""
    return float(lib().qo_e2m1_decode(int(nibble) & 0xF))


def e8m0_decode(code: int) -> float:
    """The value of an E8M0 scale code: 2^(code - 127), NaN for 0xFF."""
    return float(lib().qo_e8m0_decode(int(code)))


def accum_mx(x1, sfa, x2, sfb, group_list, group_list_type: int, rows=None, threads=None):
    """MxA8W4 accumulators: x1 E4M3 uint8 [m, k], sfa E8M0 [m, k/32], x2 E2M1 pairs
    uint8 [e, n, k/2] (lower k in the low nibble), sfb E8M0 [e, n, k/32].  Returns
    (acc, mag) in double for source rows ``rows`` (default all)."""
    x1, sfa, x2, sfb = (_c(a, np.uint8) for a in (x1, sfa, x2, sfb))
    m, k = x1.shape
    e, n = x2.shape[0], x2.shape[1]
    r = _c(rows, np.int64)
    nrows = m if r is None else r.shape[0]
    acc = np.zeros((nrows, n), np.float64)
    mag = np.zeros((nrows, n), np.float64)
    rc = lib().qo_accum_mx(_ptr(x1), _ptr(sfa), _ptr(x2), _ptr(sfb), m, k, n, e, _ptr(_c(group_list, np.int64)),
                           group_list_type, _ptr(r), nrows, _ptr(acc), _ptr(mag), threads or default_threads())
    if rc:
        raise OracleError(rc, "accum_mx")
    return acc, mag


def finalize_mx(x1, sfa, x2, sfb, group_list, group_list_type: int, *, logit=None, bias=None, row_index=None,
                shared=None, shared_offset: int = 0, output_bs: Optional[int] = None, dest_rows=None,
                want64: bool = True, want32: bool = True, threads: Optional[int] = None):
    """MxA8W4 output rows (see ``accum_mx``): (acc + bias) * logit combined by row index.
    Returns (out64, sabs64, out32) as ``finalize`` does."""
    x1, sfa, x2, sfb = (_c(a, np.uint8) for a in (x1, sfa, x2, sfb))
    m, k = x1.shape
    e, n = x2.shape[0], x2.shape[1]
    if output_bs is None:
        output_bs = m
    ri, rit = None, 0
    if row_index is not None:
        ri, rit = (_c(row_index, np.int32), 1) if row_index.dtype == np.int32 else (_c(row_index, np.int64), 0)
    sh = _c(shared, np.uint16)
    shared_bs = 0 if sh is None else sh.shape[0]
    d = _c(dest_rows, np.int64)
    nd = output_bs if d is None else d.shape[0]
    out64 = np.zeros((nd, n), np.float64) if want64 else None
    sabs = np.zeros((nd, n), np.float64) if want64 else None
    out32 = np.zeros((nd, n), np.float32) if want32 else None
    rc = lib().qo_finalize_mx(_ptr(x1), _ptr(sfa), _ptr(x2), _ptr(sfb), m, k, n, e, _ptr(_c(group_list, np.int64)),
                              group_list_type, _ptr(_c(logit, np.float32)), _ptr(_c(bias, np.float32)), _ptr(ri),
                              rit, _ptr(sh), shared_bs, shared_offset, output_bs, _ptr(d), nd, _ptr(out64),
                              _ptr(sabs), _ptr(out32), threads or default_threads())
    if rc:
        raise OracleError(rc, "finalize_mx")
    return out64, sabs, out32
