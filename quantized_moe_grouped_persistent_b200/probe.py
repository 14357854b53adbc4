"""Binding of libqgmm_probe.so (C ABI in ``include/qgmm_probe.h``): the int8
tensor-core rate of this device, measured by back-to-back CTA-pair
``tcgen05.mma.kind::i8`` with no memory traffic.  Marshalling and CUDA-event
timing only; the work runs in the probe kernel."""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
PROBE_LIB_PATH = os.path.join(HERE, "libqgmm_probe.so")
MACS_PER_MMA = 256 * 256 * 32          # one cta_group::2 kind::i8 MMA, M = 256, N = 256, K = 32 (scaled by N/256)

_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(PROBE_LIB_PATH):
            raise ImportError(f"libqgmm_probe.so not built at {PROBE_LIB_PATH}; run "
                              "quantized_moe_grouped_persistent_b200/build.py")
        L = C.CDLL(PROBE_LIB_PATH)
        L.qgmm_probe_mma_i8.argtypes = [C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]
        L.qgmm_probe_mma_i8.restype = C.c_int
        L.qgmm_probe_mma_i8_shape.argtypes = [C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                                              C.c_void_p]
        L.qgmm_probe_mma_i8_shape.restype = C.c_int
        _lib = L
    return _lib


def mma_i8_rate(iters: int = 16384, launches: int = 20, warmup: int = 3, clusters: int = 0, n: int = 256,
                a_mn_major: bool = False) -> dict:
    """Median int8 rate over `launches` timed launches of the probe on every SM pair
    (or `clusters` pairs): int ops per second, MACs per clock per SM from the SM
    clock CTA 0 saw, and that clock.  `n` and `a_mn_major` select the tile form."""
    import torch
    if clusters <= 0:
        clusters = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count // 2
    stream = torch.cuda.current_stream()
    clk = torch.zeros(2, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def launch():
        rc = lib().qgmm_probe_mma_i8_shape(clusters, iters, n, int(a_mn_major), clk.data_ptr(), status.data_ptr(),
                                           stream.cuda_stream)
        if rc:
            raise RuntimeError(f"qgmm_probe_mma_i8 returned {rc}")

    for _ in range(warmup):
        launch()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(launches + 1)]
    ev[0].record(stream)
    for i in range(launches):
        launch()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    if int(status.item()):
        raise RuntimeError("the probe's bounded wait ran out")
    ms = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(launches))
    med = ms[len(ms) // 2]
    macs = clusters * iters * MACS_PER_MMA * n // 256
    cycles, ns = (int(v) for v in clk.cpu().tolist())
    return {"tops": 2.0 * macs / (med * 1e-3) / 1e12, "tops_best": 2.0 * macs / (ms[0] * 1e-3) / 1e12,
            "ms_median": med, "mac_per_clk_per_sm": macs / (2 * clusters) / max(cycles, 1),
            "sm_ghz": cycles / max(ns, 1), "clusters": clusters, "iters": iters, "launches": launches}
