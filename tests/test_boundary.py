"""The C ABI boundary, on the host: the library loads, exports every function
``include/qgmm.h`` and ``include/qgmm_ep.h`` declare, its struct layout matches the binding, and every
host-side check returns its documented code before anything is launched.

No test here reaches a kernel launch: each call fails a host check first.
"""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgmm.h")
EP_HEADER = os.path.join(ROOT, "include", "qgmm_ep.h")


def _declared_functions(headers=(HEADER, EP_HEADER)):
    text = "".join(open(h).read() for h in headers)
    return sorted(set(re.findall(r"^(?:qgmm_status|const char \*)\s*(qgmm_\w+)\s*\(", text, re.M)))


def test_header_declares_the_abi():
    assert _declared_functions() == sorted([
        "qgmm_finalize_workspace", "qgmm_finalize", "qgmm_finalize_profiled", "qgmm_per_token_quant",
        "qgmm_per_token_quant_mxfp8", "qgmm_debug_accum", "qgmm_debug_accum_mx", "qgmm_device_status",
        "qgmm_finalize_static_scratch",
        "qgmm_status_string",
        "qgmm_finalize_launches", "qgmm_plan", "qgmm_ep_plan", "qgmm_ep_permute_rows"])
    assert _declared_functions((EP_HEADER,)) == ["qgmm_ep_permute_rows", "qgmm_ep_plan"]


def test_library_exports_every_declared_symbol(qgmm):
    out = subprocess.run(["nm", "-D", "--defined-only", qgmm.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, re.M))
    for name in _declared_functions():
        assert name in exported, name
    # nothing but the C ABI is exported from the library's own code
    assert {s for s in exported if s.startswith("qgmm")} == set(_declared_functions())


def test_probe_library_exports_its_declared_symbol(qgmm):
    """libqgmm_probe.so (include/qgmm_probe.h): the int8 tensor-rate probe; loads and
    exports exactly what its header declares.  Argument checks need no device."""
    text = open(os.path.join(ROOT, "include", "qgmm_probe.h")).read()
    declared = sorted(set(re.findall(r"^int\s+(qgmm_\w+)\s*\(", text, re.M)))
    assert declared == ["qgmm_probe_mma_i8", "qgmm_probe_mma_i8_shape"]
    from quantized_moe_grouped_persistent_b200 import probe
    out = subprocess.run(["nm", "-D", "--defined-only", probe.PROBE_LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    assert {s for s in re.findall(r" T (\w+)$", out, re.M) if s.startswith("qgmm")} == set(declared)
    L = probe.lib()
    assert L.qgmm_probe_mma_i8(0, 10, None, None, None) == 2        # no clusters
    assert L.qgmm_probe_mma_i8(4, 0, None, None, None) == 2         # no iterations


def test_problem_struct_layout_matches_header(qgmm, tmp_path):
    src = tmp_path / "layout.c"
    src.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "qgmm.h"
#define F(x) printf(#x " %zu\\n", offsetof(qgmm_problem, x));
int main(void) {
  printf("size %zu\\n", sizeof(qgmm_problem));
  F(m) F(k) F(n) F(e) F(output_bs) F(weight_type) F(group_list_type) F(row_index_type)
  F(shared_bs) F(shared_offset) F(deterministic) F(expected_m_per_expert) F(scale_type) F(transpose_x2)
  F(ld_x2) F(ld_sb) F(ld_out) F(ld_shared)
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(l.split() for l in lines if l)
    P = qgmm.QgmmProblem
    assert int(got["size"]) == C.sizeof(P)
    for name, _ in P._fields_:
        assert int(got[name]) == getattr(P, name).offset, name


def _prob(qgmm, **kw):
    base = dict(m=64, k=256, n=512, e=4, output_bs=32)
    base.update(kw)
    args = {k: base.pop(k) for k in ("m", "k", "n", "e", "output_bs")}
    return qgmm.make_problem(args["m"], args["k"], args["n"], args["e"], args["output_bs"], **base)


def _ws(qgmm, p):
    out = C.c_size_t(0)
    rc = qgmm.lib().qgmm_finalize_workspace(C.byref(p), C.byref(out))
    return rc, out.value


def test_workspace_sizes(qgmm):
    rc, n = _ws(qgmm, _prob(qgmm))
    assert rc == qgmm.QGMM_OK and n == 256
    m, nn, obs = 64, 512, 32
    rc, n = _ws(qgmm, _prob(qgmm, deterministic=True))
    al = lambda v: (v + 255) // 256 * 256
    assert rc == qgmm.QGMM_OK
    assert n == 256 + al(m * nn * 4) + al(obs * 4) + al((obs + 1) * 4) + al(m * 4)
    assert qgmm.finalize_workspace(_prob(qgmm, m=131072, k=2048, n=7168, e=256, output_bs=16384)) == 256
    # deterministic: S per-segment histograms of output_bs int32 each,
    # S = min(1024, max(1, ceil(m / 1024)), max(1, max(2^24, m*n/16) // output_bs))
    for m, nn, obs, segs in ((131072, 7168, 16384, 128), (131072, 7168, 1, 128), (1 << 24, 256, 1 << 21, 128),
                             (1 << 21, 65536, 1 << 20, 1024), (3000, 256, 1 << 23, 2), (1 << 21, 256, 5, 1024)):
        got = qgmm.finalize_workspace(_prob(qgmm, m=m, k=128, n=nn, e=4, output_bs=obs, deterministic=True))
        assert got == 256 + al(m * nn * 4) + al(segs * obs * 4) + al((obs + 1) * 4) + al(m * 4), (m, obs)


def test_workspace_sizes_mx(qgmm):
    """QGMM_W_MXFP4 adds its scale atoms after the mode's own part: (ceil(m/128) + e) * (k/128)
    atoms for x1 and e * (n/128) * (k/128) for the weights, 512 bytes each, each part rounded
    up to 256 bytes (the formula qgmm.h gives)."""
    al = lambda v: (v + 255) // 256 * 256
    for m, k, n, e, obs in ((32768, 2048, 7168, 128, 4096), (100, 256, 256, 3, 100), (1, 128, 256, 1, 1)):
        atoms = al(((m + 127) // 128 + e) * (k // 128) * 512) + al(e * (n // 128) * (k // 128) * 512)
        p = _prob(qgmm, m=m, k=k, n=n, e=e, output_bs=obs, weight_type=qgmm.QGMM_W_MXFP4, transpose_x2=True)
        assert qgmm.finalize_workspace(p) == 256 + atoms, (m, k, n, e)
        pd = _prob(qgmm, m=m, k=k, n=n, e=e, output_bs=obs, weight_type=qgmm.QGMM_W_MXFP4, transpose_x2=True,
                   deterministic=True)
        base = qgmm.finalize_workspace(_prob(qgmm, m=m, k=k, n=n, e=e, output_bs=obs, deterministic=True))
        assert qgmm.finalize_workspace(pd) == base + atoms, (m, k, n, e)


@pytest.mark.parametrize("kw,code", [
    (dict(m=0), "SHAPE"), (dict(m=(1 << 24) + 1), "SHAPE"),
    (dict(k=100), "SHAPE"), (dict(k=64), "SHAPE"), (dict(k=65536 + 128), "SHAPE"),
    (dict(n=128), "SHAPE"), (dict(n=300), "SHAPE"), (dict(n=7168 + 128), "SHAPE"),
    (dict(e=0), "SHAPE"), (dict(e=1025), "SHAPE"), (dict(output_bs=0), "SHAPE"),
    (dict(shared_bs=33), "SHAPE"), (dict(shared_bs=8, shared_offset=25), "SHAPE"),
    (dict(shared_offset=-1), "SHAPE"), (dict(expected_m_per_expert=-1), "SHAPE"),
    (dict(weight_type=4), "DTYPE"), (dict(weight_type=-1), "DTYPE"), (dict(group_list_type=2), "DTYPE"), (dict(row_index_type=5), "DTYPE"),
    (dict(scale_type=2), "DTYPE"), (dict(scale_type=-1), "DTYPE"),
    (dict(transpose_x2=1, weight_type=1), "UNSUPPORTED"), (dict(weight_type=3), "UNSUPPORTED"),
])
def test_stage_one_rejects(qgmm, kw, code):
    rc, _ = _ws(qgmm, _prob(qgmm, **kw))
    assert rc == getattr(qgmm, "QGMM_ERR_" + code)


def test_stage_one_rejects_unknown_layout_flag(qgmm):
    p = _prob(qgmm)
    p.transpose_x2 = 2                       # the struct field itself: the binding passes 0 or 1
    assert _ws(qgmm, p)[0] == qgmm.QGMM_ERR_SHAPE
    p.transpose_x2 = 1
    assert _ws(qgmm, p)[0] == qgmm.QGMM_OK


def test_stage_one_accepts_page_limits(qgmm):
    for kw in (dict(m=1), dict(m=131072, k=2048, n=7168, e=256), dict(e=1024), dict(k=65536),
               dict(shared_bs=32, shared_offset=0), dict(shared_bs=8, shared_offset=24)):
        assert _ws(qgmm, _prob(qgmm, **kw))[0] == qgmm.QGMM_OK, kw


def test_null_arguments(qgmm):
    L = qgmm.lib()
    assert L.qgmm_finalize_workspace(None, None) == qgmm.QGMM_ERR_NULL_PTR
    p = _prob(qgmm)
    assert L.qgmm_finalize_workspace(C.byref(p), None) == qgmm.QGMM_ERR_NULL_PTR
    fake = 1 << 20  # never dereferenced: every call below fails a host check
    args = [fake, fake, None, None, fake, None, None, None, None, fake, fake, 256, None]
    for idx in (0, 1, 4, 9, 10):   # x1, x2, group_list, out, workspace
        a = list(args)
        a[idx] = None
        assert L.qgmm_finalize(C.byref(p), *a) == qgmm.QGMM_ERR_NULL_PTR, idx
    ps = _prob(qgmm, shared_bs=4)
    assert L.qgmm_finalize(C.byref(ps), *args) == qgmm.QGMM_ERR_NULL_PTR   # shared rows without a pointer
    assert L.qgmm_finalize(None, *args) == qgmm.QGMM_ERR_NULL_PTR
    assert L.qgmm_per_token_quant(None, 4, 64, fake, fake, None) == qgmm.QGMM_ERR_NULL_PTR
    assert L.qgmm_debug_accum(C.byref(p), fake, fake, None, fake, fake, 256, None) == qgmm.QGMM_ERR_NULL_PTR
    assert L.qgmm_device_status(None, None, None) == qgmm.QGMM_ERR_NULL_PTR
    assert L.qgmm_finalize_profiled(C.byref(p), *args, None, None) == qgmm.QGMM_ERR_NULL_PTR


def test_alignment_and_workspace_checks(qgmm):
    L = qgmm.lib()
    p = _prob(qgmm)
    a16 = 1 << 20
    for idx in (0, 1, 9):   # x1, x2, out misaligned
        a = [a16, a16, None, None, a16, None, None, None, None, a16, a16, 256, None]
        a[idx] = a16 + 8
        assert L.qgmm_finalize(C.byref(p), *a) == qgmm.QGMM_ERR_ALIGNMENT, idx
    a = [a16, a16, a16 + 4, None, a16, None, None, None, None, a16, a16, 256, None]   # scale misaligned
    assert L.qgmm_finalize(C.byref(p), *a) == qgmm.QGMM_ERR_ALIGNMENT
    a = [a16, a16, None, None, a16, None, None, None, None, a16, a16 + 16, 256, None]  # workspace not 256-aligned
    assert L.qgmm_finalize(C.byref(p), *a) == qgmm.QGMM_ERR_ALIGNMENT
    a = [a16, a16, None, None, a16, None, None, None, None, a16, a16, 255, None]
    assert L.qgmm_finalize(C.byref(p), *a) == qgmm.QGMM_ERR_WORKSPACE_TOO_SMALL
    pd = _prob(qgmm, deterministic=True)
    a = [a16, a16, None, None, a16, None, None, None, None, a16, a16, 256, None]
    assert L.qgmm_finalize(C.byref(pd), *a) == qgmm.QGMM_ERR_WORKSPACE_TOO_SMALL
    assert L.qgmm_debug_accum(C.byref(p), a16, a16, a16, a16 + 4, a16, 256, None) == qgmm.QGMM_ERR_ALIGNMENT
    assert L.qgmm_debug_accum(C.byref(p), a16, a16, a16, a16, a16, 128, None) == qgmm.QGMM_ERR_WORKSPACE_TOO_SMALL


def test_per_token_quant_host_checks(qgmm):
    L = qgmm.lib()
    a16 = 1 << 20
    assert L.qgmm_per_token_quant(a16, 4, 12, a16, a16, None) == qgmm.QGMM_ERR_SHAPE   # k % 8
    assert L.qgmm_per_token_quant(a16, 0, 64, a16, a16, None) == qgmm.QGMM_ERR_SHAPE
    assert L.qgmm_per_token_quant(a16 + 2, 4, 64, a16, a16, None) == qgmm.QGMM_ERR_ALIGNMENT


def test_status_strings(qgmm):
    for code in range(10):
        s = qgmm.status_string(code)
        assert s and s != "unknown status"
    assert qgmm.status_string(99) == "unknown status"


def test_binding_raises_without_library(tmp_path, monkeypatch):
    import quantized_moe_grouped_persistent_b200 as q
    monkeypatch.setattr(q, "_lib", None)
    monkeypatch.setattr(q, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        q.lib()


# --- the planner, through qgmm_plan (host only: no device) --------------------
def _plan(qgmm, m, e, n=7168, k=2048, output_bs=None, sms=148, **kw):
    return qgmm.plan(qgmm.make_problem(m, k, n, e, output_bs or max(1, m // 8), **kw), sms)


@pytest.mark.parametrize("rows_per_expert,tile_rows", [(1, 16), (16, 16), (17, 32), (32, 32), (33, 64), (64, 64),
                                                      (65, 128), (4096, 128)])
def test_plan_tile_rows_follow_rows_per_expert(qgmm, rows_per_expert, tile_rows):
    e = 8
    assert _plan(qgmm, rows_per_expert * e, e)["tile_rows"] == tile_rows
    # the tuning hint (page 1: tuningConfigOptional[0]) replaces m / e
    assert _plan(qgmm, 4096 * e, e, expected_m_per_expert=rows_per_expert)["tile_rows"] == tile_rows


def test_plan_pairs_for_full_height_int8_tiles(qgmm, monkeypatch):
    monkeypatch.delenv("QGMM_PAIR", raising=False)
    monkeypatch.delenv("QGMM_PAIR_W4", raising=False)
    assert _plan(qgmm, 131072, 256)["pair"] == 1
    assert _plan(qgmm, 128, 256)["pair"] == 0                              # decode: 16-row tiles
    assert _plan(qgmm, 32768, 128, weight_type=qgmm.QGMM_W_INT4_PACKED_INT32)["pair"] == 0
    monkeypatch.setenv("QGMM_PAIR_W4", "1")
    assert _plan(qgmm, 32768, 128, weight_type=qgmm.QGMM_W_INT4_PACKED_INT32)["pair"] == 1
    monkeypatch.setenv("QGMM_PAIR", "0")
    assert _plan(qgmm, 131072, 256)["pair"] == 0


@pytest.mark.parametrize("m,e,mode", [(4096, 32, 2), (8192, 32, 2), (16384, 32, 2), (32768, 32, 1), (65536, 32, 1),
                                      (32768, 256, 1), (131072, 256, 1)])
def test_plan_tail_mode_by_wave_counts(qgmm, monkeypatch, m, e, mode):
    """Tails as M=128 pair tiles when e*28 tail tiles fit 8 waves of 148 SMs and
    m/256*28 pair tiles fit 32 waves of 74 pairs; else the single-CTA tail launch."""
    monkeypatch.delenv("QGMM_PAIR_TAILS", raising=False)
    p = _plan(qgmm, m, e)
    assert p["pair"] == 1                                  # >= 128 rows per expert: CTA pairs
    assert p["tail_mode"] == mode
    assert p["gemm_launches"] == (2 if mode == 1 else 1)
    monkeypatch.setenv("QGMM_PAIR_TAILS", "0")
    assert _plan(qgmm, m, e)["tail_mode"] == 0 and _plan(qgmm, m, e)["gemm_launches"] == 1


def test_plan_slab_width(qgmm, monkeypatch):
    """Atomic combine: the widest slab (a divisor of n/256 tiles) within half of x1's
    bytes, clamped to [32 MB, 128 MB]; the deterministic mode writes rows, no slab."""
    monkeypatch.delenv("QGMM_SLAB_NTILES", raising=False)
    assert _plan(qgmm, 131072, 256, output_bs=16384)["slab_ntiles"] == 7        # 7 x 16.8 MB <= 128 MB
    assert _plan(qgmm, 32768, 128, output_bs=4096)["slab_ntiles"] == 7          # 7 x 4.2 MB <= 33.5 MB
    assert _plan(qgmm, 8192, 32, output_bs=1024)["slab_ntiles"] == 28           # 28 x 1 MB <= 32 MB
    assert _plan(qgmm, 131072, 256, output_bs=16384, deterministic=True)["slab_ntiles"] == 28
    monkeypatch.setenv("QGMM_SLAB_NTILES", "4")
    assert _plan(qgmm, 131072, 256, output_bs=16384)["slab_ntiles"] == 4
    monkeypatch.setenv("QGMM_SLAB_NTILES", "5")                                 # not a divisor of 28: ignored
    assert _plan(qgmm, 131072, 256, output_bs=16384)["slab_ntiles"] == 7


def test_plan_grid_and_arguments(qgmm):
    assert _plan(qgmm, 131072, 256)["grid"] == 148                              # one CTA per SM, in pairs
    assert _plan(qgmm, 131072, 256, sms=132)["grid"] == 132
    tiny = _plan(qgmm, 64, 4, n=512, k=256, output_bs=32)                        # 16-row tiles, 2 n-tiles
    assert tiny["pair"] == 0 and tiny["grid"] == (64 // 16 + 4) * 2
    p = qgmm.make_problem(64, 256, 512, 4, 32)
    assert qgmm.lib().qgmm_plan(C.byref(p), 1, C.byref(qgmm.QgmmPlanInfo())) == qgmm.QGMM_ERR_SHAPE
    assert qgmm.lib().qgmm_plan(C.byref(p), 148, None) == qgmm.QGMM_ERR_NULL_PTR
    assert qgmm.lib().qgmm_plan(None, 148, C.byref(qgmm.QgmmPlanInfo())) == qgmm.QGMM_ERR_NULL_PTR


def test_plan_tile_rows_override(qgmm, monkeypatch):
    """QGMM_TILE_ROWS replaces the planner's tile height (16/32/64/128 only); CTA pairs
    need 128-row tiles."""
    monkeypatch.setenv("QGMM_TILE_ROWS", "64")
    p = _plan(qgmm, 131072, 256)
    assert p["tile_rows"] == 64 and p["pair"] == 0 and p["gemm_launches"] == 1
    monkeypatch.setenv("QGMM_TILE_ROWS", "48")                 # not a tile height: ignored
    assert _plan(qgmm, 131072, 256)["tile_rows"] == 128
    monkeypatch.setenv("QGMM_TILE_ROWS", "128")
    assert _plan(qgmm, 128, 256)["tile_rows"] == 128 and _plan(qgmm, 128, 256)["pair"] == 1
