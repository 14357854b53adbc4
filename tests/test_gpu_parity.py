"""GPU parity: the CUDA path against the CPU oracle, through the C ABI.

Bars (from the op's arithmetic):
  - int32 accumulators (qgmm_debug_accum), per-token quant codes and scales,
    and scatter indexing: bit-exact;
  - deterministic mode: bitwise equal to the oracle's fixed-order f32 result,
    and within 1e-5 of the double-precision value;
  - atomic mode: within 2e-5 of the double-precision value.
The float error of an output element is |gpu - ref| / sum|terms| (the shared
value and every contribution added into that element), the relative error of
a sum measured against its condition; where nothing is added the element must
be exactly zero.
"""
import json
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

DET_TOL = 1e-5
ATOMIC_TOL = 2e-5
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sum_rel_err(gpu: np.ndarray, ref64: np.ndarray, sabs: np.ndarray) -> float:
    den = np.where(sabs > 0, sabs, 1.0)
    err = np.abs(gpu.astype(np.float64) - ref64) / den
    return float(err.max()) if err.size else 0.0


PLAIN_FLOOR = 0.1


def plain_rel_err(gpu: np.ndarray, ref64: np.ndarray, sabs: np.ndarray) -> float:
    """max |gpu - ref| / |ref| over the elements whose value is at least PLAIN_FLOOR of
    their term magnitude (cancellation below 10x).  There the f32 pipeline's bound,
    about (5 + additions) * 2^-24 of sum|terms|, stays under 1e-5 of |ref| for up to
    ~15 additions per element, so the plain error meets the same bars."""
    sel = (sabs > 0) & (np.abs(ref64) >= PLAIN_FLOOR * sabs)
    if not sel.any():
        return 0.0
    return float((np.abs(gpu.astype(np.float64)[sel] - ref64[sel]) / np.abs(ref64[sel])).max())


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


# --------------------------------------------------------------------------- worked example
def _padded_worked_example():
    from types import SimpleNamespace
    g = json.load(open(os.path.join(GOLDEN, "per_token_worked_example.json")))
    k, n = 128, 256
    x1 = np.zeros((2, k), np.int8)
    x1[:, :2] = np.array(g["x"], np.int8)
    x2 = np.zeros((1, k, n), np.int8)
    x2[0, :2, :3] = np.array(g["weight"], np.int8)
    scale = np.ones((1, n), np.float32)
    scale[0, :3] = g["deqScale"]
    return SimpleNamespace(name="worked", tokens=2, topk=1, m=2, e=1, k=k, n=n, output_bs=2, group_list_type=1,
                           weight="int8", x1=x1, x_bf16=None, x2=x2, scale=scale,
                           pertoken_scale=np.array(g["perTokenScale"], np.float32),
                           group_list=np.array([2], np.int64), counts=np.array([2]), logit=np.ones(2, np.float32),
                           row_index=np.array([0, 1], np.int64), bias=None, shared=None, shared_offset=0), \
        np.array(g["output"], np.float64)


@pytest.mark.parametrize("deterministic", [True, False])
def test_worked_example_on_gpu(dev, deterministic):
    p, expect = _padded_worked_example()
    d = dev.DeviceProblem(p)
    out = d.run(deterministic=deterministic).cpu().numpy()
    np.testing.assert_array_equal(out[:, :3].astype(np.float64), expect)
    assert (out[:, 3:] == 0).all()
    assert d.status(deterministic) == 0
    acc = d.accum().cpu().numpy()
    np.testing.assert_array_equal(acc[:, :3], [[9, 12, 15], [19, 26, 33]])


# --------------------------------------------------------------------------- small cases
SMALL = {
    # name: (config recipe, overrides)
    "tiny": ("tiny", {}),
    "mid_small": ("mid_prefill", dict(tokens=96, e=8, k=512, n=768)),
    "decode_small": ("decode", dict(tokens=16, e=64, k=256, n=512)),
    "large_small": ("large_prefill", dict(tokens=160, e=16, k=384, n=512)),
    "w4a8_small": ("w4a8_prologue", dict(tokens=48, e=8, k=256, n=512)),
}


def _small(problem_cache, key):
    name, kw = SMALL[key]
    return problem_cache(name, **kw)


def _oracle_inputs(oracle, d):
    """x1 / pts the oracle should use: for prologue workloads, its own quantisation."""
    p = d.p
    if p.x1 is not None:
        return p.x1, p.pertoken_scale
    return oracle.per_token_quant(p.x_bf16)


@pytest.mark.parametrize("key", list(SMALL))
@pytest.mark.parametrize("hint", [0, 1, 24, 40, 100])
def test_accumulators_bit_exact(dev, oracle, problem_cache, key, hint):
    p = _small(problem_cache, key)
    d = dev.DeviceProblem(p, expected_m_per_expert=hint)
    d.quantize()
    x1, _ = _oracle_inputs(oracle, d)
    acc = d.accum().cpu().numpy()
    ref = oracle.accum(x1, p.x2, p.group_list, p.group_list_type, weight=p.weight)
    total = int(p.counts.sum())
    np.testing.assert_array_equal(acc[:total], ref[:total])
    assert d.status() == 0


@pytest.mark.parametrize("key", list(SMALL))
@pytest.mark.parametrize("deterministic", [True, False])
def test_finalize_matches_oracle(dev, oracle, problem_cache, key, deterministic):
    p = _small(problem_cache, key)
    d = dev.DeviceProblem(p)
    out = d.run(deterministic=deterministic).cpu().numpy()
    x1, pts = _oracle_inputs(oracle, d)
    o64, sabs, o32 = oracle.problem_finalize(p, x1=x1, pertoken_scale=pts)
    err = sum_rel_err(out, o64, sabs)
    plain = plain_rel_err(out, o64, sabs)
    if deterministic:
        np.testing.assert_array_equal(out, o32)
        assert err <= DET_TOL and plain <= DET_TOL, (err, plain)
    else:
        assert err <= ATOMIC_TOL and plain <= ATOMIC_TOL, (err, plain)
    assert d.status(deterministic) == 0


def test_deterministic_mode_is_bitwise_reproducible(dev, problem_cache):
    p = _small(problem_cache, "large_small")
    d = dev.DeviceProblem(p)
    a = d.run(deterministic=True).clone()
    b = d.run(deterministic=True).clone()
    assert torch.equal(a, b)


def test_group_list_forms_give_identical_output(dev, problem_cache):
    p = _small(problem_cache, "mid_small")
    d0 = dev.DeviceProblem(p)
    a = d0.run(deterministic=True).clone()
    from copy import copy
    q = copy(p)
    q.group_list_type = 1 - p.group_list_type
    q.group_list = p.counts.copy() if q.group_list_type == 1 else np.cumsum(p.counts)
    b = dev.DeviceProblem(q).run(deterministic=True)
    assert torch.equal(a, b)


def test_int32_row_index(dev, oracle, problem_cache):
    from copy import copy
    p = copy(_small(problem_cache, "tiny"))
    p.row_index = p.row_index.astype(np.int32)
    d = dev.DeviceProblem(p)
    out = d.run(deterministic=True).cpu().numpy()
    _, _, o32 = oracle.problem_finalize(p)
    np.testing.assert_array_equal(out, o32)


def test_optional_inputs_absent(dev, oracle, problem_cache, qgmm):
    """scale, pertoken_scale, logit, bias NULL (ones / zeros) and row_index NULL (identity)."""
    p = _small(problem_cache, "tiny")
    d = dev.DeviceProblem(p)
    m, n = p.m, p.n
    prob = qgmm.make_problem(m, p.k, n, p.e, m, group_list_type=p.group_list_type, deterministic=True)
    ws = torch.empty(qgmm.finalize_workspace(prob), dtype=torch.uint8, device="cuda")
    out = torch.empty((m, n), dtype=torch.float32, device="cuda")
    qgmm.finalize(prob, d.x1, d.x2, None, None, d.group_list, None, None, None, None, out, ws)
    _, _, o32 = oracle.finalize(p.x1, p.x2, p.group_list, p.group_list_type, output_bs=m)
    np.testing.assert_array_equal(out.cpu().numpy(), o32)
    assert qgmm.device_status(ws) == 0


def test_shared_input_at_offset_with_empty_experts(dev, oracle):
    from synth import make_problem
    p = make_problem("large_prefill", tokens=40, e=12, k=256, n=512, seed=99)
    p.counts[3] = 0
    # rebuild a consistent layout with expert 3 removed: route its rows to expert 4
    gl = np.cumsum(p.counts)
    extra = p.m - gl[-1]
    p.counts[4] += extra
    p.group_list = np.cumsum(p.counts).astype(np.int64)
    rng = np.random.default_rng(5)
    from synth.inputs import bf16_bits_normal
    p.shared = bf16_bits_normal(rng, (25, p.n))
    p.shared_offset = 10
    p.output_bs = 40
    for det in (True, False):
        d = dev.DeviceProblem(p)
        out = d.run(deterministic=det).cpu().numpy()
        o64, sabs, o32 = oracle.problem_finalize(p)
        if det:
            np.testing.assert_array_equal(out, o32)
        assert sum_rel_err(out, o64, sabs) <= (DET_TOL if det else ATOMIC_TOL)


def test_all_groups_empty_leaves_shared_rows(dev, qgmm):
    from types import SimpleNamespace
    rng = np.random.default_rng(1)
    k, n, e, m, obs = 256, 512, 4, 8, 6
    sh = (rng.standard_normal((3, n)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    p = SimpleNamespace(m=m, k=k, n=n, e=e, output_bs=obs, weight="int8", group_list_type=1,
                        x1=rng.integers(-127, 128, (m, k), dtype=np.int8), x_bf16=None,
                        x2=rng.integers(-127, 128, (e, k, n), dtype=np.int8),
                        scale=np.ones((e, n), np.float32), pertoken_scale=np.ones(m, np.float32),
                        group_list=np.zeros(e, np.int64), logit=np.ones(m, np.float32),
                        row_index=np.zeros(m, np.int64), bias=None, shared=sh, shared_offset=2)
    ref = np.zeros((obs, n), np.float32)
    ref[2:5] = (sh.astype(np.uint32) << 16).view(np.float32)
    for det in (True, False):
        d = dev.DeviceProblem(p)
        d.out.fill_(123.0)
        out = d.run(deterministic=det).cpu().numpy()
        np.testing.assert_array_equal(out, ref)
        assert d.status(det) == 0


@pytest.mark.parametrize("output_bs", [1, 3])
def test_deterministic_mode_with_skewed_buckets(dev, oracle, output_bs):
    """Thousands of source rows into one or three output rows: the destination buckets
    are filled in source-row order (no per-bucket sort), and the ordered sum still
    matches the oracle's fixed-order f32 bit for bit."""
    from types import SimpleNamespace
    rng = np.random.default_rng(30 + output_bs)
    m, k, n, e = 5000, 256, 512, 6
    counts = rng.multinomial(m, np.full(e, 1.0 / e)).astype(np.int64)
    p = SimpleNamespace(m=m, k=k, n=n, e=e, output_bs=output_bs, weight="int8", group_list_type=1, counts=counts,
                        x1=rng.integers(-127, 128, (m, k), dtype=np.int8), x_bf16=None,
                        x2=rng.integers(-127, 128, (e, k, n), dtype=np.int8),
                        scale=rng.uniform(1e-3, 1e-2, (e, n)).astype(np.float32),
                        pertoken_scale=rng.uniform(1e-3, 1e-2, m).astype(np.float32), group_list=counts.copy(),
                        logit=rng.uniform(0.05, 1.0, m).astype(np.float32),
                        row_index=rng.integers(0, output_bs, m).astype(np.int64), bias=None, shared=None,
                        shared_offset=0)
    d = dev.DeviceProblem(p)
    out = d.run(deterministic=True).cpu().numpy()
    _, _, o32 = oracle.problem_finalize(p, want64=False)
    np.testing.assert_array_equal(out, o32)
    assert d.status(True) == 0


# --------------------------------------------------------------------------- device-side input errors
@pytest.mark.parametrize("deterministic", [True, False])
def test_bad_row_index_is_flagged_and_writes_nothing_outside(dev, problem_cache, deterministic):
    from copy import copy
    p = copy(_small(problem_cache, "tiny"))
    p.row_index = p.row_index.copy()
    p.row_index[3] = p.output_bs + 7
    p.row_index[10] = -3
    d = dev.DeviceProblem(p)
    guard = 4
    big = torch.full((p.output_bs + 2 * guard, p.n), 7.0, dtype=torch.float32, device="cuda")
    d.run(deterministic=deterministic, out=big[guard:guard + p.output_bs])
    flags = d.status(deterministic)
    from quantized_moe_grouped_persistent_b200 import QGMM_DEV_ROW_INDEX_RANGE
    assert flags & QGMM_DEV_ROW_INDEX_RANGE
    b = big.cpu().numpy()
    assert (b[:guard] == 7.0).all() and (b[guard + p.output_bs:] == 7.0).all()


@pytest.mark.parametrize("bad,bit", [
    ("negative", "QGMM_DEV_GROUP_NEGATIVE"),
    ("not_monotone", "QGMM_DEV_GROUP_NOT_MONOTONE"),
    ("too_many", "QGMM_DEV_GROUP_TOTAL_GT_M"),
])
def test_bad_group_list_is_flagged(dev, problem_cache, bad, bit):
    from copy import copy
    import quantized_moe_grouped_persistent_b200 as q
    p = copy(_small(problem_cache, "tiny"))
    if bad == "negative":
        p.group_list_type, p.group_list = 1, np.array([5, -2, 10, 3], np.int64)
    elif bad == "not_monotone":
        p.group_list_type, p.group_list = 0, np.array([10, 5, 30, 40], np.int64)
    else:
        p.group_list_type, p.group_list = 1, np.array([30, 30, 30, 30], np.int64)
    d = dev.DeviceProblem(p)
    guard = 2
    big = torch.full((p.output_bs + 2 * guard, p.n), 5.0, dtype=torch.float32, device="cuda")
    d.run(deterministic=False, out=big[guard:guard + p.output_bs])
    assert d.status(False) & getattr(q, bit)
    acc = d.accum()
    assert d.status(False) & getattr(q, bit)
    b = big.cpu().numpy()
    assert (b[:guard] == 5.0).all() and (b[guard + p.output_bs:] == 5.0).all()
    assert torch.isfinite(acc.float()).all()


# --------------------------------------------------------------------------- prologue
def test_per_token_quant_bit_exact(dev, oracle, qgmm):
    from synth.inputs import bf16_bits_normal
    rng = np.random.default_rng(8)
    x = bf16_bits_normal(rng, (300, 2048))
    x[5] = 0                                       # all-zero row
    x[7, :8] = (np.array([127.0, 2.5, 3.5, -2.5, 0.5, 1.5, -127.0, 0.0], np.float32).view(np.uint32) >> 16)
    x[7, 8:] = 0
    # non-finite inputs (IEEE reading): NaN skipped by the absmax and coded 0; an
    # infinity gives pts = inf and a zero inverse; an all-NaN row is a zero row
    x[9, 3], x[10, 100], x[11, 5], x[11, 6], x[12, :] = 0x7FC0, 0x7F80, 0xFF80, 0x7FC0, 0x7FC0
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    q = torch.empty((300, 2048), dtype=torch.int8, device="cuda")
    s = torch.empty(300, dtype=torch.float32, device="cuda")
    qgmm.per_token_quant(xd, q, s)
    rq, rs = oracle.per_token_quant(x)
    np.testing.assert_array_equal(q.cpu().numpy(), rq)
    np.testing.assert_array_equal(s.cpu().numpy(), rs)
    np.testing.assert_array_equal(q.cpu().numpy()[7, :8], [127, 2, 4, -2, 0, 2, -127, 0])
    qs, ss = q.cpu().numpy(), s.cpu().numpy()
    assert qs[9, 3] == 0 and np.isfinite(ss[9]) and ss[9] > 0
    assert ss[10] == np.inf and ss[11] == np.inf and (qs[10:13] == 0).all() and ss[12] == 0


def test_per_token_quant_mxfp8_bit_exact(dev, oracle, qgmm):
    """Per-32-group FP8 cast: E4M3 codes and E8M0 scale codes bit for bit, on normal
    rows, a k that is not a multiple of 256, and hand-made groups: zero, NaN, +-inf,
    bf16 subnormals, a saturating top element, round-half-even ties."""
    from synth.inputs import bf16_bits_normal
    rng = np.random.default_rng(81)
    for rows, k in ((300, 2048), (37, 96)):
        x = bf16_bits_normal(rng, (rows, k))
        x[1, :32] = 0                                             # zero group
        x[2, 3], x[3, 40], x[4, 7], x[5, :32] = 0x7FC0, 0x7F80, 0xFF80, 0x7FC0
        x[6, :32] = rng.integers(1, 0x80, 32, dtype=np.uint16)    # bf16 subnormals
        x[7, 0] = 0x43E6                                          # 460: saturates
        x[8, :4] = [0x3F80, 0x3D88, 0x3D98, 0xBD88]               # amax 1, times 2^8: ties 17 -> 16, 19 -> 20
        xd = torch.from_numpy(x.view(np.int16)).cuda()
        q = torch.empty((rows, k), dtype=torch.uint8, device="cuda")
        sf = torch.empty((rows, k // 32), dtype=torch.uint8, device="cuda")
        qgmm.per_token_quant_mxfp8(xd, q, sf)
        rq, rsf = oracle.per_token_quant_mxfp8(x)
        np.testing.assert_array_equal(sf.cpu().numpy(), rsf)
        np.testing.assert_array_equal(q.cpu().numpy(), rq)
