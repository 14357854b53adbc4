"""GPU parity on edge shapes: minimum sizes, the expert limit, tile-boundary group
sizes on both the single-CTA and the CTA-pair paths, rows past the groups'
total, and unusual k / n.  Same bars as test_gpu_parity (bit-exact int32,
deterministic mode bitwise equal to the oracle's fixed-order f32, atomic mode
within 2e-5 of the oracle's error magnitude: |sharedInput| plus, per
contribution, (|acc*scale*pts| + |bias|) * |logit|).
"""
from types import SimpleNamespace

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

ATOMIC_TOL = 2e-5


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


def _problem(seed, counts, k, n, extra_rows=0, output_bs=None, weight="int8", bias=True):
    rng = np.random.default_rng(seed)
    counts = np.asarray(counts, np.int64)
    e = counts.size
    total = int(counts.sum())
    m = total + extra_rows
    obs = output_bs or max(1, (total + 3) // 4)
    x2 = (rng.integers(-127, 128, size=(e, k, n), dtype=np.int8) if weight == "int8"
          else rng.integers(0, 2 ** 32, size=(e, k, n // 8), dtype=np.uint32).view(np.int32))
    return SimpleNamespace(
        m=m, k=k, n=n, e=e, output_bs=obs, weight=weight, group_list_type=1, counts=counts,
        x1=rng.integers(-127, 128, size=(m, k), dtype=np.int8), x_bf16=None, x2=x2,
        scale=rng.uniform(1e-3, 1e-2, size=(e, n)).astype(np.float32),
        pertoken_scale=rng.uniform(1e-3, 1e-2, size=m).astype(np.float32),
        group_list=counts.copy(), logit=rng.uniform(0.05, 1.0, size=m).astype(np.float32),
        row_index=rng.integers(0, obs, size=m).astype(np.int64),
        bias=rng.normal(0, 0.01, size=(e, n)).astype(np.float32) if bias else None,
        shared=None, shared_offset=0)


def _check(dev, oracle, p, hint):
    d = dev.DeviceProblem(p, expected_m_per_expert=hint)
    o64, sabs, o32 = oracle.problem_finalize(p)
    det = d.run(deterministic=True).cpu().numpy()
    assert d.status(True) == 0
    np.testing.assert_array_equal(det, o32)
    atom = d.run(deterministic=False).cpu().numpy()
    assert d.status(False) == 0
    err = np.abs(atom.astype(np.float64) - o64) / np.where(sabs > 0, sabs, 1.0)
    assert err.max() <= ATOMIC_TOL
    total = int(p.counts.sum())
    acc = d.accum().cpu().numpy()
    ref = oracle.accum(p.x1, p.x2, p.group_list, p.group_list_type, weight=p.weight,
                       transpose_x2=bool(getattr(p, "transpose_x2", False)))
    np.testing.assert_array_equal(acc[:total], ref[:total])


def test_single_row_single_expert_minimum_sizes(dev, oracle):
    _check(dev, oracle, _problem(1, [1], 128, 256, output_bs=1), 0)


def test_expert_limit_mostly_empty(dev, oracle):
    counts = np.zeros(1024, np.int64)
    counts[[0, 511, 1023]] = [3, 40, 5]
    _check(dev, oracle, _problem(2, counts, 128, 256, bias=False), 0)


@pytest.mark.parametrize("hint", [1, 200])     # single-CTA 16-row tiles / CTA-pair 256-row tiles + tails
def test_tile_boundary_group_sizes(dev, oracle, hint):
    counts = [127, 128, 129, 0, 255, 256, 257, 383, 1]
    _check(dev, oracle, _problem(3, counts, 256, 512), hint)


@pytest.mark.parametrize("hint", [0, 200])
def test_rows_past_the_total_are_ignored(dev, oracle, hint):
    _check(dev, oracle, _problem(4, [100, 0, 300], 256, 512, extra_rows=77), hint)


@pytest.mark.parametrize("k,n", [(128, 256), (256, 1792), (4096, 256)])
def test_unusual_k_and_n(dev, oracle, k, n):
    _check(dev, oracle, _problem(5, [40, 260, 7], k, n), 0)


def test_int4_on_tile_boundaries(dev, oracle):
    _check(dev, oracle, _problem(6, [128, 129, 1, 256], 256, 512, weight="int4"), 0)


@pytest.mark.parametrize("tail_mode", ["0", "1", "2"])
def test_pair_tail_modes_are_exact(dev, oracle, monkeypatch, tail_mode):
    """The three ways of running a group's odd last 128 rows on the CTA-pair path
    (padded pair tile, single-CTA launch, M=128 pair tile) give identical results."""
    monkeypatch.setenv("QGMM_PAIR_TAILS", tail_mode)
    _check(dev, oracle, _problem(7, [1, 128, 129, 255, 256, 300, 383, 0, 640], 256, 768), 200)


@pytest.mark.parametrize("pair_w4", ["0", "1"])
def test_int4_full_height_tiles_single_and_pair(dev, oracle, monkeypatch, pair_w4):
    """int4 weights on 128-row tiles: the single-CTA kernel and the optional CTA-pair
    kernel (each CTA unpacks its own 128-column half of the packed tile) are exact."""
    monkeypatch.setenv("QGMM_PAIR_W4", pair_w4)
    _check(dev, oracle, _problem(8, [1, 129, 255, 256, 300, 0, 513], 256, 768, weight="int4"), 200)


def test_launch_count_query(dev, qgmm, monkeypatch):
    """qgmm_finalize_launches follows the plan: pair tiles + a tail launch, or one GEMM launch."""
    p = _problem(9, [300, 0, 40], 256, 512)
    monkeypatch.setenv("QGMM_PAIR_TAILS", "1")
    pair = dev.DeviceProblem(p, expected_m_per_expert=200)     # 128-row tiles: CTA pairs + tail launch
    assert qgmm.finalize_launches(pair.problem(False)) == 3    # init, pair GEMM, tail GEMM
    assert qgmm.finalize_launches(pair.problem(True)) == 8     # 5 bucketing kernels, 2 GEMM, reduce
    monkeypatch.setenv("QGMM_PAIR_TAILS", "2")                 # tails as M=128 pair tiles in one launch
    assert qgmm.finalize_launches(pair.problem(False)) == 2
    single = dev.DeviceProblem(p, expected_m_per_expert=1)     # 16-row tiles on single CTAs
    assert qgmm.finalize_launches(single.problem(False)) == 2


def test_default_tail_mode_follows_wave_counts(qgmm, monkeypatch):
    """Without QGMM_PAIR_TAILS the planner runs tails as M=128 pair tiles when both
    launches would be short (32 experts, m = 8192, n = 7168: one GEMM launch), and as
    a single-CTA tail launch once the pair launch is long (m = 32768) or the tails
    are many (256 experts)."""
    if not torch.cuda.is_available() or torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("wave counts are for a 148-SM B200")
    monkeypatch.delenv("QGMM_PAIR_TAILS", raising=False)
    launches = lambda m, e: qgmm.finalize_launches(qgmm.make_problem(m, 2048, 7168, e, m // 8))
    assert launches(8192, 32) == 2          # output init + pair GEMM
    assert launches(32768, 32) == 3         # output init + pair GEMM + tail GEMM
    assert launches(131072, 256) == 3


@pytest.mark.parametrize("weight,hint", [("int8", 0), ("int8", 200), ("int4", 0), ("int4", 200)])
def test_bf16_scale(dev, oracle, weight, hint):
    """scale given as bf16 bits (page 1: scaleOptional is FLOAT or BF16), on every
    epilogue: 16-row tiles, CTA pairs with their tail launch, and int4 tiles.  The
    oracle widens the same bits to f32; the bars are those of the f32 scale."""
    p = _problem(10, [1, 129, 255, 256, 0, 300, 40], 256, 768, weight=weight)
    rng = np.random.default_rng(11)
    f32 = rng.uniform(1e-3, 1e-2, size=p.scale.shape).astype(np.float32)
    p.scale = (f32.view(np.uint32) >> 16).astype(np.uint16)            # truncate to bf16 bits
    assert dev.DeviceProblem(p, expected_m_per_expert=hint).scale_type == 1
    _check(dev, oracle, p, hint)


@pytest.mark.parametrize("hint,env", [
    (1, {}),                              # 16-row tiles, single CTA
    (200, {"QGMM_PAIR": "0"}),            # 128-row tiles, single CTA
    (200, {"QGMM_PAIR_TAILS": "1"}),      # CTA pairs + single-CTA tail launch
    (200, {"QGMM_PAIR_TAILS": "2"}),      # CTA pairs, tails as M=128 pair tiles
])
def test_transposed_int8_weights(dev, oracle, monkeypatch, hint, env):
    """int8 x2 stored (e, n, k) (page 1, full-quant scenario: x2 may be transposed):
    K-major weight tiles on 16-row and 128-row single-CTA tiles and on CTA pairs with
    either tail form, in both combine modes, against the oracle on the same layout."""
    for k_, v in env.items():
        monkeypatch.setenv(k_, v)
    p = _problem(12, [1, 129, 255, 256, 0, 300, 40, 17], 256, 768)
    p.x2 = np.ascontiguousarray(np.swapaxes(p.x2, 1, 2))          # (e, n, k)
    p.transpose_x2 = True
    _check(dev, oracle, p, hint)
