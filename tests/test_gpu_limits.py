"""GPU parity at the interface's size limits.

- m = 2^24 rows (the largest m qgmm_problem accepts) over e = 1024 experts (the
  largest e), with ragged, partly empty groups from a Dirichlet(0.5) popularity.
  Output rows get 8 contributions on average, so row offsets, tile counts and
  output indices all run at their largest values.  The oracle computes a seeded
  sample of output rows (every contributing source row in full) and exact int32
  accumulators for a seeded sample of source rows.
- k = 65536 (the largest k), with an x1 row and a weight column at the most
  negative value so that one accumulator reaches 65536*128*128 = 2^30 (int8;
  2^26 for int4), far above 2^24 where the f32 conversion rounds.  Checked in
  full, for int8 and for int4 weights.

Bars as in test_gpu_parity: bit-exact int32; deterministic mode bitwise equal to
the oracle's fixed-order f32; atomic mode within 2e-5 of the error magnitude.
"""
from types import SimpleNamespace

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ATOMIC_TOL = 2e-5


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


def _problem(seed, m, k, n, e, output_bs, weight="int8", alpha=0.5, extremes=False):
    rng = np.random.default_rng(seed)
    pop = rng.dirichlet(np.full(e, alpha))
    if e >= 8:
        pop[[1, e // 2, e - 1]] = 0.0            # always some empty experts, first / middle / last
    counts = rng.multinomial(m, pop / pop.sum()).astype(np.int64)
    x2 = (rng.integers(-127, 128, size=(e, k, n), dtype=np.int8) if weight == "int8"
          else rng.integers(0, 2 ** 32, size=(e, k, n // 8), dtype=np.uint32).view(np.int32))
    if extremes:
        # weight column 0 at the most negative value (int4: the whole first word is -8s)
        if weight == "int8":
            x2[:, :, 0] = -128
        else:
            x2[:, :, 0] = np.array([0x88888888], dtype=np.uint32).view(np.int32)[0]
    return SimpleNamespace(
        m=m, k=k, n=n, e=e, output_bs=output_bs, weight=weight, group_list_type=0, counts=counts,
        x1=rng.integers(-127, 128, size=(m, k), dtype=np.int8), x_bf16=None, x2=x2,
        scale=rng.uniform(1e-3, 1e-2, size=(e, n)).astype(np.float32),
        pertoken_scale=rng.uniform(1e-3, 1e-2, size=m).astype(np.float32),
        group_list=np.cumsum(counts).astype(np.int64), logit=rng.uniform(0.05, 1.0, size=m).astype(np.float32),
        row_index=rng.integers(0, output_bs, size=m).astype(np.int64),
        bias=rng.normal(0, 0.01, size=(e, n)).astype(np.float32), shared=None, shared_offset=0)


def _check_rows(d, oracle, p, out_rows):
    o64, sabs, o32 = oracle.problem_finalize(p, dest_rows=out_rows)
    den = np.where(sabs > 0, sabs, 1.0)
    rows_t = torch.from_numpy(out_rows).cuda()
    for det in (True, False):
        got = d.run(deterministic=det).index_select(0, rows_t).cpu().numpy()
        assert d.status(det) == 0
        if det:
            np.testing.assert_array_equal(got, o32)
        else:
            assert float((np.abs(got.astype(np.float64) - o64) / den).max()) <= ATOMIC_TOL


def test_largest_m_over_1024_experts(dev, oracle):
    from synth import sample_rows
    m = 1 << 24
    p = _problem(24, m, 128, 256, 1024, output_bs=m // 8)
    assert (p.counts == 0).any() and p.counts.sum() == m
    d = dev.DeviceProblem(p)                 # m / e = 16384 rows per expert: CTA-pair tiles + tail launch
    _check_rows(d, oracle, p, sample_rows(2424, p.output_bs, 64))
    src = sample_rows(4848, m, 128)
    acc = d.accum()
    got = acc.index_select(0, torch.from_numpy(src).cuda()).cpu().numpy()
    del acc
    ref = oracle.accum(p.x1, p.x2, p.group_list, p.group_list_type, rows=src)
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("weight", ["int8", "int4"])
def test_largest_k(dev, oracle, weight):
    p = _problem(65536 + (weight == "int4"), 300, 65536, 256, 3, output_bs=120, weight=weight, alpha=2.0,
                 extremes=True)
    p.x1[0, :] = -128                            # with weight column 0: acc = 65536 * 128 * 128 (int8)
    p.x1[1, :] = 127
    d = dev.DeviceProblem(p)
    _check_rows(d, oracle, p, np.arange(p.output_bs, dtype=np.int64))
    acc = d.accum().cpu().numpy()
    ref = oracle.accum(p.x1, p.x2, p.group_list, p.group_list_type, weight=p.weight)
    np.testing.assert_array_equal(acc, ref)
    bound = 65536 * 128 * (128 if weight == "int8" else 8)
    assert ref[0, 0] == bound                    # the extreme sum is reached, and is exact
    assert np.abs(ref).max() > 1 << 24           # so the conversion to f32 rounds
