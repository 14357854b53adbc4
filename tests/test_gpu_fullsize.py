"""GPU parity at the full workload sizes, in the launch configuration the benchmark uses.

The oracle computes a seeded sample of output rows one by one (every source
row that lands in a sampled row, in full), plus exact int32 accumulators for a
seeded sample of source rows.  Bars as in test_gpu_parity: bit-exact int32;
deterministic mode bitwise equal to the oracle's fixed-order f32 and within
1e-5 of the double result; atomic mode within 2e-5 (error relative to the sum
of |terms| of each element).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DET_TOL = 1e-5
ATOMIC_TOL = 2e-5
FULL = ["mid_prefill", "decode", "large_prefill", "w4a8_prologue"]
SAMPLE_OUT_ROWS = {"mid_prefill": 96, "decode": 16, "large_prefill": 96, "w4a8_prologue": 96}
SAMPLE_SRC_ROWS = 128


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


@pytest.fixture(scope="module")
def loaded(dev, problem_cache):
    cache = {}

    def get(name):
        if name not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            p = problem_cache(name)
            cache[name] = (p, dev.DeviceProblem(p))
        return cache[name]
    return get


def _oracle_x1(oracle, p):
    if p.x1 is not None:
        return p.x1, p.pertoken_scale
    return oracle.per_token_quant(p.x_bf16)


@pytest.mark.parametrize("name", FULL)
def test_full_size_output_rows(loaded, oracle, name):
    from synth import sample_rows
    p, d = loaded(name)
    rows = sample_rows(777, p.output_bs, SAMPLE_OUT_ROWS[name])
    x1, pts = _oracle_x1(oracle, p)
    o64, sabs, o32 = oracle.problem_finalize(p, x1=x1, pertoken_scale=pts, dest_rows=rows)
    den = np.where(sabs > 0, sabs, 1.0)
    rows_t = torch.from_numpy(rows).cuda()
    for det in (True, False):
        out = d.run(deterministic=det)
        got = out.index_select(0, rows_t).cpu().numpy()
        assert d.status(det) == 0
        err = float((np.abs(got.astype(np.float64) - o64) / den).max())
        if det:
            np.testing.assert_array_equal(got, o32)
            assert err <= DET_TOL
        else:
            assert err <= ATOMIC_TOL, err
    if d.prologue:
        np.testing.assert_array_equal(d.x1.cpu().numpy(), x1)
        np.testing.assert_array_equal(d.pts.cpu().numpy(), pts)


@pytest.mark.parametrize("name", FULL)
def test_full_size_accumulators(loaded, oracle, name):
    from synth import sample_rows
    p, d = loaded(name)
    d.quantize()
    x1, _ = _oracle_x1(oracle, p)
    total = int(p.counts.sum())
    rows = sample_rows(4242, total, SAMPLE_SRC_ROWS)
    acc = d.accum()
    got = acc.index_select(0, torch.from_numpy(rows).cuda()).cpu().numpy()
    del acc
    ref = oracle.accum(x1, p.x2, p.group_list, p.group_list_type, weight=p.weight, rows=rows)
    np.testing.assert_array_equal(got, ref)
    assert d.status(False) == 0
