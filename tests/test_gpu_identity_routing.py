"""GPU: identity routing (row_index NULL) without sharedInput, where the atomic mode
stores each row straight into the output instead of reducing into a zeroed one.

Every output row then receives at most one source row, so the result must be the
combine's 0 + y bit for bit.  Checked against the same call with an explicit
identity row_index (the reducing path), which itself is checked against the oracle
elsewhere, and against the oracle here:
- int8 on single-CTA tiles and on CTA-pair tiles with tails, int4, E4M3 and MxA8W4;
- rows past the groups' total (output_bs > total): zeros, whatever the output held;
- an output smaller than the total: the rows that fit are stored, the others are
  flagged (QGMM_DEV_ROW_INDEX_RANGE) and nothing is written past the output.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


def _case(name):
    from synth import make_problem
    kw = {
        "int8_single": ("mid_prefill", dict(tokens=40, e=8, k=256, n=512, seed=951), 0),
        "int8_pairs": ("mid_prefill", dict(tokens=300, e=6, k=256, n=768, seed=952), 200),
        "int4": ("w4a8_prologue", dict(tokens=48, e=6, k=256, n=512, seed=953), 0),
        "fp8": ("fp8_prefill", dict(tokens=200, e=5, k=256, n=512, seed=954), 200),
        "mx": ("w4a8_mx", dict(tokens=64, e=6, k=512, n=512, seed=955), 0),
    }[name]
    p = make_problem(kw[0], **kw[1])
    p.shared = None
    p.output_bs = int(p.counts.sum())
    return p, kw[2]


def _run(dev_mod, p, hint, row_index, out_rows, fill=np.nan):
    from quantized_moe_grouped_persistent_b200 import finalize
    d = dev_mod.DeviceProblem(p, expected_m_per_expert=hint)
    d.quantize()
    d.shared_bs = 0
    d.output_bs = out_rows
    guard = 64
    buf = torch.full((out_rows + guard, p.n), fill, dtype=torch.float32, device="cuda")
    ri = None if row_index is None else torch.from_numpy(row_index).cuda()
    prob = d.problem(False)
    finalize(prob, d.x1, d.x2, d.scale, d.pts, d.group_list, d.logit, ri, d.bias, None, buf[:out_rows],
             d.workspace(False))
    return buf, d.status(False)


@pytest.mark.parametrize("name", ["int8_single", "int8_pairs", "int4", "fp8", "mx"])
def test_direct_store_equals_the_reducing_path_bitwise(dev, name):
    p, hint = _case(name)
    total = int(p.counts.sum())
    ident = np.arange(p.m, dtype=np.int64)
    direct, st0 = _run(dev, p, hint, None, total)
    reduced, st1 = _run(dev, p, hint, ident, total)
    assert st0 == 0 and st1 == 0
    assert torch.equal(direct[:total], reduced[:total])
    assert torch.isnan(direct[total:]).all()           # the guard rows are untouched


@pytest.mark.parametrize("name", ["int8_single", "int8_pairs"])
def test_direct_store_matches_oracle_and_zeroes_rows_past_the_total(dev, oracle, name):
    p, hint = _case(name)
    total = int(p.counts.sum())
    out_rows = total + 37
    buf, st = _run(dev, p, hint, None, out_rows)
    assert st == 0
    got = buf[:out_rows].cpu().numpy()
    _, _, o32 = oracle.finalize(p.x1 if p.x1 is not None else None, p.x2, p.group_list, p.group_list_type,
                                weight=p.weight, scale=p.scale, pertoken_scale=p.pertoken_scale, logit=p.logit,
                                bias=p.bias, row_index=np.arange(p.m, dtype=np.int64), output_bs=out_rows)
    np.testing.assert_array_equal(got, o32)            # one contribution per row: the fixed-order f32 value
    assert (got[total:] == 0).all()
    assert torch.isnan(buf[out_rows:]).all()


def test_output_smaller_than_the_total_is_flagged(dev):
    from quantized_moe_grouped_persistent_b200 import QGMM_DEV_ROW_INDEX_RANGE
    p, hint = _case("int8_single")
    total = int(p.counts.sum())
    short = total - 11
    direct, st = _run(dev, p, hint, None, short)
    reduced, _ = _run(dev, p, hint, np.arange(p.m, dtype=np.int64), short)
    assert st & QGMM_DEV_ROW_INDEX_RANGE
    assert torch.equal(direct[:short], reduced[:short])
    assert torch.isnan(direct[short:]).all()
