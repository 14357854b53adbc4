"""qgmm_finalize_static_scratch: the entry point for callers that cannot allocate.

Some callers are handed only their inputs and outputs -- a plugin slot in a
host inference engine with no workspace, or a serving loop that must not call
cudaMalloc/cudaFree because those can synchronise the device.  For them the
library offers qgmm_finalize without a workspace argument; its scratch is a
16 MiB array inside the library.  These tests call it through the C ABI and
check that it gives the output of the workspace-taking entry point, on two
calls in a row, in both combine modes.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

torch = pytest.importorskip("torch")

ATOMIC_TOL = 2e-5


def test_oversized_problem_is_rejected_before_launch(qgmm):
    """Deterministic workspace above 16 MiB: QGMM_ERR_SCRATCH_LIMIT.  NULL operands
    guarantee that nothing could be launched even if the check were missing."""
    p = qgmm.make_problem(8192, 2048, 7168, 32, 1024, deterministic=True)
    assert qgmm.finalize_workspace(p) > qgmm.QGMM_STATIC_SCRATCH_BYTES
    rc = qgmm.lib().qgmm_finalize_static_scratch(C.byref(p), *([None] * 11))
    assert rc == qgmm.QGMM_ERR_SCRATCH_LIMIT
    assert "scratch" in qgmm.status_string(rc)


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


def _problems():
    """(problem, tiling hint): decode-sized single-CTA tiles; a 200-rows-per-expert hint,
    which plans full-height tiles on CTA pairs, here with groups of 1 to 3 half tiles of
    128 rows (so pair tiles and odd tails); int4 weights after the per-token quant
    prologue."""
    from synth import make_problem
    return [(make_problem("decode", tokens=16, e=64, k=512, n=1024), 0),          # bias, many empty experts
            (make_problem("large_prefill", tokens=64, e=16, k=256, n=512), 0),    # bf16 sharedInput rows
            (make_problem("large_prefill", tokens=360, e=12, k=256, n=512, seed=82), 200),
            (make_problem("w4a8_prologue", tokens=48, e=8, k=256, n=512), 0)]


@pytest.mark.gpu
@pytest.mark.parametrize("tails", ["1", "2"])
@pytest.mark.parametrize("deterministic", [True, False])
def test_static_scratch_matches_workspace_entry_point(dev, qgmm, oracle, deterministic, tails, monkeypatch):
    # odd tails of the pair path: a single-CTA launch after the pair launch (1), or
    # M = 128 pair tiles inside it (2); the library reads the switch at each call
    monkeypatch.setenv("QGMM_PAIR_TAILS", tails)
    for p, hint in _problems():
        d = dev.DeviceProblem(p, expected_m_per_expert=hint)
        if hint:
            assert qgmm.plan(d.problem(deterministic), 148)["pair"] == 1
        prob = d.problem(deterministic)
        assert qgmm.finalize_workspace(prob) <= qgmm.QGMM_STATIC_SCRATCH_BYTES
        ref = d.run(deterministic=deterministic).clone()
        assert d.status(deterministic) == 0
        ref_h = ref.cpu().numpy()
        if p.x1 is None:                                         # prologue workload: the oracle's own codes
            q, s = oracle.per_token_quant(p.x_bf16)
            _, sabs, _ = oracle.problem_finalize(p, x1=q, pertoken_scale=s, want32=False)
        else:
            _, sabs, _ = oracle.problem_finalize(p, want32=False)
        den = np.where(sabs > 0, sabs, 1.0)
        for _ in range(2):                                       # two calls in a row share the array
            out = torch.full_like(ref, float("nan"))
            qgmm.finalize_static_scratch(prob, d.x1, d.x2, d.scale, d.pts, d.group_list, d.logit, d.row_index,
                                         d.bias, d.shared, out)
            torch.cuda.synchronize()
            got = out.cpu().numpy()
            if deterministic:
                np.testing.assert_array_equal(got, ref_h)
            else:
                err = np.abs(got.astype(np.float64) - ref_h.astype(np.float64)) / den
                assert err.max() <= ATOMIC_TOL, err.max()
