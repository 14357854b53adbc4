"""Failure detection on the GPU without a fault: every in-kernel wait is bounded.

A test-only switch (QGMM_TEST_STALL_PRODUCER=1, read at call time) makes the
grouped GEMM's producer issue no copy.  The MMA warp's wait for operands then
runs out after its one-second bound; the kernel must set QGMM_DEV_TIMEOUT in
the status word, release its tensor memory and return, leaving the context
usable: the next ordinary call on the same operands matches the oracle.
The single-CTA kernel and the CTA-pair kernel are covered, the latter with its
tail launch and with tails as M=128 pair tiles.
"""
import time

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


@pytest.mark.parametrize("case", ["single_cta", "cta_pair_tail_launch", "cta_pair_tail128"])
def test_bounded_wait_runs_out_and_context_survives(dev, qgmm, oracle, problem_cache, monkeypatch, case):
    if case == "single_cta":
        p, hint = problem_cache("tiny"), 0                                        # 16-row tiles, one CTA
    else:
        p, hint = problem_cache("mid_prefill", tokens=96, e=8, k=512, n=768), 200   # pair tiles + tails
        monkeypatch.setenv("QGMM_PAIR_TAILS", "1" if case == "cta_pair_tail_launch" else "2")
    d = dev.DeviceProblem(p, expected_m_per_expert=hint)
    monkeypatch.setenv("QGMM_TEST_STALL_PRODUCER", "1")
    t0 = time.time()
    d.run(deterministic=False)
    flags = d.status(False)
    elapsed = time.time() - t0
    monkeypatch.delenv("QGMM_TEST_STALL_PRODUCER")
    assert flags & qgmm.QGMM_DEV_TIMEOUT
    assert elapsed < 30.0
    # the context still works and the next call is exact
    out = d.run(deterministic=True).cpu().numpy()
    assert d.status(True) == 0
    _, _, o32 = oracle.problem_finalize(p)
    np.testing.assert_array_equal(out, o32)
