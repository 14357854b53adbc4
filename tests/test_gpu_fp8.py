"""GPU parity of the FLOAT8 E4M3 mode (page 1, Atlas 350: x1 and x2 FLOAT8_E4M3FN
with a per-channel scale and a per-token pertokenScale), through the C ABI.

The tensor core sums E4M3 products in f32 (tcgen05.mma kind::f8f6f4), so the
accumulators are not exact; the oracle's are (double).  Bound, from the
arithmetic: a K = 32 MMA step adds its 32 products into the f32 accumulator, at
most one rounding of 2^-24 relative per step on top of the step's own sum, so
|acc_gpu - acc_exact| <= 2 * (k / 32) * 2^-24 * sum|products| (a factor 2 for
the step's inner sum).  The output then carries the f32 dequant and combine,
bounded as in the int8 tests (1e-5 / 2e-5 of the element's term magnitude, the
FP8 term magnitude using sum|products| in place of |acc|).  Small integers
(the worked example) sum exactly, so that case is bitwise.
"""
import json
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def acc_tol(k: int) -> float:
    return 2.0 * (k / 32) * 2.0 ** -24


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


def test_worked_example_in_fp8_on_gpu(dev):
    from types import SimpleNamespace
    g = json.load(open(os.path.join(GOLDEN, "per_token_worked_example.json")))
    code = {1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48, 5: 0x4A, 6: 0x4C}
    k, n = 128, 256
    x1 = np.zeros((2, k), np.uint8)
    x1[:, :2] = np.vectorize(code.get)(np.array(g["x"]))
    x2 = np.zeros((1, k, n), np.uint8)
    x2[0, :2, :3] = np.vectorize(code.get)(np.array(g["weight"]))
    scale = np.ones((1, n), np.float32)
    scale[0, :3] = g["deqScale"]
    p = SimpleNamespace(m=2, k=k, n=n, e=1, output_bs=2, group_list_type=1, weight="fp8", x1=x1, x_bf16=None,
                        x2=x2, scale=scale, pertoken_scale=np.array(g["perTokenScale"], np.float32),
                        group_list=np.array([2], np.int64), counts=np.array([2]), logit=np.ones(2, np.float32),
                        row_index=np.array([0, 1], np.int64), bias=None, shared=None, shared_offset=0)
    d = dev.DeviceProblem(p)
    for det in (True, False):
        out = d.run(deterministic=det).cpu().numpy()
        np.testing.assert_array_equal(out[:, :3], np.array(g["output"], np.float32))
        assert (out[:, 3:] == 0).all()
    acc = d.accum().cpu().numpy().view(np.float32)
    np.testing.assert_array_equal(acc[:, :3], [[9, 12, 15], [19, 26, 33]])


CASES = {
    # name: (make_problem kwargs, tiling hint): single-CTA tiles, and CTA-pair tiles with tails
    "small_tiles": (dict(tokens=64, e=8, k=256, n=512), 0),
    "pairs": (dict(tokens=300, e=10, k=512, n=768, seed=66), 200),
    "large_k": (dict(tokens=40, e=3, k=4096, n=256, seed=67), 0),
}


def _problem(name):
    from synth import make_problem
    kw, hint = CASES[name]
    return make_problem("fp8_prefill", **kw), hint


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_accumulators_within_the_f32_bound(dev, oracle, name):
    p, hint = _problem(name)
    d = dev.DeviceProblem(p, expected_m_per_expert=hint)
    acc = d.accum().cpu().numpy().view(np.float32).astype(np.float64)
    ref, mag = oracle.accum_f8(p.x1, p.x2, p.group_list, p.group_list_type)
    total = int(p.counts.sum())
    err = np.abs(acc[:total] - ref[:total]) / np.where(mag[:total] > 0, mag[:total], 1.0)
    assert err.max() <= acc_tol(p.k), (err.max(), acc_tol(p.k))
    assert d.status() == 0


@pytest.mark.parametrize("deterministic", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_fp8_finalize_matches_oracle(dev, oracle, name, deterministic):
    p, hint = _problem(name)
    d = dev.DeviceProblem(p, expected_m_per_expert=hint)
    out = d.run(deterministic=deterministic).cpu().numpy()
    o64, sabs, _ = oracle.problem_finalize(p, want32=False)
    err = np.abs(out.astype(np.float64) - o64) / np.where(sabs > 0, sabs, 1.0)
    tol = acc_tol(p.k) + (1e-5 if deterministic else 2e-5)
    assert err.max() <= tol, (err.max(), tol)
    assert d.status(deterministic) == 0


def test_fp8_transposed_weights(dev, oracle):
    p, _ = _problem("small_tiles")
    d0 = dev.DeviceProblem(p)
    ref = d0.run(deterministic=True).clone()
    from copy import copy
    q = copy(p)
    q.x2 = np.ascontiguousarray(np.swapaxes(p.x2, 1, 2))
    q.transpose_x2 = True
    d1 = dev.DeviceProblem(q)
    out = d1.run(deterministic=True)
    assert torch.equal(out, ref)         # the same products in the same order: bitwise
