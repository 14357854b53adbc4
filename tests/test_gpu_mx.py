"""GPU parity of the MxA8W4 mode (page 1, Atlas 350: E4M3 activations and FP4 E2M1
weights, each with an E8M0 scale per 32 k-elements), through the C ABI.

- An exact case: small-integer E4M3 activations and E2M1 weights, and scales that
  differ by row, by column and by 32-element block (powers of two between 2^-2 and
  2^2), so every partial sum is a short dyadic number that f32 holds exactly.  The
  accumulators must equal the oracle's bit for bit, which pins which scale the
  tensor core applies to which row, column and block.
- Seeded workloads (activations through the per-32-group FP8 cast on the GPU, the
  oracle casting the same bf16 values itself): accumulators within the f32 bound of
  the FP8 mode, 2 (k/32) 2^-24 of the sum of |scaled products|; outputs within that
  plus the int8 path's 1e-5 / 2e-5 of the term magnitude.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def acc_tol(k: int) -> float:
    return 2.0 * (k / 32) * 2.0 ** -24


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


def _exact_case():
    from types import SimpleNamespace
    rng = np.random.default_rng(2024)
    m, k, n, e = 160, 256, 256, 2
    counts = np.array([130, 30], np.int64)               # a full 128-row tile plus ragged ones
    e4m3 = {-2: 0xC0, -1: 0xB8, 0: 0x00, 1: 0x38, 2: 0x40}
    e2m1 = {-2.0: 0xC, -1.5: 0xB, -1.0: 0xA, -0.5: 0x9, 0.0: 0x0, 0.5: 0x1, 1.0: 0x2, 1.5: 0x3, 2.0: 0x4}
    xv = rng.integers(-2, 3, (m, k))
    x1 = np.vectorize(e4m3.get)(xv).astype(np.uint8)
    wv = rng.choice(list(e2m1), size=(e, n, k))
    nib = np.vectorize(e2m1.get)(wv).astype(np.uint8)
    x2 = (nib[:, :, 0::2] | (nib[:, :, 1::2] << 4)).astype(np.uint8)
    i, b = np.meshgrid(np.arange(m), np.arange(k // 32), indexing="ij")
    sfa = (125 + (i * 7 + b * 3) % 5).astype(np.uint8)   # 2^-2 .. 2^2, varying by row and block
    g, j, b = np.meshgrid(np.arange(e), np.arange(n), np.arange(k // 32), indexing="ij")
    sfb = (125 + (g * 2 + j * 5 + b) % 5).astype(np.uint8)   # varying by expert, column and block
    return SimpleNamespace(m=m, k=k, n=n, e=e, output_bs=m, group_list_type=1, weight="mxfp4", x1=x1,
                           x_bf16=None, x2=x2, transpose_x2=True, scale=sfb, pertoken_scale=sfa,
                           group_list=counts.copy(), counts=counts, logit=np.ones(m, np.float32),
                           row_index=np.arange(m, dtype=np.int64), bias=None, shared=None, shared_offset=0)


def test_mx_exact_small_integers_pin_the_scale_layout(dev, oracle):
    p = _exact_case()
    d = dev.DeviceProblem(p)
    acc = d.accum().cpu().numpy().astype(np.float64)
    ref, _ = oracle.accum_mx(p.x1, p.pertoken_scale, p.x2, p.scale, p.group_list, p.group_list_type)
    np.testing.assert_array_equal(acc, ref)
    assert d.status() == 0
    for det in (True, False):
        out = d.run(deterministic=det).cpu().numpy().astype(np.float64)
        np.testing.assert_array_equal(out, ref)          # identity routing, unit logit, no bias


CASES = {
    "small": dict(tokens=40, e=8, k=256, n=256),
    "ragged": dict(tokens=90, e=6, k=512, n=512, seed=71),
    "large_k": dict(tokens=24, e=3, k=4096, n=256, seed=72),
}


def _mx_oracle_inputs(oracle, p):
    q, sfa = oracle.per_token_quant_mxfp8(p.x_bf16)
    return q, sfa


@pytest.mark.parametrize("name", list(CASES))
def test_mx_accumulators_within_the_f32_bound(dev, oracle, problem_cache, name):
    p = problem_cache("w4a8_mx", **CASES[name])
    d = dev.DeviceProblem(p)
    d.quantize()
    q, sfa = _mx_oracle_inputs(oracle, p)
    np.testing.assert_array_equal(d.x1.cpu().numpy(), q)
    np.testing.assert_array_equal(d.pts.cpu().numpy(), sfa)
    acc = d.accum().cpu().numpy().astype(np.float64)
    ref, mag = oracle.accum_mx(q, sfa, p.x2, p.scale, p.group_list, p.group_list_type)
    total = int(p.counts.sum())
    err = np.abs(acc[:total] - ref[:total]) / np.where(mag[:total] > 0, mag[:total], 1.0)
    assert err.max() <= acc_tol(p.k), (err.max(), acc_tol(p.k))


@pytest.mark.parametrize("deterministic", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_mx_finalize_matches_oracle(dev, oracle, problem_cache, name, deterministic):
    p = problem_cache("w4a8_mx", **CASES[name])
    d = dev.DeviceProblem(p)
    out = d.run(deterministic=deterministic).cpu().numpy()
    q, sfa = _mx_oracle_inputs(oracle, p)
    o64, sabs, _ = oracle.finalize_mx(q, sfa, p.x2, p.scale, p.group_list, p.group_list_type, logit=p.logit,
                                      bias=p.bias, row_index=p.row_index, output_bs=p.output_bs, want32=False)
    err = np.abs(out.astype(np.float64) - o64) / np.where(sabs > 0, sabs, 1.0)
    tol = acc_tol(p.k) + (1e-5 if deterministic else 2e-5)
    assert err.max() <= tol, (err.max(), tol)
    assert d.status(deterministic) == 0
