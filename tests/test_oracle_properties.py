"""Property-based pins of the CPU oracle: the fixed-seed pins of test_oracle.py over
drawn shapes, group sizes (empty groups included) and weight layouts.

Each property is fixed by something other than the oracle: numpy's int64 matmul (a
library routine), nibble unpacking written here with numpy bit operations, or an
exact algebraic invariant of the op.
"""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

SETTINGS = settings(max_examples=30, deadline=None, derandomize=True)


@st.composite
def grouped(draw, max_e=5, max_rows=9):
    e = draw(st.integers(1, max_e))
    counts = np.array(draw(st.lists(st.integers(0, max_rows), min_size=e, max_size=e)), np.int64)
    k = draw(st.integers(1, 48))
    n = 8 * draw(st.integers(1, 4))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return e, counts, k, n, np.random.default_rng(seed)


def _numpy_acc(x1, w, counts):
    off = np.concatenate([[0], np.cumsum(counts)])
    out = np.zeros((x1.shape[0], w.shape[2]), np.int64)
    for g in range(len(counts)):
        out[off[g]:off[g + 1]] = x1[off[g]:off[g + 1]].astype(np.int64) @ w[g].astype(np.int64)
    return out


@SETTINGS
@given(grouped())
def test_accum_is_numpy_matmul_per_group(oracle, case):
    e, counts, k, n, rng = case
    m = int(counts.sum()) + 2                                 # two rows past the total
    x1 = rng.integers(-128, 128, size=(m, k), dtype=np.int8)
    w = rng.integers(-128, 128, size=(e, k, n), dtype=np.int8)
    ref = _numpy_acc(x1, w, counts)
    total = int(counts.sum())
    got = oracle.accum(x1, w, counts, 1).astype(np.int64)
    np.testing.assert_array_equal(got[:total], ref[:total])
    got0 = oracle.accum(x1, w, np.cumsum(counts), 0).astype(np.int64)
    np.testing.assert_array_equal(got0[:total], ref[:total])


@SETTINGS
@given(grouped())
def test_int4_words_equal_their_unpacked_nibbles(oracle, case):
    """Word j//8 of a row holds column j in bits 4*(j%8) .. +3, two's complement."""
    e, counts, k, n, rng = case
    m = int(counts.sum())
    x1 = rng.integers(-128, 128, size=(max(m, 1), k), dtype=np.int8)
    words = rng.integers(0, 2 ** 32, size=(e, k, n // 8), dtype=np.uint64).astype(np.uint32)
    shifts = (4 * np.arange(8, dtype=np.uint32))
    nib = ((words[..., None] >> shifts) & 0xF).astype(np.int16)           # (e, k, n/8, 8)
    w8 = np.where(nib >= 8, nib - 16, nib).reshape(e, k, n).astype(np.int8)
    got = oracle.accum(x1, words.view(np.int32), counts, 1, weight="int4").astype(np.int64)
    np.testing.assert_array_equal(got[:m], _numpy_acc(x1, w8, counts)[:m])


@SETTINGS
@given(grouped())
def test_transposed_weights_same_result(oracle, case):
    e, counts, k, n, rng = case
    m = max(int(counts.sum()), 1)
    x1 = rng.integers(-127, 128, size=(m, k), dtype=np.int8)
    w = rng.integers(-127, 128, size=(e, k, n), dtype=np.int8)
    scale = rng.uniform(1e-3, 1e-2, size=(e, n)).astype(np.float32)
    ri = rng.integers(0, 3, size=m).astype(np.int64)
    a = oracle.finalize(x1, w, counts, 1, scale=scale, row_index=ri, output_bs=3)
    b = oracle.finalize(x1, np.ascontiguousarray(np.swapaxes(w, 1, 2)), counts, 1, scale=scale, row_index=ri,
                        output_bs=3, transpose_x2=True)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


@SETTINGS
@given(grouped(), st.integers(1, 6))
def test_destination_relabelling_permutes_output_rows(oracle, case, obs):
    """Renaming destination rows by a permutation permutes the output rows, bit for bit
    (each row's contributions and their ascending source order are unchanged)."""
    e, counts, k, n, rng = case
    m = max(int(counts.sum()), 1)
    x1 = rng.integers(-127, 128, size=(m, k), dtype=np.int8)
    w = rng.integers(-127, 128, size=(e, k, n), dtype=np.int8)
    kw = dict(scale=rng.uniform(1e-3, 1e-2, size=(e, n)).astype(np.float32),
              pertoken_scale=rng.uniform(1e-3, 1e-2, size=m).astype(np.float32),
              logit=rng.uniform(0.05, 1.0, size=m).astype(np.float32),
              bias=rng.normal(0, 0.01, size=(e, n)).astype(np.float32), output_bs=obs)
    ri = rng.integers(0, obs, size=m).astype(np.int64)
    perm = rng.permutation(obs)
    o64, _, o32 = oracle.finalize(x1, w, counts, 1, row_index=ri, **kw)
    p64, _, p32 = oracle.finalize(x1, w, counts, 1, row_index=perm[ri], **kw)
    np.testing.assert_array_equal(p32[perm], o32)
    np.testing.assert_array_equal(p64[perm], o64)


@SETTINGS
@given(grouped())
def test_power_of_two_logit_scales_exactly(oracle, case):
    """Multiplying every logit by 4 multiplies each contribution, and so each f32 sum,
    by exactly 4 (no shared input: every term scales)."""
    e, counts, k, n, rng = case
    m = max(int(counts.sum()), 1)
    x1 = rng.integers(-127, 128, size=(m, k), dtype=np.int8)
    w = rng.integers(-127, 128, size=(e, k, n), dtype=np.int8)
    kw = dict(scale=rng.uniform(1e-3, 1e-2, size=(e, n)).astype(np.float32),
              bias=rng.normal(0, 0.01, size=(e, n)).astype(np.float32),
              row_index=rng.integers(0, 2, size=m).astype(np.int64), output_bs=2)
    lg = rng.uniform(0.05, 1.0, size=m).astype(np.float32)
    _, _, o32 = oracle.finalize(x1, w, counts, 1, logit=lg, **kw)
    _, _, q32 = oracle.finalize(x1, w, counts, 1, logit=lg * np.float32(4), **kw)
    np.testing.assert_array_equal(q32, o32 * np.float32(4))
