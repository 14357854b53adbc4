"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test names what fixes the expected value: the worked example printed on
the PER_TOKEN matmul page, numpy's integer matmul (a library routine), closed
forms of special cases, exact algebraic invariants, or a hand-worked case.
"""
import json
import os

import numpy as np
import pytest

from synth import make_problem
from synth.inputs import make_routing, _layout  # routing only, no weights

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_problem(rng, e, counts, k, n, total_extra=0, weight="int8"):
    m = int(np.sum(counts)) + total_extra
    x1 = rng.integers(-127, 128, size=(m, k), dtype=np.int8)
    if weight == "int8":
        x2 = rng.integers(-127, 128, size=(e, k, n), dtype=np.int8)
    else:
        x2 = rng.integers(0, 2 ** 32, size=(e, k, n // 8), dtype=np.uint32).view(np.int32)
    return x1, x2


def _einsum_acc(x1, x2_int8, counts):
    """Library reference: per-group int64 matmul by numpy."""
    off = np.concatenate([[0], np.cumsum(counts)])
    out = np.zeros((x1.shape[0], x2_int8.shape[2]), np.int64)
    for g in range(len(counts)):
        a, b = off[g], off[g + 1]
        out[a:b] = x1[a:b].astype(np.int64) @ x2_int8[g].astype(np.int64)
    return out


# --- worked example (PER_TOKEN matmul page, 计算示例) --------------------------
@pytest.mark.parametrize("gtype", [0, 1])
def test_worked_example_exact(oracle, gtype):
    g = _golden("per_token_worked_example.json")
    x = np.array(g["x"], np.int8)
    w = np.array(g["weight"], np.int8)[None]              # e = 1
    scale = np.array(g["deqScale"], np.float32)[None]
    pts = np.array(g["perTokenScale"], np.float32)
    expect = np.array(g["output"], np.float64)
    gl = np.array([2], np.int64)                           # both forms: end = count = 2
    o64, sabs, o32 = oracle.finalize(x, w, gl, gtype, scale=scale, pertoken_scale=pts,
                                     row_index=np.array([0, 1], np.int64), output_bs=2)
    np.testing.assert_array_equal(o64, expect)
    np.testing.assert_array_equal(o32.astype(np.float64), expect)
    np.testing.assert_array_equal(oracle.accum(x, w, gl, gtype), [[9, 12, 15], [19, 26, 33]])


# --- BF16 scale (page 1: scaleOptional is FLOAT or BF16) ---------------------
def test_worked_example_with_bf16_scale(oracle):
    """The worked example with deqScale given as bf16 bits.  1.0 = sign 0, exponent
    127, mantissa 0 -> 0x3F80; 2.0 -> exponent 128 -> 0x4000; 3.0 = 1.5 * 2 -> exponent
    128, mantissa 0b1000000 -> 0x4040.  The output is the printed one, exactly."""
    g = _golden("per_token_worked_example.json")
    assert g["deqScale"] == [1, 2, 3]
    x = np.array(g["x"], np.int8)
    w = np.array(g["weight"], np.int8)[None]
    scale_bf16 = np.array([[0x3F80, 0x4000, 0x4040]], np.uint16)
    o64, _, o32 = oracle.finalize(x, w, np.array([2], np.int64), 1, scale=scale_bf16,
                                  pertoken_scale=np.array(g["perTokenScale"], np.float32),
                                  row_index=np.array([0, 1], np.int64), output_bs=2)
    expect = np.array(g["output"], np.float64)
    np.testing.assert_array_equal(o64, expect)
    np.testing.assert_array_equal(o32.astype(np.float64), expect)


def test_bf16_widening_matches_the_format_definition(oracle):
    """Every bf16 bit pattern against the format's definition: sign, 8-bit exponent
    (bias 127), 7-bit fraction; exponent 0 is subnormal (fraction * 2^-133), 255 is
    infinity (fraction 0) or NaN."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):                 # signalling-NaN patterns quieten in the cast
        got = oracle.bf16_to_f32(bits).astype(np.float64)
    b = bits.astype(np.int64)
    sign = np.where(b >> 15, -1.0, 1.0)
    ex, fr = (b >> 7) & 0xFF, b & 0x7F
    normal = sign * (1.0 + fr / 128.0) * np.exp2(np.minimum(ex, 254).astype(np.float64) - 127.0)
    sub = sign * fr * 2.0 ** -133
    want = np.where(ex == 0, sub, np.where(ex == 255, np.where(fr == 0, sign * np.inf, np.nan), normal))
    nan = np.isnan(want)
    assert np.isnan(got[nan]).all()
    np.testing.assert_array_equal(got[~nan], want[~nan])


# --- transposed x2 (page 1, full-quant scenario: (e, n, k)) -----------------
def test_worked_example_with_transposed_weight(oracle):
    """The worked example with its weight [k=2, n=3] given as [n=3, k=2]."""
    g = _golden("per_token_worked_example.json")
    x = np.array(g["x"], np.int8)
    wt = np.array(g["weight"], np.int8).T[None]           # (e=1, n, k)
    o64, _, _ = oracle.finalize(x, wt, np.array([2], np.int64), 1, transpose_x2=True,
                                scale=np.array(g["deqScale"], np.float32)[None],
                                pertoken_scale=np.array(g["perTokenScale"], np.float32),
                                row_index=np.array([0, 1], np.int64), output_bs=2)
    np.testing.assert_array_equal(o64, np.array(g["output"], np.float64))
    np.testing.assert_array_equal(oracle.accum(x, wt, np.array([2], np.int64), 1, transpose_x2=True),
                                  [[9, 12, 15], [19, 26, 33]])


def test_transposed_accum_matches_numpy_matmul(oracle):
    rng = np.random.default_rng(131)
    e, k, n = 3, 64, 24
    counts = np.array([5, 0, 7])
    x1, x2 = _rand_problem(rng, e, counts, k, n)
    x2t = np.ascontiguousarray(np.swapaxes(x2, 1, 2))       # (e, n, k)
    off = np.concatenate([[0], np.cumsum(counts)])
    ref = np.concatenate([x1[off[g]:off[g + 1]].astype(np.int64) @ x2t[g].astype(np.int64).T for g in range(e)])
    np.testing.assert_array_equal(oracle.accum(x1, x2t, counts, 1, transpose_x2=True).astype(np.int64), ref)


# --- deterministic order: the shared value first, then ascending source rows -----
def test_f32_sum_order_is_shared_first_then_ascending_rows(oracle):
    """Hand-worked f32 sums whose result depends on the order.  Three rows reach
    output row 0 with y = 2^24, 1, -2^24: in ascending order 2^24 + 1 rounds back to
    2^24 (ties to even) and the sum is 0; descending, it would be 1.  The exact value
    (f64) is 1.  With a shared value of 2^24 and y = 1, 1: shared first gives 2^24 twice
    rounded back, so 2^24; contributions first would give 2^24 + 2."""
    w = np.ones((1, 1, 1), np.int8)
    t = float(1 << 24)
    o64, _, o32 = oracle.finalize(np.ones((3, 1), np.int8), w, np.array([3], np.int64), 1,
                                  pertoken_scale=np.array([t, 1.0, -t], np.float32),
                                  row_index=np.zeros(3, np.int64), output_bs=1)
    assert o64[0, 0] == 1.0 and o32[0, 0] == 0.0
    shared = np.array([[0x4B80]], np.uint16)                 # bf16 2^24: exponent 151, fraction 0
    o64, _, o32 = oracle.finalize(np.ones((2, 1), np.int8), w, np.array([2], np.int64), 1,
                                  pertoken_scale=np.array([1.0, 1.0], np.float32),
                                  row_index=np.zeros(2, np.int64), output_bs=1, shared=shared, shared_offset=0)
    assert o64[0, 0] == t + 2 and o32[0, 0] == t


def test_f32_dequant_multiplies_scale_first_then_pertoken_scale(oracle):
    """The f32 dequant is (f32(acc) * scale) * pts, two roundings in that order (page
    "matmul支持pertoken量化模式", 计算示例: (x.w) * deqScale * perTokenScale).  Worked
    by hand with u = 2^-23 (spacing u in [1, 2), 2u in [2, 4)), acc = 3,
    scale = 1 + u, pts = 1 + 3u:
      (3 * (1+u)) = 3 + 3u, a tie between 3+2u and 3+4u -> 3+4u (even significand);
      (3+4u) * (1+3u) = 3 + 13u + 12u^2, above the midpoint 3+13u -> 3 + 14u.
    The other orders round to 3 + 12u: (1+u)(1+3u) = 1 + 4u + 3u^2 -> 1+4u, times 3 is
    3+12u exactly; 3(1+3u) = 3+9u, a tie -> 3+8u, times (1+u) = 3+11u+8u^2 -> 3+12u.
    In f32 bits 3 + 14u is 0x40400007 (3.0 is 0x40400000, seven steps of 2u)."""
    u = 2.0 ** -23
    o64, _, o32 = oracle.finalize(np.array([[3]], np.int8), np.ones((1, 1, 1), np.int8), np.array([1], np.int64), 1,
                                  scale=np.array([[1 + u]], np.float32),
                                  pertoken_scale=np.array([1 + 3 * u], np.float32), output_bs=1)
    assert o32.view(np.uint32)[0, 0] == 0x40400007
    assert o64[0, 0] == 3 + 12 * u + 9 * u * u        # exact in double (48 significant bits)
    # bias comes after both scales: acc = 1, scale = 1, pts = 2, bias = 1 -> 1*1*2 + 1 = 3,
    # where adding it before the per-token scale would give (1 + 1) * 2 = 4
    o64, _, o32 = oracle.finalize(np.array([[1]], np.int8), np.ones((1, 1, 1), np.int8), np.array([1], np.int64), 1,
                                  pertoken_scale=np.array([2.0], np.float32), bias=np.array([[1.0]], np.float32),
                                  output_bs=1)
    assert o32[0, 0] == 3.0 and o64[0, 0] == 3.0


def test_int32_to_f32_conversion_rounds_to_nearest_even(oracle):
    """Above 2^24 not every integer is an f32.  Hand-built accumulators, each on its own
    row and weight column, with unit scales (so out = f32(acc)):
      2^24 + 1 = 1040*127*127 + 127*24 + 9*1, a tie between 2^24 and 2^24+2 -> 2^24;
      2^24 + 3 = 1040*127*127 + 127*24 + 11*1, a tie between 2^24+2 and 2^24+4 -> 2^24+4;
      2^25 + 3 = 2080*127*127 + 127*48 + 19*1, spacing 4: nearer 2^25+4 than 2^25
    (truncation would give 2^24, 2^24+2 and 2^25)."""
    k = 2082
    x1 = np.zeros((3, k), np.int8)
    w = np.zeros((1, k, 3), np.int8)
    x1[0, :1041], x1[0, 1041] = 127, 9
    x1[1, :1041], x1[1, 1041] = 127, 11
    w[0, :1040, 0], w[0, 1040, 0], w[0, 1041, 0] = 127, 24, 1
    w[0, :, 1] = w[0, :, 0]
    x1[2, :2081], x1[2, 2081] = 127, 19
    w[0, :2080, 2], w[0, 2080, 2], w[0, 2081, 2] = 127, 48, 1
    gl = np.array([3], np.int64)
    acc = oracle.accum(x1, w, gl, 1)
    assert [acc[c, c] for c in range(3)] == [(1 << 24) + 1, (1 << 24) + 3, (1 << 25) + 3]
    o64, _, o32 = oracle.finalize(x1, w, gl, 1, output_bs=3)
    assert [float(o32[c, c]) for c in range(3)] == [16777216.0, 16777220.0, 33554436.0]
    assert [o64[c, c] for c in range(3)] == [16777217.0, 16777219.0, 33554435.0]


# --- library routine: numpy integer matmul per group ------------------------
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_accum_matches_numpy_matmul(oracle, seed):
    rng = np.random.default_rng(100 + seed)
    e, k, n = 5, 96, 40
    counts = rng.integers(0, 7, size=e)
    counts[1] = 0                                           # an empty expert
    x1, x2 = _rand_problem(rng, e, counts, k, n)
    ref = _einsum_acc(x1, x2, counts)
    for gtype, gl in ((1, counts), (0, np.cumsum(counts))):
        got = oracle.accum(x1, x2, gl.astype(np.int64), gtype)
        np.testing.assert_array_equal(got.astype(np.int64), ref)
    rows = np.array([0, int(counts.sum()) - 1], np.int64)
    np.testing.assert_array_equal(oracle.accum(x1, x2, counts, 1, rows=rows), ref[rows])


def test_accum_extreme_values_exact(oracle):
    """All-(-127) activations against all-127 weights: -k*127*127 exactly."""
    k, n = 2048, 16
    x1 = np.full((3, k), -127, np.int8)
    x2 = np.full((1, k, n), 127, np.int8)
    got = oracle.accum(x1, x2, np.array([3], np.int64), 1)
    assert (got == -k * 127 * 127).all()


def _pack_int4(vals):
    """Independent packing for the test: value j of a word sits in bits 4*(j%8).."""
    e, k, n = vals.shape
    u = (vals.astype(np.int64) & 0xF).reshape(e, k, n // 8, 8)
    words = np.zeros((e, k, n // 8), np.uint64)
    for s in range(8):
        words |= (u[..., s].astype(np.uint64) << np.uint64(4 * s))
    return words.astype(np.uint32).view(np.int32)


def test_int4_path_equals_int8_path(oracle):
    rng = np.random.default_rng(7)
    e, k, n = 3, 64, 48
    counts = np.array([4, 0, 5])
    vals = rng.integers(-8, 8, size=(e, k, n)).astype(np.int8)
    x1 = rng.integers(-127, 128, size=(int(counts.sum()), k), dtype=np.int8)
    a8 = oracle.accum(x1, vals, counts, 1)
    a4 = oracle.accum(x1, _pack_int4(vals), counts, 1, weight="int4")
    np.testing.assert_array_equal(a4, a8)
    np.testing.assert_array_equal(a8.astype(np.int64), _einsum_acc(x1, vals, counts))
    # sign-bit nibble: -8 and 7 are both representable
    assert vals.min() == -8 and vals.max() == 7


# --- closed forms of special cases -------------------------------------------
def test_unit_scales_reduce_to_matmul_plus_index_add(oracle):
    """scale = pts = logit = 1, no bias: out = index_add(rows -> tokens) of the matmul."""
    rng = np.random.default_rng(11)
    tokens, topk, e, k, n = 9, 3, 4, 32, 24
    experts, w = make_routing(rng, tokens, topk, e, "uniform", 0.0)
    ri, logit, counts = _layout(experts, w, e)
    m = tokens * topk
    x1 = rng.integers(-3, 4, size=(m, k), dtype=np.int8)   # keeps every sum exact in f32
    x2 = rng.integers(-3, 4, size=(e, k, n), dtype=np.int8)
    acc = _einsum_acc(x1, x2, counts)
    ref = np.zeros((tokens, n), np.float64)
    np.add.at(ref, ri, acc.astype(np.float64))
    o64, sabs, o32 = oracle.finalize(x1, x2, counts, 1, row_index=ri, output_bs=tokens)
    np.testing.assert_array_equal(o64, ref)
    np.testing.assert_array_equal(o32.astype(np.float64), ref)
    np.testing.assert_array_equal(sabs, _abs_index_add(ri, acc, tokens))


def test_error_magnitude_counts_bias_before_cancellation(oracle):
    """One contribution (3*0.5*2 - 2.5)*4 = 2: the error magnitude is (3 + 2.5)*4 = 22,
    not |2|, because f32 rounding acts on the parts before the bias cancels them."""
    x1 = np.array([[1]], np.int8)
    x2 = np.array([[[3]]], np.int8)
    o64, sabs, o32 = oracle.finalize(
        x1, x2, np.array([1], np.int64), 1, scale=np.array([[0.5]], np.float32),
        pertoken_scale=np.array([2.0], np.float32), logit=np.array([4.0], np.float32),
        bias=np.array([[-2.5]], np.float32), row_index=np.array([0], np.int64), output_bs=1)
    assert o64[0, 0] == 2.0 and o32[0, 0] == 2.0
    assert sabs[0, 0] == 22.0


def _abs_index_add(ri, acc, tokens):
    out = np.zeros((tokens, acc.shape[1]), np.float64)
    np.add.at(out, ri, np.abs(acc).astype(np.float64))
    return out


def test_shared_input_alone_lands_at_offset(oracle):
    """x1 = 0 and no bias: the output is the bf16 sharedInput rows at the offset, zeros elsewhere."""
    rng = np.random.default_rng(5)
    e, k, n, m, out_bs, bs, off = 2, 16, 32, 6, 10, 4, 3
    x1 = np.zeros((m, k), np.int8)
    x2 = rng.integers(-127, 128, size=(e, k, n), dtype=np.int8)
    sh_f = rng.standard_normal((bs, n)).astype(np.float32)
    sh = (sh_f.view(np.uint32) >> 16).astype(np.uint16)   # truncate to bf16 bits
    sh_exact = (sh.astype(np.uint32) << 16).view(np.float32)
    ri = rng.integers(0, out_bs, size=m).astype(np.int64)
    o64, _, o32 = oracle.finalize(x1, x2, np.array([2, 4], np.int64), 1,
                                  scale=np.ones((e, n), np.float32), logit=np.full(m, 0.5, np.float32),
                                  row_index=ri, shared=sh, shared_offset=off, output_bs=out_bs)
    ref = np.zeros((out_bs, n), np.float32)
    ref[off:off + bs] = sh_exact
    np.testing.assert_array_equal(o32, ref)
    np.testing.assert_array_equal(o64, ref.astype(np.float64))


def test_bias_sits_inside_the_routing_weight(oracle):
    """One row, scale = pts = 1, logit = 2: out = 2 * (acc + bias) (reading: bias before logit)."""
    rng = np.random.default_rng(9)
    k, n = 8, 16
    x1 = rng.integers(-5, 6, size=(1, k), dtype=np.int8)
    x2 = rng.integers(-5, 6, size=(1, k, n), dtype=np.int8)
    bias = np.array(rng.integers(-64, 64, size=(1, n)), np.float32) / 8   # exact in f32
    acc = x1.astype(np.int64) @ x2[0].astype(np.int64)
    o64, _, o32 = oracle.finalize(x1, x2, np.array([1], np.int64), 1, bias=bias,
                                  logit=np.array([2.0], np.float32), output_bs=1)
    np.testing.assert_array_equal(o64, 2.0 * (acc + bias.astype(np.float64)))
    np.testing.assert_array_equal(o32.astype(np.float64), 2.0 * (acc + bias.astype(np.float64)))


# --- invariants --------------------------------------------------------------
def test_logit_doubling_doubles_output_exactly(oracle):
    p = make_problem("tiny", n=64)
    a64, _, a32 = oracle.problem_finalize(p)
    p.logit = (p.logit * np.float32(2)).astype(np.float32)
    b64, _, b32 = oracle.problem_finalize(p)
    np.testing.assert_array_equal(b64, 2 * a64)
    np.testing.assert_array_equal(b32, 2 * a32)


def test_group_list_forms_agree_and_empty_experts_change_nothing(oracle):
    p = make_problem("tiny", n=64, e=6)
    base = oracle.problem_finalize(p)
    counts = p.counts
    alt = oracle.finalize(p.x1, p.x2, np.cumsum(counts), 0, scale=p.scale,
                          pertoken_scale=p.pertoken_scale, logit=p.logit, row_index=p.row_index,
                          output_bs=p.output_bs)
    for a, b in zip(base, alt):
        np.testing.assert_array_equal(a, b)
    # insert two empty experts (with arbitrary weights) in front and in the middle
    rng = np.random.default_rng(3)
    junk = rng.integers(-127, 128, size=(1, p.k, p.n), dtype=np.int8)
    x2b = np.concatenate([junk, p.x2[:3], junk, p.x2[3:]])
    scb = np.concatenate([p.scale[:1], p.scale[:3], p.scale[:1], p.scale[3:]])
    cb = np.concatenate([[0], counts[:3], [0], counts[3:]]).astype(np.int64)
    ins = oracle.finalize(p.x1, x2b, cb, 1, scale=scb, pertoken_scale=p.pertoken_scale,
                          logit=p.logit, row_index=p.row_index, output_bs=p.output_bs)
    for a, b in zip(base, ins):
        np.testing.assert_array_equal(a, b)


def test_rows_past_the_total_are_ignored(oracle):
    rng = np.random.default_rng(21)
    e, k, n = 3, 32, 16
    counts = np.array([2, 3, 1])
    x1, x2 = _rand_problem(rng, e, counts, k, n, total_extra=4)
    ri = np.arange(x1.shape[0], dtype=np.int64) % 5
    a = oracle.finalize(x1, x2, counts, 1, row_index=ri, output_bs=5)
    x1b = x1.copy()
    x1b[6:] = rng.integers(-127, 128, size=(4, k), dtype=np.int8)
    ri_b = ri.copy()
    ri_b[6:] = 4
    b = oracle.finalize(x1b, x2, counts, 1, row_index=ri_b, output_bs=5)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_int32_row_index_same_as_int64(oracle):
    p = make_problem("tiny", n=64)
    a = oracle.problem_finalize(p)
    p.row_index = p.row_index.astype(np.int32)
    b = oracle.problem_finalize(p)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_f32_order_within_rounding_of_f64(oracle):
    p = make_problem("tiny")
    o64, sabs, o32 = oracle.problem_finalize(p)
    err = np.abs(o32.astype(np.float64) - o64) / np.maximum(sabs, 1e-30)
    assert err.max() < 8 * 2.0 ** -24 * 4


def test_dest_row_subset_matches_full(oracle):
    p = make_problem("tiny", n=128)
    full = oracle.problem_finalize(p)
    rows = np.array([0, 5, 17, 31], np.int64)
    sub = oracle.problem_finalize(p, dest_rows=rows)
    for f, s in zip(full, sub):
        np.testing.assert_array_equal(f[rows], s)


@pytest.mark.parametrize("name", ["tiny", "mid_prefill", "decode", "large_prefill", "w4a8_prologue"])
def test_routing_invariants(name):
    """Sum of counts = m and every output row receives exactly topK contributions."""
    from synth.inputs import CONFIGS, SEED_BASE
    s = CONFIGS[name]
    rng = np.random.default_rng(SEED_BASE + s.index)
    experts, w = make_routing(rng, s.tokens, s.topk, s.e, s.routing, s.routing_param)
    ri, logit, counts = _layout(experts, w, s.e)
    assert counts.sum() == s.tokens * s.topk
    assert (np.bincount(ri, minlength=s.tokens) == s.topk).all()
    # each token's slots go to distinct experts
    assert all(len(set(r)) == s.topk for r in experts[:256])
    # logit rows per token sum to one (softmax weights)
    sums = np.zeros(s.tokens)
    np.add.at(sums, ri, logit.astype(np.float64))
    np.testing.assert_allclose(sums, 1.0, rtol=1e-6)


# --- groupList validation (parameter constraints, page 1) --------------------
def test_group_list_errors(oracle):
    m = 10
    with pytest.raises(oracle.OracleError) as ei:
        oracle.group_offsets(np.array([2, -1, 3]), 1, m)
    assert ei.value.code == oracle.QO_ERR_NEGATIVE_COUNT
    with pytest.raises(oracle.OracleError) as ei:
        oracle.group_offsets(np.array([2, 5, 4]), 0, m)
    assert ei.value.code == oracle.QO_ERR_NOT_MONOTONE
    with pytest.raises(oracle.OracleError) as ei:
        oracle.group_offsets(np.array([6, 5]), 1, m)
    assert ei.value.code == oracle.QO_ERR_TOTAL_GT_M
    np.testing.assert_array_equal(oracle.group_offsets(np.array([2, 2, 7]), 0, m), [0, 2, 2, 7])
    np.testing.assert_array_equal(oracle.group_offsets(np.array([2, 0, 5]), 1, m), [0, 2, 2, 7])


# --- per-token quant ---------------------------------------------------------
def _bf16_bits(vals):
    v = np.asarray(vals, np.float32)
    bits = v.view(np.uint32)
    assert ((bits & 0xFFFF) == 0).all(), "test values must be exact in bf16"
    return (bits >> 16).astype(np.uint16)


def test_per_token_quant_hand_cases(oracle):
    # absmax 127 gives inverse exactly 1, so q = round-half-even(x): 2.5->2, 3.5->4, -2.5->-2, 0.5->0
    row0 = [127.0, 2.5, 3.5, -2.5, 0.5, 1.5, -127.0, 0.0]
    # absmax 2: inverse 63.5; 2 -> 127, -1 -> -63.5 -> -64, 0.5 -> 31.75 -> 32, 0.25 -> 15.875 -> 16
    row1 = [2.0, -1.0, 0.5, 0.25, 0.0, -2.0, 1.0, 0.125]
    row2 = [0.0] * 8
    q, pts = oracle.per_token_quant(_bf16_bits([row0, row1, row2]))
    np.testing.assert_array_equal(q[0], [127, 2, 4, -2, 0, 2, -127, 0])
    np.testing.assert_array_equal(q[1], [127, -64, 32, 16, 0, -127, 64, 8])
    np.testing.assert_array_equal(q[2], 0)
    assert pts[0] == np.float32(1.0)
    assert pts[1] == np.float32(2.0) / np.float32(127.0)
    assert pts[2] == 0.0


def test_per_token_quant_non_finite_inputs(oracle):
    """Reading for inputs the pages do not cover, with IEEE f32 semantics: the absmax
    skips NaN; an infinity makes absmax = pts = inf and the inverse 0; a NaN product
    (NaN input, or inf * 0) quantises to 0.
      row 0: 1, NaN, -2, 0.5 -> absmax 2, inverse 63.5: 63.5 -> 64 (tie to even),
             NaN -> 0, -127, 31.75 -> 32; pts = 2/127
      row 1: +inf, 1, -3 -> pts inf, every code 0 (inf * 0 is NaN, 1 * 0 = 0)
      row 2: -inf, NaN, 5 -> pts inf, every code 0
      row 3: all NaN -> absmax 0, pts 0, inverse 0, every code 0"""
    nan, pinf, ninf = 0x7FC0, 0x7F80, 0xFF80
    x = np.zeros((4, 8), np.uint16)
    x[0, [0, 2, 3]] = _bf16_bits([1.0, -2.0, 0.5])
    x[0, 1] = nan
    x[0, 4] = nan                                                # a NaN after the row's max as well
    x[1, 0] = pinf
    x[1, 1:3] = _bf16_bits([1.0, -3.0])
    x[2, :2] = [ninf, nan]
    x[2, 2] = _bf16_bits([5.0])[0]
    x[3, :] = nan
    q, pts = oracle.per_token_quant(x)
    np.testing.assert_array_equal(q[0], [64, 0, -127, 32, 0, 0, 0, 0])   # element 4 is the second NaN
    np.testing.assert_array_equal(q[1:], 0)
    assert pts[0] == np.float32(2.0) / np.float32(127.0)
    assert pts[1] == np.inf and pts[2] == np.inf and pts[3] == 0.0


def test_per_token_quant_bounds(oracle):
    from synth.inputs import bf16_bits_normal
    rng = np.random.default_rng(17)
    x = bf16_bits_normal(rng, (64, 512))
    q, pts = oracle.per_token_quant(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.abs(q).max() <= 127
    assert (np.abs(q).max(axis=1) == 127).all()
    np.testing.assert_array_equal(pts, (np.abs(xf).max(axis=1).astype(np.float32) / np.float32(127)))
    recon = q.astype(np.float64) * pts.astype(np.float64)[:, None]
    assert (np.abs(xf - recon) <= pts.astype(np.float64)[:, None] * 0.50002).all()


# --- per-32-group FP8 E4M3 cast ----------------------------------------------
def test_e4m3_codes_against_the_format_definition(oracle):
    """E4M3FN: sign, 4 exponent bits with bias 7, 3 fraction bits, subnormals m * 2^-9
    at exponent 0, S.1111.111 NaN, no infinities, largest finite 1.75 * 2^8 = 448.
    Hand-known codes; every non-NaN code round-trips; the finite codes increase
    strictly; each midpoint between neighbours rounds to the even code (the code's
    last bit is the fraction's); and torch's float8_e4m3fn conversion (a library
    routine, round to nearest even) agrees on random in-range values."""
    known = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3C: 1.5, 0x40: 2.0,
             0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for c, v in known.items():
        assert oracle.e4m3_decode(c) == v and oracle.e4m3_encode(v) == c, hex(c)
    assert np.isnan(oracle.e4m3_decode(0x7F)) and np.isnan(oracle.e4m3_decode(0xFF))
    assert oracle.e4m3_encode(-0.0) == 0x80 and oracle.e4m3_encode(float("nan")) == 0x7F
    finite = [c for c in range(256) if c & 0x7F != 0x7F]
    for c in finite:
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)
    vals = [oracle.e4m3_decode(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    for c in range(0x7E):
        mid = np.float32((vals[c] + vals[c + 1]) / 2)            # exact: one more fraction bit
        assert oracle.e4m3_encode(float(mid)) == (c if c % 2 == 0 else c + 1), hex(c)
    for v in (449.0, 463.9, 464.0, 1e6, float("inf")):           # saturation, not NaN
        assert oracle.e4m3_encode(v) == 0x7E and oracle.e4m3_encode(-v) == 0xFE
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 2.0 ** rng.integers(-12, 8, 4000),
                        [(vals[c] + vals[c + 1]) / 2 for c in range(0x7E)]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_mxfp8_cast_hand_worked_groups(oracle):
    """One row of four 32-element groups (reading: an E8M0 scale per group whose
    exponent puts the group's largest magnitude in E4M3's top binade).
      group 0: 1.0, -0.30078125, 0.5 -> amax 1 (f32 exponent 127), sf = 119, x * 2^8:
               256 -> 0x78; -77 = -2^6 * 1.203 -> fraction 1.625/8 rounds to 2/8 -> -80 -> 0xEA;
               128 -> 0x70
      group 1: 3.0, 1.75, 0.00099945 -> amax 3 (exponent 128), sf = 120, x * 2^7:
               384 = 1.5 * 2^8 -> 0x7C; 224 = 1.75 * 2^7 -> 0x76; 0.1279 = 1.023 * 2^-3 -> 0x20
      group 2: 460 (exponent 135), sf = 127, x * 1 = 460 past 448 -> saturates to 0x7E
      group 3: all zero -> sf = 0, codes 0"""
    x = np.zeros((1, 128), np.uint16)
    x[0, [0, 1, 2]] = [0x3F80, 0xBE9A, 0x3F00]
    x[0, [32, 33, 34]] = [0x4040, 0x3FE0, 0x3A83]
    x[0, 64] = 0x43E6                                            # 460 = 1.796875 * 2^8
    q, sf = oracle.per_token_quant_mxfp8(x)
    np.testing.assert_array_equal(sf[0], [119, 120, 127, 0])
    np.testing.assert_array_equal(q[0, :3], [0x78, 0xEA, 0x70])
    np.testing.assert_array_equal(q[0, 32:35], [0x7C, 0x76, 0x20])
    assert q[0, 64] == 0x7E
    assert (q[0, 3:32] == 0).all() and (q[0, 35:64] == 0).all() and (q[0, 65:] == 0).all()


def test_mxfp8_cast_bounds_and_non_finite(oracle):
    """Every group's largest magnitude lands in [256, 448] (E4M3's top binade, or the
    saturated 448); |x - q * 2^(sf-127)| is at most half an E4M3 step (2^-4 of the
    element's binade, 2^-9 on the subnormal grid) after scaling, except where the
    top element saturated.  Non-finite inputs: NaN is skipped by the group's absmax
    and encodes as 0x7F; an infinity makes sf = 247 (f32 exponent 255 - 8) and
    saturates to 448 while the group's finite values scale to 0."""
    from synth.inputs import bf16_bits_normal
    x = bf16_bits_normal(np.random.default_rng(23), (16, 256))
    q, sf = oracle.per_token_quant_mxfp8(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(16, 8, 32)
    dq = np.vectorize(oracle.e4m3_decode)(q).astype(np.float64).reshape(16, 8, 32)
    scaled = xf * np.exp2(127.0 - sf.astype(np.float64))[:, :, None]
    top = np.abs(dq).max(axis=2)
    assert ((top >= 256) & (top <= 448)).all()
    step = np.where(np.abs(scaled) < 2.0 ** -6, 2.0 ** -9, np.exp2(np.floor(np.log2(np.maximum(np.abs(scaled),
                                                                                            1e-300))) - 3))
    ok = (np.abs(scaled - dq) <= step / 2) | (np.abs(dq) == 448)
    assert ok.all()
    y = np.zeros((1, 64), np.uint16)
    y[0, :4] = [0x7FC0, 0x3F80, 0xC000, 0x7FC0]                   # NaN, 1, -2, NaN (after the max too)
    y[0, 32:34] = [0x7F80, 0x3F80]                                # +inf, 1
    q, sf = oracle.per_token_quant_mxfp8(y)
    assert sf[0, 0] == 120 and q[0, 0] == 0x7F and q[0, 1] == 0x70 and q[0, 2] == 0xF8 and q[0, 3] == 0x7F
    assert sf[0, 1] == 247 and q[0, 32] == 0x7E and q[0, 33] == 0


# --- FP8 E4M3 operands (Atlas 350 per-token / per-channel mode) ----------------
def test_worked_example_in_fp8(oracle):
    """The worked example of "matmul支持pertoken量化模式", 计算示例, with x and w given
    as FLOAT8 E4M3 codes (1, 2, 3, 4, 5, 6 are exact E4M3 values: 0x38, 0x40, 0x44,
    0x48, 0x4A, 0x4C): the same output [[9, 24, 45], [38, 104, 198]]."""
    g = _golden("per_token_worked_example.json")
    code = {1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48, 5: 0x4A, 6: 0x4C}
    x = np.vectorize(code.get)(np.array(g["x"])).astype(np.uint8)
    w = np.vectorize(code.get)(np.array(g["weight"])).astype(np.uint8)[None]
    for gtype, gl in ((0, [2]), (1, [2])):
        o64, _, o32 = oracle.finalize(x, w, np.array(gl, np.int64), gtype, weight="fp8",
                                      scale=np.array([g["deqScale"]], np.float32),
                                      pertoken_scale=np.array(g["perTokenScale"], np.float32),
                                      row_index=np.array([0, 1], np.int64), output_bs=2)
        np.testing.assert_array_equal(o64, g["output"])
        np.testing.assert_array_equal(o32, np.array(g["output"], np.float32))


def test_fp8_accum_matches_library_matmul_and_is_exact(oracle):
    """Accumulators of E4M3 operands equal numpy's float64 matmul of the values that
    torch's float8_e4m3fn decoding gives (library routines), group by group; and a
    sum whose exact value needs more than f32's 24 bits (448*448 + 2^-9*2^-9) is
    exact; the magnitude is the sum of |products|."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(41)
    counts = np.array([5, 0, 9, 3], np.int64)
    m, k, n, e = 17, 64, 24, 4
    x1 = rng.integers(0, 256, (m, k), dtype=np.uint8)
    x2 = rng.integers(0, 256, (e, k, n), dtype=np.uint8)
    x1[(x1 & 0x7F) == 0x7F] = 0x38                             # no NaN codes
    x2[(x2 & 0x7F) == 0x7F] = 0xB8
    dec = lambda a: torch.from_numpy(a).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    acc, mag = oracle.accum_f8(x1, x2, counts, 1)
    off = np.concatenate([[0], np.cumsum(counts)])
    for g in range(e):
        r = slice(off[g], off[g + 1])
        np.testing.assert_array_equal(acc[r], dec(x1[r]) @ dec(x2[g]))
        np.testing.assert_array_equal(mag[r], np.abs(dec(x1[r])) @ np.abs(dec(x2[g])))
    assert (acc[off[-1]:] == 0).all()
    a = np.array([[0x7E, 0x01]], np.uint8)                      # 448, 2^-9
    w = np.array([[[0x7E], [0x01]]], np.uint8)
    acc, _ = oracle.accum_f8(a, w, np.array([1], np.int64), 1)
    assert acc[0, 0] == 448.0 * 448.0 + 2.0 ** -18 and np.float32(acc[0, 0]) == 200704.0


# --- MxA8W4: E4M3 activations, E2M1 weights, E8M0 scales per 32 k -------------
def test_e2m1_and_e8m0_code_points(oracle):
    """FP4 E2M1 (sign, 2 exponent bits with bias 1, 1 fraction bit, subnormal 0.5 at
    exponent 0): the 16 code points by hand.  E8M0 (2^(c-127), 0xFF NaN): every code
    against torch's float8_e8m0fnu decoding (a library routine)."""
    vals = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        v = oracle.e2m1_decode(c)
        assert v == (-vals[c - 8] if c >= 8 else vals[c]) and (np.signbit(v) == (c >= 8)), c
    torch = pytest.importorskip("torch")
    codes = np.arange(255, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    np.testing.assert_array_equal([oracle.e8m0_decode(int(c)) for c in codes], ref)
    assert np.isnan(oracle.e8m0_decode(0xFF))


def test_mx_hand_worked_blocks(oracle):
    """One row, one output column, k = 64 (two blocks of 32), by hand:
      block 0: x = 1.0 (0x38) everywhere, w = 1.5 (nibble 3) everywhere: sum 48;
               scales 2^0 (127) and 2^1 (128): 96
      block 1: x[32] = 2.0 (0x40), x[33] = 1.0, the rest 0; w[32] = -6 (nibble 0xF, the
               byte's low nibble: even k), w[33] = 0.5 (nibble 1, high nibble): sum
               -12 + 0.5 = -11.5; scales 2^-1 (126) and 2^0: -5.75
      acc = 90.25; bias 1, logit 0.5: (90.25 + 1) * 0.5 = 45.625.
    The other nibble order would give block 1 = 2*0.5 + 1*(-6) = -5 -> out 47.25."""
    x1 = np.zeros((1, 64), np.uint8)
    x1[0, :32] = 0x38
    x1[0, 32], x1[0, 33] = 0x40, 0x38
    w = np.zeros((1, 1, 32), np.uint8)
    w[0, 0, :16] = 0x33
    w[0, 0, 16] = 0x1F                                  # k = 32: low nibble 0xF, k = 33: high nibble 1
    sfa = np.array([[127, 126]], np.uint8)
    sfb = np.array([[[128, 127]]], np.uint8)
    acc, mag = oracle.accum_mx(x1, sfa, w, sfb, np.array([1], np.int64), 1)
    assert acc[0, 0] == 90.25 and mag[0, 0] == 96 + 0.5 * 12.5
    o64, sabs, o32 = oracle.finalize_mx(x1, sfa, w, sfb, np.array([1], np.int64), 1,
                                        logit=np.array([0.5], np.float32), bias=np.array([[1.0]], np.float32),
                                        output_bs=1)
    assert o64[0, 0] == 45.625 and o32[0, 0] == np.float32(45.625)


def test_mx_accum_matches_blockwise_library_matmul(oracle):
    """Accumulators against numpy float64 matmuls, block by block, of torch-decoded E4M3
    activations and E2M1 weights (decoded through a table of the 16 code points),
    scaled by torch-decoded E8M0 scales, with empty and ragged groups."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(77)
    counts = np.array([3, 0, 6, 2], np.int64)
    m, k, n, e = 13, 96, 10, 4
    x1 = rng.integers(0, 256, (m, k), dtype=np.uint8)
    x1[(x1 & 0x7F) == 0x7F] = 0x30
    w = rng.integers(0, 256, (e, n, k // 2), dtype=np.uint8)
    sfa = rng.integers(118, 136, (m, k // 32), dtype=np.uint8)
    sfb = rng.integers(118, 136, (e, n, k // 32), dtype=np.uint8)
    table = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])
    wv = np.empty((e, n, k))
    wv[:, :, 0::2] = table[w & 0xF]
    wv[:, :, 1::2] = table[w >> 4]
    xv = torch.from_numpy(x1).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    e8 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    acc, _ = oracle.accum_mx(x1, sfa, w, sfb, counts, 1)
    off = np.concatenate([[0], np.cumsum(counts)])
    for g in range(e):
        r = slice(off[g], off[g + 1])
        ref = np.zeros((counts[g], n))
        for b in range(k // 32):
            kb = slice(32 * b, 32 * b + 32)
            ref += (xv[r, kb] @ wv[g][:, kb].T) * e8(sfa[r, b])[:, None] * e8(sfb[g, :, b])[None, :]
        np.testing.assert_allclose(acc[r], ref, rtol=1e-13, atol=0)
    assert (acc[off[-1]:] == 0).all()
