"""Pins of the CPU oracle against what the pages and mathematics fix (no GPU).

Each test ties the C oracle to something other than itself: exact integer facts, a library routine
on a special case that reduces to it, closed forms, invariants, or the independent dense restatement
of the HSTULayer sketch ("4.4 推荐模型的 Scaling").  The equations are those of "Actions Speak Louder
than Words" (paper notes), section 3.1, Eqs. 1-3.
"""
import math

import numpy as np
import pytest

import oracle
from oracle.dense_ref import hstu_layer_dense
from workloads import random_case, to_bf16_bits, widen_bf16, make_inputs


def _silu(x):
    return x / (1.0 + np.exp(-x))


def _run(inp, layer=0, **kw):
    return oracle.layer_fwd_inputs(inp, layer=layer, **kw)


def _dense(inp, layer=0):
    w, p = inp.workload, inp.layers[layer]
    return hstu_layer_dense(inp.lengths, inp.X, p.W1, p.b1, p.W2, p.b2, p.ln_w, p.ln_b,
                            num_heads=w.num_heads, d_qk=w.head_dim, d_v=w.head_dim,
                            timestamps=inp.timestamps, pos_table=inp.pos_table,
                            time_table=inp.time_table, alibi_slopes=inp.alibi_slopes,
                            scale=inp.scale, ln_eps=inp.ln_eps)


# ----------------------------------------------------------------------------------------------
# Bucket indices: exact integer facts
# ----------------------------------------------------------------------------------------------

def test_time_bucket_is_floor_log2_of_one_plus_delta():
    # floor(log2(1 + delta)) is (1 + delta).bit_length() - 1 for integers
    for delta in [0, 1, 2, 3, 4, 6, 7, 8, 59, 60, 1023, 1024, 86399, 2**31 - 2, 2**31 - 1,
                  2**40 - 1, 2**40, 2**62]:
        expect = min((1 + delta).bit_length() - 1, 127)
        assert oracle.time_bucket(10**6 + delta, 10**6, 128) == expect, delta
    # known small values written out
    assert [oracle.time_bucket(d, 0, 64) for d in range(8)] == [0, 1, 1, 2, 2, 2, 2, 3]
    # clamp to the last bucket, and negative differences count as zero
    assert oracle.time_bucket(2**40, 0, 32) == 31
    assert oracle.time_bucket(5, 9, 32) == 0


def test_pos_bucket_clamps_to_last():
    assert [oracle.pos_bucket(i, 0, 4) for i in range(7)] == [0, 1, 2, 3, 3, 3, 3]
    assert oracle.pos_bucket(10, 3, 100) == 7
    assert oracle.pos_bucket(8191, 0, 8192) == 8191


def test_round_bf16_ties_to_even():
    # bf16 keeps 8 significant bits: the spacing just above 1 is 2^-7
    assert oracle.round_bf16(1.0 + 2**-8) == 1.0                      # tie -> even (1.0)
    assert oracle.round_bf16(1.0 + 3 * 2**-8) == 1.0 + 2**-6         # tie -> even (..10)
    assert oracle.round_bf16(1.0 + 2**-8 + 2**-20) == 1.0 + 2**-7    # above the tie
    assert oracle.round_bf16(-3.0) == -3.0
    assert oracle.round_bf16(0.0) == 0.0
    # agrees with the bit-level rounding of the input generator on float32 values
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 6, 2000)).astype(np.float32)
    ours = np.array([oracle.round_bf16(float(v)) for v in x])
    ref = widen_bf16(to_bf16_bits(x))
    np.testing.assert_array_equal(ours, ref)


# ----------------------------------------------------------------------------------------------
# Brute force: the dense padded restatement of the sketch, on tiny inputs
# ----------------------------------------------------------------------------------------------

CASES = [
    dict(seed=1, lengths=[5], d=8, H=2, hd=4),
    dict(seed=2, lengths=[3, 16, 1], d=16, H=2, hd=8),
    dict(seed=3, lengths=[7, 0, 12], d=12, H=3, hd=4),
    dict(seed=4, lengths=[16, 9], d=8, H=1, hd=8, P=4, Tb=3),   # clamping of both buckets
    dict(seed=5, lengths=[11, 13], d=16, H=4, hd=4, alibi=True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"seed{c['seed']}")
def test_oracle_matches_dense_restatement(case):
    inp = random_case(**case)
    y = _run(inp)
    y_dense = _dense(inp)
    # both fp64; only the summation order differs
    assert np.max(np.abs(y - y_dense)) <= 1e-12 * max(1.0, np.max(np.abs(y_dense)))
    # the attention must matter in these cases (the comparison is not vacuous)
    _, _, av, _ = _run(inp, return_intermediates=True)
    assert np.max(np.abs(av)) > 1e-3


@pytest.mark.parametrize("which", ["pos", "time", "none"])
def test_oracle_matches_dense_restatement_partial_bias(which):
    inp = random_case(seed=6, lengths=[9, 14], d=8, H=2, hd=4, P=6, Tb=5)
    if which != "pos":
        inp.time_table = inp.time_table if which == "time" else None
        inp.pos_table = None
    else:
        inp.time_table = None
    y, y_dense = _run(inp), _dense(inp)
    assert np.max(np.abs(y - y_dense)) <= 1e-12 * np.max(np.abs(y_dense))


def test_dense_restatement_sees_the_bias():
    # sanity of the brute force itself: changing one bucket of a table changes the output
    inp = random_case(seed=8, lengths=[10], d=8, H=2, hd=4, P=16, Tb=8)
    y0 = _dense(inp)
    inp.pos_table = inp.pos_table.copy()
    inp.pos_table[1, 3] += 1.0
    y1 = _dense(inp)
    assert np.max(np.abs(y1 - y0)) > 1e-6


# ----------------------------------------------------------------------------------------------
# Library special cases: the projections are matmuls, checked against numpy's
# ----------------------------------------------------------------------------------------------

def test_projections_against_numpy_matmul():
    inp = random_case(seed=9, lengths=[20, 7], d=16, H=2, hd=8)
    p = inp.layers[0]
    y, uvqk, av, g = _run(inp, return_intermediates=True)
    X = inp.X.astype(np.float64)
    z = X @ p.W1.astype(np.float64) + p.b1
    np.testing.assert_allclose(uvqk, _silu(z), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(y, g @ p.W2.astype(np.float64) + p.b2 + X, rtol=1e-13, atol=1e-13)


def test_layernorm_statistics():
    # G / U = LN(AV): per row mean ln_b-free part 0 and variance var/(var+eps) when ln_w=1, ln_b=0
    inp = random_case(seed=10, lengths=[12, 5], d=16, H=2, hd=8)
    p = inp.layers[0]
    p.ln_w[:] = 1.0
    p.ln_b[:] = 0.0
    _, uvqk, av, g = _run(inp, return_intermediates=True)
    wv = av.shape[1]
    n = g / uvqk[:, :wv]                     # U is block 0
    var = av.var(axis=1)
    np.testing.assert_allclose(n.mean(axis=1), 0.0, atol=1e-9)
    np.testing.assert_allclose(n.var(axis=1), var / (var + inp.ln_eps), rtol=1e-9)


# ----------------------------------------------------------------------------------------------
# Closed forms
# ----------------------------------------------------------------------------------------------

def test_closed_form_zero_queries_zero_bias():
    # Q = SiLU(0) = 0 and rab = 0  =>  AV = 0  =>  LN(0) = ln_b  =>  Y = (ln_b * U) W2 + b2 + X
    inp = random_case(seed=11, lengths=[6, 10, 3], d=16, H=2, hd=8)
    p = inp.layers[0]
    H, hd = 2, 8
    q0, q1 = 2 * H * hd, 3 * H * hd
    p.W1[:, q0:q1] = 0.0
    p.b1[q0:q1] = 0.0
    inp.pos_table[:] = 0.0
    inp.time_table[:] = 0.0
    y, _, av, _ = _run(inp, return_intermediates=True)
    assert np.all(av == 0.0)
    X = inp.X.astype(np.float64)
    U = _silu(X @ p.W1[:, :H * hd].astype(np.float64) + p.b1[:H * hd])
    expect = (p.ln_b * U) @ p.W2.astype(np.float64) + p.b2 + X
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-12)


def test_closed_form_single_token():
    # n = 1: AV_0 = scale * SiLU(q_0 . k_0 + pos[0] + time[0]) * v_0 for every head
    inp = random_case(seed=12, lengths=[1], d=8, H=2, hd=4, P=5, Tb=3)
    p = inp.layers[0]
    _, uvqk, av, _ = _run(inp, return_intermediates=True)
    z = _silu(inp.X.astype(np.float64) @ p.W1 + p.b1)[0]
    H, hd = 2, 4
    for h in range(H):
        v = z[H * hd + h * hd: H * hd + (h + 1) * hd]
        q = z[2 * H * hd + h * hd: 2 * H * hd + (h + 1) * hd]
        k = z[3 * H * hd + h * hd: 3 * H * hd + (h + 1) * hd]
        s = q @ k + inp.pos_table[h, 0] + inp.time_table[h, 0]
        np.testing.assert_allclose(av[0, h * hd:(h + 1) * hd], inp.scale * s / (1 + math.exp(-s)) * v,
                                   rtol=1e-13)


def test_closed_form_prefix_sum():
    # K = 0 and a constant position bias c_h: AV_i = scale * SiLU(c_h) * sum_{j<=i} v_j
    inp = random_case(seed=13, lengths=[9, 4], d=8, H=2, hd=4, P=6, Tb=4)
    p = inp.layers[0]
    H, hd = 2, 4
    k0 = 3 * H * hd
    p.W1[:, k0:] = 0.0
    p.b1[k0:] = 0.0
    inp.pos_table[:] = np.array([0.3, -1.7], np.float32)[:, None]
    inp.time_table[:] = 0.0
    c = inp.pos_table[:, 0].astype(np.float64)          # the stored (float32) values
    _, uvqk, av, _ = _run(inp, return_intermediates=True)
    V = uvqk[:, H * hd:2 * H * hd]
    for s in range(2):
        a, b = inp.seq_offsets[s], inp.seq_offsets[s + 1]
        csum = np.cumsum(V[a:b], axis=0)
        for h in range(H):
            f = inp.scale * c[h] / (1 + math.exp(-c[h]))
            np.testing.assert_allclose(av[a:b, h * hd:(h + 1) * hd], f * csum[:, h * hd:(h + 1) * hd],
                                       rtol=1e-12, atol=1e-15)


def test_alibi_equals_linear_position_table():
    # ALiBi -m_h (i - j) is the position table pos[h][p] = -m_h p when P exceeds every distance
    inp = random_case(seed=14, lengths=[13, 6], d=16, H=4, hd=4, alibi=True)
    y_alibi = _run(inp)
    P = 16
    inp.pos_table = (-inp.alibi_slopes[:, None].astype(np.float64) * np.arange(P)[None, :])
    inp.alibi_slopes = None
    inp.time_table = None
    y_pos = _run(inp)
    np.testing.assert_allclose(y_alibi, y_pos, rtol=1e-14, atol=1e-14)


def test_alibi_zero_slopes_equals_no_bias():
    inp = random_case(seed=15, lengths=[8, 5], d=8, H=2, hd=4, alibi=True)
    inp.alibi_slopes = np.zeros_like(inp.alibi_slopes)
    y0 = _run(inp)
    inp.alibi_slopes = None
    y1 = _run(inp)
    np.testing.assert_array_equal(y0, y1)


def test_scale_is_linear_in_av():
    inp = random_case(seed=16, lengths=[10, 3], d=8, H=2, hd=4)
    _, _, av1, _ = _run(inp, return_intermediates=True)
    inp.scale = 2.0 * inp.scale
    _, _, av2, _ = _run(inp, return_intermediates=True)
    np.testing.assert_array_equal(av2, 2.0 * av1)           # doubling is exact in binary fp


# ----------------------------------------------------------------------------------------------
# Invariants (bit-exact in the oracle)
# ----------------------------------------------------------------------------------------------

def test_causality():
    inp = random_case(seed=17, lengths=[12, 9], d=8, H=2, hd=4)
    y0 = _run(inp)
    i = 5                                  # local row of sequence 0
    inp.X = inp.X.copy()
    inp.X[i + 1:12] += 3.0                 # future tokens of the same sequence
    inp.timestamps = inp.timestamps.copy()
    inp.timestamps[i + 1:12] += 10**6
    y1 = _run(inp)
    np.testing.assert_array_equal(y0[:i + 1], y1[:i + 1])
    assert np.max(np.abs(y0[i + 1:12] - y1[i + 1:12])) > 1e-3
    np.testing.assert_array_equal(y0[12:], y1[12:])


def test_jagged_independence_and_permutation():
    inp = random_case(seed=18, lengths=[7, 11, 4], d=8, H=2, hd=4)
    y = _run(inp)
    off = inp.seq_offsets
    # replacing another sequence's tokens leaves sequence 1 unchanged
    inp2 = random_case(seed=18, lengths=[7, 11, 4], d=8, H=2, hd=4)
    inp2.X = inp2.X.copy()
    inp2.X[:off[1]] = np.random.default_rng(0).standard_normal((off[1], 8))
    inp2.X[off[2]:] *= -2.0
    y2 = _run(inp2)
    np.testing.assert_array_equal(y[off[1]:off[2]], y2[off[1]:off[2]])
    # permuting the batch permutes the outputs
    perm = [2, 0, 1]
    segs = [slice(off[s], off[s + 1]) for s in range(3)]
    inp3 = random_case(seed=18, lengths=[7, 11, 4], d=8, H=2, hd=4)
    inp3.X = np.concatenate([inp.X[segs[s]] for s in perm])
    inp3.timestamps = np.concatenate([inp.timestamps[segs[s]] for s in perm])
    inp3.lengths = inp.lengths[perm]
    inp3.seq_offsets = np.concatenate([[0], np.cumsum(inp3.lengths)])
    y3 = _run(inp3)
    np.testing.assert_array_equal(y3, np.concatenate([y[segs[s]] for s in perm]))


def test_empty_sequences_and_empty_batch():
    inp = random_case(seed=19, lengths=[0, 5, 0], d=8, H=2, hd=4)
    ref = random_case(seed=19, lengths=[5], d=8, H=2, hd=4)
    ref.X, ref.timestamps = inp.X, inp.timestamps
    np.testing.assert_array_equal(_run(inp), _run(ref))
    inp0 = random_case(seed=19, lengths=[0, 0], d=8, H=2, hd=4)
    assert _run(inp0).shape == (0, 8)


# ----------------------------------------------------------------------------------------------
# The row-sampled evaluation is the full evaluation restricted to some rows
# ----------------------------------------------------------------------------------------------

def test_row_sampling_matches_full_layer():
    inp = random_case(seed=20, lengths=[17, 1, 30], d=16, H=2, hd=8)
    y, _, av, _ = _run(inp, return_intermediates=True)
    rows = [0, 16, 17, 18, 25, 47]
    yr, avr = oracle.layer_rows_inputs(inp, rows)
    np.testing.assert_array_equal(yr, y[rows])
    np.testing.assert_array_equal(avr, av[rows])


# ----------------------------------------------------------------------------------------------
# Token assembly (GenRank action-oriented tokens)
# ----------------------------------------------------------------------------------------------

def test_token_embed_sum_rounded_to_bf16():
    rng = np.random.default_rng(3)
    it = to_bf16_bits(rng.standard_normal((50, 16)).astype(np.float32))
    at = to_bf16_bits(rng.standard_normal((8, 16)).astype(np.float32))
    ii = rng.integers(0, 50, 40)
    ai = rng.integers(0, 8, 40)
    X = oracle.token_embed(ii, ai, widen_bf16(it), widen_bf16(at))
    # the sum of two bf16 values is exact in float32; round that to bf16 bit-wise
    s32 = (widen_bf16(it, np.float32)[ii] + widen_bf16(at, np.float32)[ai]).astype(np.float32)
    np.testing.assert_array_equal(X, widen_bf16(to_bf16_bits(s32)))


def test_workload_recipes_have_the_stated_shapes():
    inp = make_inputs("tiny_fp32")
    assert inp.workload.d_model == 64 and inp.layers[0].W1.shape == (64, 256)
    assert len(inp.lengths) == 4 and inp.lengths.min() >= 8 and inp.lengths.max() <= 64
    assert inp.pos_table.shape == (2, 64) and inp.time_table.shape == (2, 32)
    assert np.all(np.diff(inp.timestamps[:inp.lengths[0]]) >= 0)
