"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle, on the same seeded inputs.

Small cases run the whole oracle and compare every element; they span several 128-row tiles with
ragged tails, empty and single-token sequences, every bias variant and both head sizes.  The
full-size workloads run the GPU exactly as bench.py does (hstu_layer_fwd on the whole batch) and
compare sampled rows that the oracle evaluates one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import (assert_bf16_close, assert_f32_close, assert_layer_part_close, dev,
                            host, round_bf16)
from workloads import WORKLOADS, make_inputs, random_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hstu():
    import hstu_sequential_transduction_layer_b200 as m
    return m


def _bias_variant(inp, which):
    if which == "pos":
        inp.time_table = None
    elif which == "time":
        inp.pos_table = None
    elif which == "none":
        inp.pos_table = inp.time_table = None
    return inp


def _gpu_layer(hstu, inp, layer=0, X=None, dtype="bf16"):
    w, p = inp.workload, inp.layers[layer]
    Xd = dev(inp.X if X is None else X, dtype)
    out = hstu.hstu_layer_fwd(
        Xd, dev(inp.seq_offsets), dev(inp.timestamps), dev(p.W1, dtype), dev(p.b1, dtype),
        dev(p.W2, dtype), dev(p.b2, dtype), dev(p.ln_w, dtype), dev(p.ln_b, dtype),
        dev(inp.pos_table, "f32"), dev(inp.time_table, "f32"), dev(inp.alibi_slopes, "f32"),
        inp.scale, num_heads=w.num_heads, max_seq_len=max(1, int(inp.lengths.max(initial=1))),
        ln_eps=inp.ln_eps)
    assert hstu.device_status() == hstu.HSTU_OK
    return host(out)


# ------------------------------------------------------------------------------------------------
# Each kernel on its own
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("T,d,hd", [(1, 64, 64), (300, 128, 64), (129, 256, 128), (517, 512, 64)])
def test_f1_kernel(hstu, T, d, hd):
    rng = np.random.default_rng(T + d)
    H = d // hd
    X = round_bf16(rng.standard_normal((T, d)))
    W1 = round_bf16(rng.uniform(-1, 1, (d, 4 * d)) * np.sqrt(6 / (5 * d)))
    b1 = round_bf16(rng.normal(0, 0.1, 4 * d))
    ref = oracle.f1(X, W1, b1)
    s = hstu.make_shape(1, T, T, d, H, hd, hd, hstu.HSTU_BF16)
    out = torch.empty((T, 4 * d), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_f1_fwd(s, dev(X), dev(W1), dev(b1), out)
    assert_bf16_close(host(out), ref, "f1")


# (the residual joins the accumulator on the tensor core when K = wv is at most 512 and at least
# the tile width; (77, 256, 128) and (260, 256, 1024) take the epilogue's residual loads instead)
@pytest.mark.parametrize("T,d,wv", [(1, 64, 64), (300, 128, 128), (200, 192, 256), (129, 512, 512),
                                    (77, 256, 128), (260, 256, 1024)])
def test_f2_kernel(hstu, T, d, wv):
    rng = np.random.default_rng(T + wv)
    G = round_bf16(rng.standard_normal((T, wv)))
    W2 = round_bf16(rng.uniform(-1, 1, (wv, d)) * np.sqrt(3 / wv))
    b2 = round_bf16(rng.normal(0, 0.1, d))
    X = round_bf16(rng.standard_normal((T, d)))
    ref = oracle.f2(G, W2, b2, X)
    hd = 64 if wv % 128 else 128
    s = hstu.make_shape(1, T, T, d, wv // hd, hd, hd, hstu.HSTU_BF16)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_f2_fwd(s, dev(G), dev(W2), dev(b2), dev(X), out)
    assert_bf16_close(host(out), ref, "f2")
    assert_bf16_close(host(out) - X, ref - X, "f2 without residual")


def _attention_inputs(seed, lengths, d, hd, P=64, Tb=16, alibi=False):
    inp = random_case(seed, lengths, d, d // hd, hd, P=P, Tb=Tb, dtype="bf16", alibi=alibi)
    p = inp.layers[0]
    uvqk = round_bf16(oracle.f1(inp.X, p.W1, p.b1))   # bf16 storage of Eq. 1's output
    return inp, uvqk


ATTN_CASES = [
    dict(seed=31, lengths=[1, 127, 128, 129, 300, 0, 2], d=128, hd=64, which="rab"),
    dict(seed=32, lengths=[513, 5, 256], d=256, hd=128, which="rab"),
    dict(seed=33, lengths=[200, 64], d=128, hd=64, which="pos", P=40),
    dict(seed=34, lengths=[200, 64], d=128, hd=64, which="time", Tb=5),
    dict(seed=35, lengths=[190, 1, 70], d=256, hd=128, which="none"),
    dict(seed=36, lengths=[333, 129], d=256, hd=64, which="alibi"),
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: f"seed{c['seed']}-{c['which']}")
def test_attention_kernel(hstu, case):
    c = dict(case)
    which = c.pop("which")
    inp, uvqk = _attention_inputs(c.pop("seed"), c.pop("lengths"), c.pop("d"), c["hd"],
                                  P=c.get("P", 64), Tb=c.get("Tb", 16), alibi=(which == "alibi"))
    _bias_variant(inp, which)
    hd = c["hd"]
    H = inp.workload.num_heads
    ref = oracle.attention(inp.seq_offsets, uvqk, num_heads=H, d_qk=hd, d_v=hd,
                           timestamps=inp.timestamps, pos_table=inp.pos_table,
                           time_table=inp.time_table, alibi_slopes=inp.alibi_slopes,
                           scale=inp.scale)
    T = inp.T
    s = hstu.make_shape(len(inp.lengths), T, int(inp.lengths.max()), inp.workload.d_model, H, hd,
                        hd, hstu.HSTU_BF16,
                        0 if inp.pos_table is None else inp.pos_table.shape[1],
                        0 if inp.time_table is None else inp.time_table.shape[1])
    av = torch.empty((T, H * hd), dtype=torch.float32, device="cuda")   # fp32 AV (LayerNorm input)
    hstu.hstu_attention_fwd(s, dev(uvqk), dev(inp.seq_offsets), dev(inp.timestamps),
                            dev(inp.pos_table, "f32"), dev(inp.time_table, "f32"),
                            dev(inp.alibi_slopes, "f32"), inp.scale, av)
    assert hstu.device_status() == hstu.HSTU_OK
    assert_bf16_close(host(av), ref, "attention")


# The kernel stages the halved position table in shared memory for distances below 7168 at head
# dim 128 (8192 at 64); tiles reaching farther take the exact path, which reads the table from
# global memory and clamps at P-1.  Sequences long enough to reach both, every row compared.
FAR_CASES = [
    dict(seed=37, lengths=[7500, 8300], d=128, hd=128, P=8192, Tb=128),
    dict(seed=38, lengths=[8500, 300], d=64, hd=64, P=16384, Tb=128),
    dict(seed=39, lengths=[7400], d=128, hd=128, P=2048, Tb=128),
]


@pytest.mark.parametrize("case", FAR_CASES, ids=lambda c: f"seed{c['seed']}-hd{c['hd']}-P{c['P']}")
def test_attention_far_distances(hstu, case):
    hd, d = case["hd"], case["d"]
    inp, uvqk = _attention_inputs(case["seed"], case["lengths"], d, hd, P=case["P"], Tb=case["Tb"])
    inp.scale = 1.0 / 8192
    H = inp.workload.num_heads
    ref = oracle.attention(inp.seq_offsets, uvqk, num_heads=H, d_qk=hd, d_v=hd,
                           timestamps=inp.timestamps, pos_table=inp.pos_table,
                           time_table=inp.time_table, scale=inp.scale)
    T = inp.T
    s = hstu.make_shape(len(inp.lengths), T, int(inp.lengths.max()), d, H, hd, hd, hstu.HSTU_BF16,
                        inp.pos_table.shape[1], inp.time_table.shape[1])
    av = torch.empty((T, H * hd), dtype=torch.float32, device="cuda")
    hstu.hstu_attention_fwd(s, dev(uvqk), dev(inp.seq_offsets), dev(inp.timestamps),
                            dev(inp.pos_table, "f32"), dev(inp.time_table, "f32"), None,
                            inp.scale, av)
    assert hstu.device_status() == hstu.HSTU_OK
    got = host(av)
    assert_bf16_close(got, ref, "attention, far distances")
    # the rows whose keys reach past the staged distances, on their own
    far = 7168 if hd == 128 else 8192
    for b, n in enumerate(inp.lengths):
        if n > far:
            a = int(inp.seq_offsets[b])
            assert_bf16_close(got[a + far - 128:a + n], ref[a + far - 128:a + n],
                              f"attention, rows reaching past {far} in sequence {b}")


@pytest.mark.parametrize("T,wv", [(1, 256), (300, 512), (77, 1024), (40, 4096), (90, 192)])
def test_ln_gate_kernel(hstu, T, wv):
    rng = np.random.default_rng(T + wv)
    hd = 64
    H = wv // hd
    n1 = 4 * wv
    av = (rng.standard_normal((T, wv)) * 1e-3 + 2e-4).astype(np.float32).astype(np.float64)
    uvqk = round_bf16(rng.standard_normal((T, n1)))
    ln_w = round_bf16(rng.uniform(0.5, 1.5, wv))
    ln_b = round_bf16(rng.normal(0, 0.5, wv))
    ref = oracle.ln_gate(av, uvqk, ln_w, ln_b, num_heads=H, d_qk=hd, d_v=hd)
    s = hstu.make_shape(1, T, T, wv, H, hd, hd, hstu.HSTU_BF16)
    g = torch.empty((T, wv), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_ln_gate_fwd(s, dev(av, "f32"), dev(uvqk), dev(ln_w), dev(ln_b), g)
    assert_bf16_close(host(g), ref, "ln_gate")


@pytest.mark.parametrize("T,d", [(1, 128), (300, 128), (129, 256), (1000, 256), (517, 512),
                                 (4097, 512)])
def test_ln_f2_fused_kernel(hstu, T, d):
    # LayerNorm(AV) * U, then f2 and the residual, in one kernel: against the oracle's two steps
    rng = np.random.default_rng(T + 7 * d)
    hd = 64
    H = d // hd
    n1 = 4 * d
    av = (rng.standard_normal((T, d)) * 1e-3 + 2e-4).astype(np.float32).astype(np.float64)
    uvqk = round_bf16(rng.standard_normal((T, n1)))
    ln_w = round_bf16(rng.uniform(0.5, 1.5, d))
    ln_b = round_bf16(rng.normal(0, 0.5, d))
    W2 = round_bf16(rng.uniform(-1, 1, (d, d)) * np.sqrt(3 / d))
    b2 = round_bf16(rng.normal(0, 0.1, d))
    X = round_bf16(rng.standard_normal((T, d)))
    g = oracle.ln_gate(av, uvqk, ln_w, ln_b, num_heads=H, d_qk=hd, d_v=hd)
    ref = oracle.f2(round_bf16(g), W2, b2, X)   # G is stored as bf16 in both GPU paths
    s = hstu.make_shape(1, T, T, d, H, hd, hd, hstu.HSTU_BF16)
    out = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_ln_f2_fwd(s, dev(av, "f32"), dev(uvqk), dev(ln_w), dev(ln_b), dev(W2), dev(b2),
                        dev(X), out)
    assert hstu.device_status() == hstu.HSTU_OK
    got = host(out)
    assert_bf16_close(got, ref, "ln_f2")
    assert_layer_part_close(got, ref, X, "ln_f2 without residual")
    # and the two-step path on the same inputs
    g_d = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_ln_gate_fwd(s, dev(av, "f32"), dev(uvqk), dev(ln_w), dev(ln_b), g_d)
    two = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_f2_fwd(s, g_d, dev(W2), dev(b2), dev(X), two)
    assert_layer_part_close(got, host(two), X, "ln_f2 vs the two steps")


def test_token_embed_bit_exact(hstu):
    rng = np.random.default_rng(5)
    itab = rng.standard_normal((1000, 1024)).astype(np.float32)
    atab = rng.standard_normal((8, 1024)).astype(np.float32)
    ii = rng.integers(0, 1000, 777)
    ai = rng.integers(0, 8, 777)
    ref = oracle.token_embed(ii, ai, round_bf16(itab), round_bf16(atab))
    X = hstu.hstu_token_embed_fwd(dev(ii), dev(ai), dev(itab), dev(atab))
    assert hstu.device_status() == hstu.HSTU_OK
    np.testing.assert_array_equal(host(X), ref)


# ------------------------------------------------------------------------------------------------
# The whole layer
# ------------------------------------------------------------------------------------------------

def test_layer_tiny_fp32(hstu):
    inp = make_inputs("tiny_fp32")
    ref = oracle.layer_fwd_inputs(inp)
    got = _gpu_layer(hstu, inp, dtype="f32")
    assert_f32_close(got, ref, "tiny_fp32")
    assert_f32_close(got - inp.X, ref - inp.X, "tiny_fp32 without residual")


@pytest.mark.parametrize("seed,lengths,d,H,hd", [(41, [5, 64, 1, 30], 64, 2, 32),
                                                  (42, [3, 17, 0], 48, 3, 16),
                                                  (43, [100], 128, 1, 128)])
def test_layer_fp32_random(hstu, seed, lengths, d, H, hd):
    inp = random_case(seed, lengths, d, H, hd, P=32, Tb=12, dtype="f32")
    ref = oracle.layer_fwd_inputs(inp)
    assert_f32_close(_gpu_layer(hstu, inp, dtype="f32"), ref, "fp32 layer")


LAYER_CASES = [
    dict(seed=51, lengths=[1, 127, 128, 129, 257, 0], d=128, hd=64, which="rab"),
    dict(seed=52, lengths=[300, 45], d=256, hd=128, which="rab"),
    dict(seed=53, lengths=[220, 2], d=128, hd=64, which="alibi"),
    dict(seed=54, lengths=[150], d=192, hd=64, which="none"),
]


@pytest.mark.parametrize("case", LAYER_CASES, ids=lambda c: f"seed{c['seed']}-{c['which']}")
def test_layer_bf16_small(hstu, case):
    which = case["which"]
    inp = random_case(case["seed"], case["lengths"], case["d"], case["d"] // case["hd"], case["hd"],
                      P=96, Tb=24, dtype="bf16", alibi=(which == "alibi"))
    _bias_variant(inp, which)
    ref = oracle.layer_fwd_inputs(inp)
    got = _gpu_layer(hstu, inp)
    assert_bf16_close(got, ref, "layer")
    assert_layer_part_close(got, ref, inp.X, "layer without residual")


def test_layer_retrieval_two_layers(hstu):
    inp = make_inputs("retrieval")
    y1 = oracle.layer_fwd_inputs(inp, layer=0)
    x2 = round_bf16(y1)                      # the layer's output is stored as bf16
    y2 = oracle.layer_fwd_inputs(inp, layer=1, X=x2)
    g1 = _gpu_layer(hstu, inp, layer=0)
    assert_bf16_close(g1, y1, "retrieval layer 1")
    g2 = _gpu_layer(hstu, inp, layer=1, X=g1)
    assert_bf16_close(g2, y2, "retrieval layer 2")
    assert_layer_part_close(g1, y1, inp.X, "retrieval layer 1 without residual")


def test_layer_empty_and_degenerate(hstu):
    # all sequences empty but one single token; and a batch of zero tokens
    inp = random_case(61, [0, 1, 0], 128, 2, 64, dtype="bf16")
    assert_bf16_close(_gpu_layer(hstu, inp), oracle.layer_fwd_inputs(inp), "single token")
    inp0 = random_case(62, [0, 0], 128, 2, 64, dtype="bf16")
    assert _gpu_layer(hstu, inp0).shape == (0, 128)


def test_jagged_independence_on_gpu(hstu):
    # a sequence's output does not depend on the other sequences of the batch (bit-exact)
    inp = random_case(71, [200, 333, 17], 128, 2, 64, dtype="bf16")
    full = _gpu_layer(hstu, inp)
    sub = random_case(71, [333], 128, 2, 64, dtype="bf16")
    a, b = inp.seq_offsets[1], inp.seq_offsets[2]
    sub.X, sub.timestamps = inp.X[a:b], inp.timestamps[a:b]
    np.testing.assert_array_equal(_gpu_layer(hstu, sub), full[a:b])


def test_bad_offsets_are_reported_not_faulting(hstu):
    inp = random_case(72, [40, 60], 128, 2, 64, dtype="bf16")
    inp.seq_offsets = np.array([0, 70, 50], np.int64)     # not monotone, wrong end
    w, p = inp.workload, inp.layers[0]
    out = hstu.hstu_layer_fwd(dev(inp.X), dev(inp.seq_offsets), dev(inp.timestamps), dev(p.W1),
                              dev(p.b1), dev(p.W2), dev(p.b2), dev(p.ln_w), dev(p.ln_b),
                              dev(inp.pos_table, "f32"), dev(inp.time_table, "f32"), None,
                              inp.scale, num_heads=2, max_seq_len=64)
    assert hstu.device_status() == hstu.HSTU_ERR_DEVICE_BAD_OFFSETS
    assert out.shape == (100, 128)
    assert hstu.device_status() == hstu.HSTU_OK            # reading clears it


# ------------------------------------------------------------------------------------------------
# Full-size workloads, sampled rows
# ------------------------------------------------------------------------------------------------

def _sample_rows(inp, seqs, local):
    rows = []
    for s in seqs:
        a, n = int(inp.seq_offsets[s]), int(inp.lengths[s])
        rows += sorted({a + min(max(i if i >= 0 else n + i, 0), n - 1) for i in local})
    return rows


@pytest.mark.parametrize("name", ["long_seq", "alibi_rank", "large"])
def test_layer_full_size_sampled(hstu, name):
    inp = make_inputs(name)
    w = inp.workload
    if w.token_embed:
        # GenRank token assembly on the GPU, checked bit-exact against the oracle's, then the layer
        ids = np.unique(inp.item_ids)
        X_ref = oracle.token_embed(np.searchsorted(ids, inp.item_ids), inp.action_ids,
                                   round_bf16_bits(inp.item_table_bits[ids]),
                                   round_bf16_bits(inp.action_table_bits))
        Xd = hstu.hstu_token_embed_fwd(dev(inp.item_ids), dev(inp.action_ids),
                                       bits_dev(inp.item_table_bits), bits_dev(inp.action_table_bits))
        np.testing.assert_array_equal(host(Xd), X_ref)
        inp.X = X_ref
    order = np.argsort(inp.lengths)
    if name == "long_seq":
        seqs, local = [0, 5], [0, 1, 127, 128, 129, 1000, 4095, 4096, -2, -1]
    elif name == "alibi_rank":
        seqs, local = [int(order[0]), int(order[-1]), 7], [0, 127, 128, 1500, -129, -1]
    else:  # large: the shortest sequences whole-tail and early rows of the longest (oracle cost)
        seqs, local = [int(order[0]), int(order[1])], [0, 127, 128, 255, -1]
    rows = _sample_rows(inp, seqs, local)
    if name == "large":
        # early rows of the longest sequence, and the rows whose keys reach past the 7168 position
        # buckets the hd=128 kernel stages in shared memory (exact path, table read from global)
        a, n = int(inp.seq_offsets[order[-1]]), int(inp.lengths[order[-1]])
        assert n > 7169
        rows += [a, a + 129, a + 700, a + 7167, a + 7168, a + 7169, a + n - 1]
    ref, av_ref = oracle.layer_rows_inputs(inp, rows)
    got = _gpu_layer(hstu, inp)[rows]
    assert_bf16_close(got, ref, name)
    assert_layer_part_close(got, ref, inp.X[rows].astype(np.float64), f"{name} without residual")
    # the attention output itself, through the step entry points (same kernels)
    av = _gpu_av(hstu, inp)[rows]
    assert_bf16_close(av, av_ref, f"{name} AV")


def _gpu_av(hstu, inp):
    w, p = inp.workload, inp.layers[0]
    H, hd, T = w.num_heads, w.head_dim, inp.T
    s = hstu.make_shape(len(inp.lengths), T, int(inp.lengths.max()), w.d_model, H, hd, hd,
                        hstu.HSTU_BF16,
                        0 if inp.pos_table is None else inp.pos_table.shape[1],
                        0 if inp.time_table is None else inp.time_table.shape[1])
    uvqk = torch.empty((T, 4 * H * hd), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_f1_fwd(s, dev(inp.X), dev(p.W1), dev(p.b1), uvqk)
    av = torch.empty((T, H * hd), dtype=torch.float32, device="cuda")
    hstu.hstu_attention_fwd(s, uvqk, dev(inp.seq_offsets), dev(inp.timestamps),
                            dev(inp.pos_table, "f32"), dev(inp.time_table, "f32"),
                            dev(inp.alibi_slopes, "f32"), inp.scale, av)
    assert hstu.device_status() == hstu.HSTU_OK
    return host(av)


def round_bf16_bits(bits):
    from workloads import widen_bf16
    return widen_bf16(bits, np.float64)


def bits_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)
