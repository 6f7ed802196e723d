"""M-FALCON candidate scoring on the GPU against the oracle ("Actions Speak Louder than Words" paper
notes, section 3.6): candidates see their user's history (K/V from the history's UVQK, the
encoder-level cache) and themselves, at the position right after the history.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import assert_bf16_close, assert_layer_part_close, dev, host, round_bf16
from workloads import draw_candidates, random_case


@pytest.fixture(scope="module")
def hstu():
    import hstu_sequential_transduction_layer_b200 as m
    return m


def _case(seed, hist, cand, H, hd, bias="rab", spread=500, P=96, Tb=24):
    d = H * hd
    inp = random_case(seed, hist, d, H, hd, P=P, Tb=Tb, dtype="bf16", alibi=(bias == "alibi"))
    if bias in ("pos", "none"):
        inp.time_table = None
    if bias == "none":
        inp.pos_table = None
    c = draw_candidates(inp, cand, spread_s=spread)
    p = inp.layers[0]
    uh = round_bf16(oracle.f1(inp.X, p.W1, p.b1))
    uc = round_bf16(oracle.f1(c.X, p.W1, p.b1))
    return inp, c, uh, uc


def _tables(inp):
    return (dev(inp.pos_table, "f32"), dev(inp.time_table, "f32"), dev(inp.alibi_slopes, "f32"))


def _shape(hstu, inp):
    w = inp.workload
    P = 0 if inp.pos_table is None else inp.pos_table.shape[1]
    Tb = 0 if inp.time_table is None else inp.time_table.shape[1]
    return hstu.make_shape(len(inp.lengths), inp.T, max(1, int(inp.lengths.max())), w.d_model,
                           w.num_heads, w.head_dim, w.head_dim, hstu.HSTU_BF16, P, Tb)


def _gpu_av(hstu, inp, c, uh, uc, rows=None):
    """Candidate AV on the GPU, for all candidates or for the candidate subset `rows` (kept in user
    order, scored against the same history)."""
    w = inp.workload
    if rows is None:
        counts, sel = c.counts, np.arange(len(c.X))
    else:
        sel = np.asarray(rows)
        counts = np.array([np.sum((sel >= c.offsets[b]) & (sel < c.offsets[b + 1]))
                           for b in range(len(c.counts))])
    coff = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    s = _shape(hstu, inp)
    pos, tim, ali = _tables(inp)
    av = torch.full((len(sel), w.num_heads * w.head_dim), float("nan"), dtype=torch.float32,
                    device="cuda")
    ts = dev(inp.timestamps) if inp.time_table is not None else None
    cts = dev(c.timestamps[sel]) if inp.time_table is not None else None
    hstu.hstu_candidate_attention_fwd(s, dev(uh), dev(inp.seq_offsets), ts, dev(uc[sel]),
                                      dev(coff), cts, pos, tim, ali, inp.scale, av,
                                      max_candidates=max(1, int(counts.max())))
    assert hstu.device_status() == hstu.HSTU_OK
    return host(av)


def _oracle_av(inp, c, uh, uc):
    w = inp.workload
    has_t = inp.time_table is not None
    return oracle.candidate_attention(
        inp.seq_offsets, uh, c.offsets, uc, num_heads=w.num_heads, d_qk=w.head_dim,
        d_v=w.head_dim, hist_timestamps=inp.timestamps if has_t else None,
        cand_timestamps=c.timestamps if has_t else None, pos_table=inp.pos_table,
        time_table=inp.time_table, alibi_slopes=inp.alibi_slopes, scale=inp.scale)


@pytest.mark.gpu
@pytest.mark.parametrize("seed,hist,cand,H,hd,bias", [
    (31, [300, 0, 129, 1, 700], [3, 2, 130, 1, 257], 2, 64, "rab"),
    (32, [128, 513], [256, 5], 2, 128, "rab"),
    (33, [200, 64, 0], [7, 300, 4], 2, 64, "alibi"),
    (34, [390, 17], [129, 64], 2, 64, "pos"),
    (35, [255, 256, 257], [1, 2, 3], 2, 64, "none"),
    (36, [1000, 40], [600, 9], 1, 128, "alibi"),
])
def test_candidate_attention_matches_oracle(hstu, seed, hist, cand, H, hd, bias):
    inp, c, uh, uc = _case(seed, hist, cand, H, hd, bias)
    assert_bf16_close(_gpu_av(hstu, inp, c, uh, uc), _oracle_av(inp, c, uh, uc),
                      f"candidate AV ({bias}, hd={hd})")


@pytest.mark.gpu
def test_micro_batches_give_the_same_rows_bit_for_bit(hstu):
    inp, c, uh, uc = _case(37, [520, 300], [300, 140], 2, 64, "rab")
    full = _gpu_av(hstu, inp, c, uh, uc)
    idx = np.arange(len(c.X))
    for part in (idx[0::2], idx[1::2]):
        np.testing.assert_array_equal(_gpu_av(hstu, inp, c, uh, uc, rows=part), full[part])


@pytest.mark.gpu
@pytest.mark.parametrize("bias", ["rab", "alibi"])
def test_candidate_layer_matches_oracle(hstu, bias):
    inp, c, uh, uc = _case(38, [333, 0, 256], [40, 3, 200], 2, 64, bias)
    w, p = inp.workload, inp.layers[0]
    has_t = inp.time_table is not None
    ref = oracle.candidate_layer_fwd(
        inp.seq_offsets, uh, c.offsets, c.X, p.W1, p.b1, p.W2, p.b2, p.ln_w, p.ln_b,
        num_heads=w.num_heads, d_qk=w.head_dim, d_v=w.head_dim,
        hist_timestamps=inp.timestamps if has_t else None,
        cand_timestamps=c.timestamps if has_t else None, pos_table=inp.pos_table,
        time_table=inp.time_table, alibi_slopes=inp.alibi_slopes, scale=inp.scale)
    s = _shape(hstu, inp)
    pos, tim, ali = _tables(inp)
    out = torch.empty((len(c.X), w.d_model), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_candidate_layer_fwd(s, dev(uh), dev(inp.seq_offsets),
                                  dev(inp.timestamps) if has_t else None, dev(c.X),
                                  dev(c.offsets), dev(c.timestamps) if has_t else None,
                                  dev(p.W1), dev(p.b1), dev(p.W2), dev(p.b2), dev(p.ln_w),
                                  dev(p.ln_b), pos, tim, ali, inp.scale, out,
                                  max_candidates=int(c.counts.max()))
    assert hstu.device_status() == hstu.HSTU_OK
    got = host(out)
    assert_bf16_close(got, ref, f"candidate layer ({bias})")
    assert_layer_part_close(got, ref, c.X.astype(np.float64), f"candidate layer ({bias})")


@pytest.mark.gpu
def test_long_history_sampled_rows(hstu):
    """Two users with 4096-token histories and 1024 candidates each; all rows against the oracle."""
    inp, c, uh, uc = _case(39, [4096, 3000], [1024, 777], 2, 64, "rab", spread=3600)
    assert_bf16_close(_gpu_av(hstu, inp, c, uh, uc), _oracle_av(inp, c, uh, uc),
                      "candidate AV, long histories")


def test_candidate_entry_points_validate_on_the_host(hstu):
    import ctypes
    s = hstu.make_shape(2, 100, 64, 128, 2, 64, 64, hstu.HSTU_BF16, 16, 8)
    fake = ctypes.c_void_p(1 << 20)
    lib = hstu.library()
    # more candidates per user than the schedule can number
    rc = lib.hstu_candidate_attention_fwd(ctypes.byref(s), fake, fake, fake, 10, 1 << 30, fake,
                                          fake, fake, fake, fake, None, ctypes.c_float(1.0), fake,
                                          fake, 1 << 30, None)
    assert rc == hstu.HSTU_ERR_UNSUPPORTED
    # a time table without candidate timestamps
    rc = lib.hstu_candidate_attention_fwd(ctypes.byref(s), fake, fake, fake, 10, 10, fake, fake,
                                          None, fake, fake, None, ctypes.c_float(1.0), fake, fake,
                                          1 << 30, None)
    assert rc == hstu.HSTU_ERR_INVALID_ARG
    # fp32 is not implemented on this path
    s32 = hstu.make_shape(2, 100, 64, 128, 2, 64, 64, hstu.HSTU_F32, 16, 8)
    rc = lib.hstu_candidate_attention_fwd(ctypes.byref(s32), fake, fake, fake, 10, 10, fake, fake,
                                          fake, fake, fake, None, ctypes.c_float(1.0), fake, fake,
                                          1 << 30, None)
    assert rc == hstu.HSTU_ERR_UNSUPPORTED
    # no candidates: nothing to do
    rc = lib.hstu_candidate_attention_fwd(ctypes.byref(s), fake, fake, fake, 0, 0, None, fake,
                                          None, None, None, None, ctypes.c_float(1.0), None, None,
                                          0, None)
    assert rc == hstu.HSTU_OK
