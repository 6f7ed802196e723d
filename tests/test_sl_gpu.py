"""Stochastic Length on the GPU against the oracle, bit for bit ("Actions Speak Louder than Words"
paper notes, section 3.3): integer work, and the one floating-point decision (the cut) taken in
fp64 on both sides from the same inputs.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads import draw_stochastic_length_randoms


@pytest.fixture(scope="module")
def hstu():
    import hstu_sequential_transduction_layer_b200 as m
    return m


def _run(hstu, off, max_len, alpha, u, keys):
    d = "cuda"
    B, T = len(off) - 1, int(off[-1])
    new_off = torch.full((B + 1,), -1, dtype=torch.int64, device=d)
    index = torch.full((max(T, 1),), -1, dtype=torch.int64, device=d)
    hstu.hstu_stochastic_length(torch.from_numpy(off).to(d), max_len, alpha,
                                torch.from_numpy(np.asarray(u, np.float64)).to(d),
                                torch.from_numpy(keys.view(np.int32)).to(d), new_off, index)
    assert hstu.device_status() == hstu.HSTU_OK
    no = new_off.cpu().numpy()
    return no, index.cpu().numpy()[:no[-1]]


CASES = [
    ("mixed", [0, 1, 776, 777, 900, 4096, 3000, 5, 1351, 1352, 8192], 4096, 1.6),
    ("alpha_1.3", [2000, 17, 4096, 600, 1024], 4096, 1.3),
    ("alpha_2_keeps_all", [100, 4096, 7], 4096, 2.0),
    ("many_short", list(np.random.default_rng(3).integers(0, 300, 500)), 1024, 1.5),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,lengths,max_len,alpha", CASES)
def test_plan_and_selection_match_oracle_bit_for_bit(hstu, name, lengths, max_len, alpha):
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    u, keys = draw_stochastic_length_randoms(off, seed=len(lengths))
    # half of the long sequences are forced to the cut side, half to the whole side
    u = u.copy()
    u[::2] = np.maximum(u[::2], 0.999)
    ro, ri = oracle.stochastic_length(off, max_len, alpha, u, keys)
    go, gi = _run(hstu, off, max_len, alpha, u, keys)
    np.testing.assert_array_equal(go, ro)
    np.testing.assert_array_equal(gi, ri)


@pytest.mark.gpu
def test_ties_are_broken_by_position(hstu):
    lengths = [5000, 3333, 4096]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    keys = np.random.default_rng(9).integers(0, 4, int(off[-1])).astype(np.uint32)   # heavy ties
    u = np.full(len(lengths), 0.9999)
    ro, ri = oracle.stochastic_length(off, 4096, 1.6, u, keys)
    go, gi = _run(hstu, off, 4096, 1.6, u, keys)
    np.testing.assert_array_equal(go, ro)
    np.testing.assert_array_equal(gi, ri)


@pytest.mark.gpu
@pytest.mark.parametrize("workload,alpha", [("long_seq", 1.6), ("large", 1.7)])
def test_full_size_batches_and_gather(hstu, workload, alpha):
    inp = workloads.make_inputs(workload)
    off = inp.seq_offsets
    max_len = int(inp.lengths.max())
    u, keys = draw_stochastic_length_randoms(off, seed=11)
    ro, ri = oracle.stochastic_length(off, max_len, alpha, u, keys)
    d = "cuda"
    B, T = len(off) - 1, int(off[-1])
    new_off = torch.empty(B + 1, dtype=torch.int64, device=d)
    index = torch.empty(T, dtype=torch.int64, device=d)
    hstu.hstu_stochastic_length(torch.from_numpy(off).to(d), max_len, alpha,
                                torch.from_numpy(u).to(d),
                                torch.from_numpy(keys.view(np.int32)).to(d), new_off, index)
    np.testing.assert_array_equal(new_off.cpu().numpy(), ro)
    np.testing.assert_array_equal(index.cpu().numpy()[:ro[-1]], ri)
    # the shortened batch: X rows and timestamps gathered with the count read on the device
    Xbits = workloads.to_bf16_bits(inp.X)
    X = torch.from_numpy(Xbits.view(np.int16)).to(d)
    ts = torch.from_numpy(inp.timestamps).to(d)
    Xn = torch.full((T, X.shape[1]), -1, dtype=torch.int16, device=d)
    tsn = torch.full((T,), -1, dtype=torch.int64, device=d)
    hstu.hstu_gather_rows(index, X, Xn, row_count=new_off[B:])
    hstu.hstu_gather_rows(index, ts, tsn, row_count=new_off[B:])
    assert hstu.device_status() == hstu.HSTU_OK
    n_new = int(ro[-1])
    np.testing.assert_array_equal(Xn.cpu().numpy()[:n_new], Xbits.view(np.int16)[ri])
    np.testing.assert_array_equal(tsn.cpu().numpy()[:n_new], inp.timestamps[ri])
    assert np.all(Xn.cpu().numpy()[n_new:] == -1)           # rows past the count untouched


def test_host_validation(hstu):
    lib = hstu.library()
    fake = ctypes.c_void_p(1 << 20)
    for alpha in (0.0, 2.5, float("nan")):
        rc = lib.hstu_stochastic_length(2, 10, fake, 10, ctypes.c_double(alpha), fake, fake, fake,
                                        fake, fake, 1 << 20, None)
        assert rc == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_gather_rows(10, None, 12, fake, fake, 10, fake, None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_gather_rows(0, None, 16, None, None, 0, None, None) == hstu.HSTU_OK
