"""hstu_attention_fwd_noalloc: the attention step for callers that cannot allocate device memory
around the call.  It must give the results of hstu_attention_fwd bit for bit, call after call,
while keeping its tile schedule in the library's fixed device scratch array instead of a caller
workspace, and those results must match the oracle.

Two scheduling regimes are covered: the static one (each CTA takes a fixed stride of the item
list) and the dynamically claimed one, used when the batch's K/V exceed 256 MB, where the CTAs
claim items from a counter that lives in the shared scratch array and so carries over from the
previous call unless the call resets it.

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import assert_bf16_close, dev, host, round_bf16
from workloads import random_case


@pytest.fixture(scope="module")
def hstu():
    import hstu_sequential_transduction_layer_b200 as m
    return m


def _shape(hstu, inp, d, hd):
    return hstu.make_shape(len(inp.lengths), inp.T, int(inp.lengths.max()), d, d // hd, hd, hd,
                           hstu.HSTU_BF16, inp.pos_table.shape[1], inp.time_table.shape[1])


def _case(hstu, seed, lengths, d, hd):
    inp = random_case(seed, lengths, d, d // hd, hd, P=96, Tb=24, dtype="bf16")
    p = inp.layers[0]
    uvqk = round_bf16(oracle.f1(inp.X, p.W1, p.b1))
    H = d // hd
    ref = oracle.attention(inp.seq_offsets, uvqk, num_heads=H, d_qk=hd, d_v=hd,
                           timestamps=inp.timestamps, pos_table=inp.pos_table,
                           time_table=inp.time_table, scale=inp.scale)
    args = (dev(uvqk), dev(inp.seq_offsets), dev(inp.timestamps), dev(inp.pos_table, "f32"),
            dev(inp.time_table, "f32"), None, inp.scale)
    return _shape(hstu, inp, d, hd), args, (inp.T, H * hd), ref


def _both(hstu, s, args, out_shape):
    ref = torch.empty(out_shape, dtype=torch.float32, device="cuda")
    hstu.hstu_attention_fwd(s, *args, ref)
    got = torch.full(out_shape, float("nan"), dtype=torch.float32, device="cuda")
    hstu.hstu_attention_fwd_noalloc(s, *args, got)
    assert hstu.device_status() == hstu.HSTU_OK
    return got, ref


def test_scratch_address_cache_follows_the_context(hstu):
    # host-only: the scratch array's device address is reused only in the context it was looked
    # up in (a device reset replaces the context and may move the array)
    assert hstu.library().hstu_selftest_scratch_cache() == 0


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(hstu):
    # two different problems back to back: the second call must not see the first one's schedule;
    # both entry points run the same kernels on the same schedule, so they agree bit for bit
    cases = [(81, [300, 1, 129, 513], 128, 64), (82, [700, 40], 256, 128)]
    for seed, lengths, d, hd in cases:
        s, args, out_shape, oracle_av = _case(hstu, seed, lengths, d, hd)
        got, ref = _both(hstu, s, args, out_shape)
        assert torch.equal(got, ref), f"noalloc differs from the workspace entry point, case {seed}"
        assert_bf16_close(host(got), oracle_av, f"noalloc vs oracle, case {seed}")


def _dynamic_case(seed, n_seqs, n, d, hd):
    # K/V of 4*hd*T*H bytes above 256 MB: the attention kernel claims items dynamically.  U|V|Q|K
    # is drawn directly (values of the size f1's SiLU outputs take) instead of running f1 on the
    # CPU for 140k rows.
    inp = random_case(seed, [n] * n_seqs, d, d // hd, hd, P=1024, Tb=64, dtype="bf16",
                      scale=1.0 / n)
    rng = np.random.default_rng(np.random.SeedSequence([seed, 99]))
    uvqk = round_bf16(rng.standard_normal((inp.T, 4 * d), dtype=np.float32) * 0.5)
    return inp, uvqk


@pytest.mark.gpu
def test_noalloc_dynamic_regime_after_a_static_call(hstu):
    d, hd = 512, 64
    H = d // hd
    inp, uvqk = _dynamic_case(83, 70, 2000, d, hd)
    assert 4 * hd * inp.T * H > 256 << 20          # the dynamically claimed regime
    s = _shape(hstu, inp, d, hd)
    assert hstu.attention_workspace_size(s) <= 8 << 20
    args = (dev(uvqk), dev(inp.seq_offsets), dev(inp.timestamps), dev(inp.pos_table, "f32"),
            dev(inp.time_table, "f32"), None, inp.scale)
    # a static-regime call first leaves its own schedule and counter in the scratch array
    s0, args0, shape0, _ = _case(hstu, 84, [257, 33], 128, 64)
    got0, ref0 = _both(hstu, s0, args0, shape0)
    assert torch.equal(got0, ref0)
    # then two dynamic-regime calls in a row; item order may differ between runs, but every item
    # writes its own rows with a fixed order of operations, so results are bit-identical
    ref = torch.empty((inp.T, H * hd), dtype=torch.float32, device="cuda")
    hstu.hstu_attention_fwd(s, *args, ref)
    for call in range(2):
        got = torch.full((inp.T, H * hd), float("nan"), dtype=torch.float32, device="cuda")
        hstu.hstu_attention_fwd_noalloc(s, *args, got)
        assert hstu.device_status() == hstu.HSTU_OK
        assert torch.equal(got, ref), f"dynamic regime, call {call}"
    # the oracle on the first and the last sequence (sequences are independent)
    got = host(got)
    for b in (0, len(inp.lengths) - 1):
        a, e = int(inp.seq_offsets[b]), int(inp.seq_offsets[b + 1])
        av = oracle.attention(np.array([0, e - a], np.int64), uvqk[a:e], num_heads=H, d_qk=hd,
                              d_v=hd, timestamps=inp.timestamps[a:e], pos_table=inp.pos_table,
                              time_table=inp.time_table, scale=inp.scale)
        assert_bf16_close(got[a:e], av, f"dynamic regime vs oracle, sequence {b}")


def test_noalloc_rejects_a_schedule_larger_than_its_scratch(hstu):
    # validation happens on the host before anything touches a GPU
    big = hstu.make_shape(10_000_000, 1 << 30, 4096, 512, 8, 64, 64, hstu.HSTU_BF16, 16, 8)
    fake = ctypes.c_void_p(1 << 20)
    rc = hstu.library().hstu_attention_fwd_noalloc(ctypes.byref(big), fake, fake, fake, fake, fake,
                                                   None, ctypes.c_float(1.0), fake, None)
    assert rc == hstu.HSTU_ERR_UNSUPPORTED
