"""hstu_attention_fwd_noalloc: the attention step for callers that cannot allocate device memory
around the call.  It must give the results of hstu_attention_fwd, call after call, while keeping
its tile schedule in the library's fixed device scratch array instead of a caller workspace.

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


def _case(hstu, seed, lengths, d, hd):
    inp = random_case(seed, lengths, d, d // hd, hd, P=96, Tb=24, dtype="bf16")
    p = inp.layers[0]
    uvqk = round_bf16(oracle.f1(inp.X, p.W1, p.b1))
    H = d // hd
    s = hstu.make_shape(len(inp.lengths), inp.T, int(inp.lengths.max()), d, H, hd, hd,
                        hstu.HSTU_BF16, inp.pos_table.shape[1], inp.time_table.shape[1])
    args = (dev(uvqk), dev(inp.seq_offsets), dev(inp.timestamps), dev(inp.pos_table, "f32"),
            dev(inp.time_table, "f32"), None, inp.scale)
    return s, args, (inp.T, H * hd)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(hstu):
    # two different problems back to back: the second call must not see the first one's schedule
    cases = [(81, [300, 1, 129, 513], 128, 64), (82, [700, 40], 256, 128)]
    for seed, lengths, d, hd in cases:
        s, args, out_shape = _case(hstu, seed, lengths, d, hd)
        ref = torch.empty(out_shape, dtype=torch.float32, device="cuda")
        hstu.hstu_attention_fwd(s, *args, ref)
        got = torch.full(out_shape, float("nan"), dtype=torch.float32, device="cuda")
        hstu.hstu_attention_fwd_noalloc(s, *args, got)
        assert hstu.device_status() == hstu.HSTU_OK
        assert_bf16_close(host(got), host(ref), f"noalloc vs workspace, case {seed}")


def test_noalloc_rejects_a_schedule_larger_than_its_scratch(hstu):
    # validation happens on the host before anything touches a GPU
    big = hstu.make_shape(10_000_000, 1 << 30, 4096, 512, 8, 64, 64, hstu.HSTU_BF16, 16, 8)
    fake = ctypes.c_void_p(1 << 20)
    rc = hstu.library().hstu_attention_fwd_noalloc(ctypes.byref(big), fake, fake, fake, fake, fake,
                                                   None, ctypes.c_float(1.0), fake, None)
    assert rc == hstu.HSTU_ERR_UNSUPPORTED
