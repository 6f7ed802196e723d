"""Backward of Eq. 2 on the GPU (tcgen05, head dims 64 and 128) against the fp64 oracle ("Actions Speak
Louder than Words" paper notes, section 3.1; training).  P and dS enter the tensor-core products in
bf16, so dq, dk, dv are held to the bf16 criteria; the table gradients sum fp32 scores."""
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


def _run(hstu, seed, lengths, H, bias, P=96, Tb=24, hd=64):
    d = H * hd
    inp = random_case(seed, lengths, d, H, hd, P=P, Tb=Tb, dtype="bf16", alibi=(bias == "alibi"))
    if bias in ("pos", "none"):
        inp.time_table = None
    if bias == "none":
        inp.pos_table = None
    p = inp.layers[0]
    uvqk = round_bf16(oracle.f1(inp.X, p.W1, p.b1))
    dav = round_bf16(np.random.default_rng(seed + 100).normal(0, 1.0, (inp.T, H * hd)))
    has_t = inp.time_table is not None
    ref = oracle.attention_bwd(inp.seq_offsets, uvqk, dav, num_heads=H, d_qk=hd, d_v=hd,
                               timestamps=inp.timestamps if has_t else None,
                               pos_table=inp.pos_table, time_table=inp.time_table,
                               alibi_slopes=inp.alibi_slopes, scale=inp.scale)
    Pn = 0 if inp.pos_table is None else inp.pos_table.shape[1]
    Tn = 0 if inp.time_table is None else inp.time_table.shape[1]
    s = hstu.make_shape(len(lengths), inp.T, int(max(lengths)), d, H, hd, hd, hstu.HSTU_BF16, Pn, Tn)
    f = lambda *shape: torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    dq, dk, dv = f(inp.T, H * hd), f(inp.T, H * hd), f(inp.T, H * hd)
    dpos = f(H, Pn) if Pn else None
    dtim = f(H, Tn) if Tn else None
    hstu.hstu_attention_bwd(s, dev(uvqk), dev(inp.seq_offsets), dev(inp.timestamps) if has_t else None,
                            dev(inp.pos_table, "f32"), dev(inp.time_table, "f32"),
                            dev(inp.alibi_slopes, "f32"), inp.scale, dev(dav), dq, dk, dv, dpos, dtim)
    assert hstu.device_status() == hstu.HSTU_OK
    got = {"dq": host(dq), "dk": host(dk), "dv": host(dv),
           "dpos": host(dpos) if dpos is not None else None,
           "dtime": host(dtim) if dtim is not None else None}
    return got, ref


@pytest.mark.gpu
@pytest.mark.parametrize("seed,lengths,H,bias", [
    (41, [300, 1, 129, 513], 2, "rab"),
    (42, [256, 1000], 2, "pos"),
    (43, [700, 31], 2, "alibi"),
    (44, [128, 255, 257], 1, "none"),
])
def test_attention_backward_matches_oracle(hstu, seed, lengths, H, bias):
    got, ref = _run(hstu, seed, lengths, H, bias)
    for k in ("dq", "dk", "dv"):
        assert_bf16_close(got[k], ref[k], f"{k} ({bias})")
    for k in ("dpos", "dtime"):
        if ref[k] is not None:
            assert_bf16_close(got[k], ref[k], f"{k} ({bias})")


@pytest.mark.gpu
def test_attention_backward_longer_sequences(hstu):
    got, ref = _run(hstu, 45, [2048, 1500], 2, "rab", P=1024, Tb=64)
    for k in ("dq", "dk", "dv", "dpos", "dtime"):
        assert_bf16_close(got[k], ref[k], f"{k} (2 x ~2k)")


@pytest.mark.gpu
@pytest.mark.parametrize("seed,lengths,H,bias", [
    (61, [300, 1, 129, 513], 2, "rab"),
    (62, [256, 0, 1000], 2, "pos"),
    (63, [700, 31], 2, "alibi"),
    (64, [128, 255, 257], 1, "none"),
    (65, [1, 2, 127, 128, 129], 3, "rab"),
])
def test_attention_backward_head_dim_128(hstu, seed, lengths, H, bias):
    """Head dim 128: dK, dV and the table gradients from the key-stationary kernel, dQ from the
    query-stationary one; ragged lengths around the 128-row tile, an empty sequence, one token."""
    got, ref = _run(hstu, seed, lengths, H, bias, hd=128)
    for k in ("dq", "dk", "dv"):
        assert_bf16_close(got[k], ref[k], f"{k} ({bias}, hd=128)")
    for k in ("dpos", "dtime"):
        if ref[k] is not None:
            assert_bf16_close(got[k], ref[k], f"{k} ({bias}, hd=128)")


@pytest.mark.gpu
def test_attention_backward_head_dim_128_longer(hstu):
    got, ref = _run(hstu, 66, [1800, 2100], 2, "rab", P=1024, Tb=64, hd=128)
    for k in ("dq", "dk", "dv", "dpos", "dtime"):
        assert_bf16_close(got[k], ref[k], f"{k} (2 x ~2k, hd=128)")


def test_backward_host_validation(hstu):
    lib = hstu.library()
    fake = ctypes.c_void_p(1 << 20)
    # head dims other than 64 and 128, and d_qk != d_v
    for hq, hv in ((32, 32), (256, 256), (64, 128)):
        sh = hstu.make_shape(1, 10, 10, 256, 2, hq, hv, hstu.HSTU_BF16, 16, 0)
        rc = lib.hstu_attention_bwd(ctypes.byref(sh), fake, fake, None, fake, None, None,
                                    ctypes.c_float(1.0), fake, fake, fake, fake, fake, None, fake,
                                    1 << 30, None)
        assert rc == hstu.HSTU_ERR_UNSUPPORTED, (hq, hv)
    s64 = hstu.make_shape(1, 10, 10, 128, 2, 64, 64, hstu.HSTU_BF16, 16, 0)
    # a position table without a place for its gradient
    rc = lib.hstu_attention_bwd(ctypes.byref(s64), fake, fake, None, fake, None, None,
                                ctypes.c_float(1.0), fake, fake, fake, fake, None, None, fake, 1 << 30, None)
    assert rc == hstu.HSTU_ERR_INVALID_ARG
