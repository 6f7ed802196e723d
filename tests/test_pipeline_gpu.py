"""The host-to-host layer pipeline (copy in, layer, copy out on three streams) against direct
hstu_layer_fwd calls on the same batches, bit for bit, and its argument checks."""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import dev, host
from workloads import random_case


@pytest.fixture(scope="module")
def hstu():
    import hstu_sequential_transduction_layer_b200 as m
    return m


def _batch(seed, lengths, d=128, H=2):
    return random_case(seed, lengths, d, H, 64, P=64, Tb=16, dtype="bf16")


@pytest.mark.gpu
def test_pipeline_matches_direct_calls_bit_for_bit(hstu):
    batches = [_batch(61, [300, 1, 129]), _batch(62, [77, 512]), _batch(63, [1000]),
               _batch(64, [5, 6, 7, 8]), _batch(65, [256, 255])]
    base = batches[0]
    p = base.layers[0]
    w = base.workload
    params = [dev(a) for a in (p.W1, p.b1, p.W2, p.b2, p.ln_w, p.ln_b)]
    pos, tim = dev(base.pos_table, "f32"), dev(base.time_table, "f32")
    cap = hstu.make_shape(8, 1200, 1024, w.d_model, w.num_heads, 64, 64, hstu.HSTU_BF16,
                          base.pos_table.shape[1], base.time_table.shape[1], base.ln_eps)
    pipe = hstu.LayerPipeline(cap, depth=2)
    outs, refs = [], []
    for inp in batches:
        X = torch.from_numpy(host(dev(inp.X)).astype(np.float32)).to(torch.bfloat16).pin_memory()
        off = torch.from_numpy(inp.seq_offsets).pin_memory()
        ts = torch.from_numpy(inp.timestamps).pin_memory()
        out = torch.full_like(X, float("nan")).pin_memory()
        s = hstu.make_shape(len(inp.lengths), inp.T, int(inp.lengths.max()), w.d_model,
                            w.num_heads, 64, 64, hstu.HSTU_BF16, base.pos_table.shape[1],
                            base.time_table.shape[1], base.ln_eps)
        pipe.submit(s, X, off, ts, *params, pos, tim, None, base.scale, out)
        outs.append(out)
        ref = hstu.hstu_layer_fwd(X.cuda(), off.cuda(), ts.cuda(), *params, pos, tim, None,
                                  base.scale, num_heads=w.num_heads,
                                  max_seq_len=int(inp.lengths.max()), ln_eps=base.ln_eps)
        refs.append(ref.cpu())
    pipe.sync()
    pipe.close()
    assert hstu.device_status() == hstu.HSTU_OK
    for o, r in zip(outs, refs):
        assert torch.equal(o.view(torch.int16), r.view(torch.int16))


def test_pipeline_argument_checks(hstu):
    lib = hstu.library()
    cap = hstu.make_shape(2, 100, 64, 128, 2, 64, 64, hstu.HSTU_BF16, 16, 8)
    out = ctypes.c_void_p()
    # depth below 2: refused before any device call
    assert lib.hstu_layer_pipeline_create(ctypes.byref(cap), 1, ctypes.byref(out)) == \
        hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_layer_pipeline_create(ctypes.byref(cap), 2, None) == hstu.HSTU_ERR_INVALID_ARG
    empty = hstu.make_shape(0, 0, 0, 128, 2, 64, 64, hstu.HSTU_BF16, 16, 8)
    assert lib.hstu_layer_pipeline_create(ctypes.byref(empty), 2, ctypes.byref(out)) == \
        hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_layer_pipeline_sync(None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_layer_pipeline_submit(None, ctypes.byref(cap), *([None] * 12),
                                          ctypes.c_float(1.0), None) == hstu.HSTU_ERR_INVALID_ARG
    lib.hstu_layer_pipeline_destroy(None)
