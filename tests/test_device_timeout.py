"""Failure detection on the device without a fault: the bounded mbarrier wait that every pipelined
kernel uses must give up on a barrier that nothing completes, report HSTU_ERR_DEVICE_TIMEOUT through
the device status word, make later waits of the block return at once, and leave the context usable.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import assert_bf16_close, dev, host, round_bf16


@pytest.fixture(scope="module")
def hstu():
    import hstu_sequential_transduction_layer_b200 as m
    return m


@pytest.mark.gpu
def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable(hstu):
    assert hstu.device_status() == hstu.HSTU_OK        # also clears anything left before
    limit = 20_000_000                                  # 20 ms
    res = torch.full((4,), -1, dtype=torch.int64, device="cuda")
    hstu.selftest_bounded_wait(limit, res)
    status = hstu.device_status()
    first_ok, second_ok, first_ns, second_ns = host(res).tolist()
    assert status == hstu.HSTU_ERR_DEVICE_TIMEOUT
    assert first_ok == 0 and second_ok == 0
    assert limit <= first_ns < limit + 100_000_000      # gave up after the limit, not much later
    assert second_ns < limit // 2                       # the raised flag ends the next wait early
    assert hstu.device_status() == hstu.HSTU_OK        # reading cleared the word

    # the context still runs kernels correctly
    rng = np.random.default_rng(5)
    T, d = 200, 128
    X = round_bf16(rng.standard_normal((T, d)))
    W1 = round_bf16(rng.uniform(-1, 1, (d, 4 * d)) * np.sqrt(6 / (5 * d)))
    b1 = round_bf16(rng.normal(0, 0.1, 4 * d))
    s = hstu.make_shape(1, T, T, d, 2, 64, 64, hstu.HSTU_BF16)
    out = torch.empty((T, 4 * d), dtype=torch.bfloat16, device="cuda")
    hstu.hstu_f1_fwd(s, dev(X), dev(W1), dev(b1), out)
    assert hstu.device_status() == hstu.HSTU_OK
    assert_bf16_close(host(out), oracle.f1(X, W1, b1), "f1 after the timeout self-test")


@pytest.mark.parametrize("limit", [0, 1_000_000_001])
def test_selftest_rejects_limits_out_of_range_before_launch(hstu, limit):
    fake = ctypes.c_void_p(1 << 20)
    rc = hstu.library().hstu_selftest_bounded_wait(limit, fake, None)
    assert rc == hstu.HSTU_ERR_INVALID_ARG
