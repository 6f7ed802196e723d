"""The C ABI library loads, exports every symbol include/hstu.h declares, and rejects invalid
arguments on the host before touching a GPU (no GPU needed: nothing here launches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu.h")


@pytest.fixture(scope="module")
def hstu():
    from hstu_sequential_transduction_layer_b200 import build
    build.build()
    import hstu_sequential_transduction_layer_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["hstu_layer_fwd", "hstu_layer_fwd_workspace_size", "hstu_f1_fwd",
              "hstu_attention_fwd", "hstu_ln_gate_fwd", "hstu_f2_fwd", "hstu_token_embed_fwd",
              "hstu_status_string", "hstu_get_device_status"]:
        assert n in names


def test_library_exports_every_declared_symbol(hstu):
    lib = hstu.library()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in hstu.h but not exported"
    assert sorted(hstu.EXPORTED) == declared_functions()


def test_exports_are_plain_c_symbols(hstu):
    out = os.popen(f"nm -D --defined-only {hstu.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, re.M), f"{name} is not an unmangled text symbol"


def test_status_strings(hstu):
    assert hstu.status_string(0) == "HSTU_OK"
    assert hstu.status_string(1) == "HSTU_ERR_INVALID_ARG"
    assert hstu.status_string(5) == "HSTU_ERR_DEVICE_BAD_OFFSETS"
    assert hstu.status_string(99) == "HSTU_ERR_UNKNOWN"
    assert hstu.version().count(".") == 2


def _shape(hstu, **kw):
    base = dict(num_seqs=2, total_tokens=100, max_seq_len=64, d_model=128, num_heads=2, d_qk=64,
                d_v=64, dtype=hstu.HSTU_BF16, n_pos_buckets=16, n_time_buckets=8)
    base.update(kw)
    return hstu.make_shape(**base)


def test_workspace_size(hstu):
    s = _shape(hstu)
    n = hstu.workspace_size(s)
    T, n1, wv = 100, 4 * 128, 128
    assert n >= 2 * (T * n1 + 2 * T * wv)
    assert hstu.workspace_size(_shape(hstu, d_model=0)) == 0            # invalid shape
    assert hstu.workspace_size(_shape(hstu, d_qk=32, d_v=32)) == 0      # unsupported bf16 head size
    f32 = _shape(hstu, dtype=hstu.HSTU_F32, d_qk=32, d_v=32, d_model=64)
    assert hstu.workspace_size(f32) >= 4 * (100 * 256 + 2 * 100 * 64)


FAKE = 1 << 20  # an aligned address that is never dereferenced: validation fails before any use


def _call_layer(hstu, shape, **ptrs):
    P = {k: ctypes.c_void_p(FAKE + 4096 * i) for i, k in enumerate(
        ["X", "off", "ts", "W1", "b1", "W2", "b2", "lnw", "lnb", "pos", "tim", "ali", "out", "ws"])}
    P["ali"] = None
    P.update(ptrs)
    return hstu.library().hstu_layer_fwd(
        ctypes.byref(shape), P["X"], P["off"], P["ts"], P["W1"], P["b1"], P["W2"], P["b2"],
        P["lnw"], P["lnb"], P["pos"], P["tim"], P["ali"], ctypes.c_float(1 / 64), P["out"], P["ws"],
        ptrs.get("ws_bytes", 1 << 40), None)


def test_host_validation_rejects_bad_arguments(hstu):
    ok = _shape(hstu)
    E, U = hstu.HSTU_ERR_INVALID_ARG, hstu.HSTU_ERR_UNSUPPORTED
    assert _call_layer(hstu, _shape(hstu, num_seqs=-1)) == E
    assert _call_layer(hstu, _shape(hstu, dtype=7)) == E
    assert _call_layer(hstu, _shape(hstu, d_model=96)) == U             # bf16 needs d % 64 == 0
    assert _call_layer(hstu, _shape(hstu, d_qk=64, d_v=128)) == U
    assert _call_layer(hstu, ok, X=None) == E
    assert _call_layer(hstu, ok, W1=ctypes.c_void_p(FAKE + 2)) == E     # misaligned for bf16
    assert _call_layer(hstu, ok, ali=ctypes.c_void_p(FAKE)) == E        # ALiBi together with tables
    assert _call_layer(hstu, ok, ts=None) == E                          # time table needs timestamps
    assert _call_layer(hstu, ok, out=ctypes.c_void_p(FAKE)) == E        # out aliases X
    assert _call_layer(hstu, ok, ws_bytes=16) == E                      # workspace too small
    assert _call_layer(hstu, _shape(hstu, num_seqs=0)) == E             # tokens without sequences
    # an empty batch is a no-op and succeeds without touching anything
    assert _call_layer(hstu, _shape(hstu, num_seqs=0, total_tokens=0)) == hstu.HSTU_OK
    lib = hstu.library()
    assert lib.hstu_token_embed_fwd(10, 12, None, None, None, 5, None, 5, None, None) == E  # d % 8
    assert lib.hstu_token_embed_fwd(0, 16, None, None, None, 5, None, 5, None, None) == hstu.HSTU_OK


def test_ln_f2_host_validation(hstu):
    # the fused LayerNorm * U -> f2 entry point covers bf16 with H*d_v == d in {128, 256, 512}
    lib = hstu.library()
    E, U = hstu.HSTU_ERR_INVALID_ARG, hstu.HSTU_ERR_UNSUPPORTED
    P = [ctypes.c_void_p(FAKE + 4096 * i) for i in range(8)]

    def call(shape, ptrs=P):
        return lib.hstu_ln_f2_fwd(ctypes.byref(shape), *ptrs, None)

    assert call(_shape(hstu, d_model=192, num_heads=3)) == U            # d not 128/256/512
    assert call(_shape(hstu, d_model=256, num_heads=2)) == U            # H*d_v != d
    assert call(_shape(hstu, dtype=hstu.HSTU_F32, d_qk=32, d_v=32, d_model=64)) == U
    assert call(_shape(hstu), [None] + P[1:]) == E                      # no AV
    assert call(_shape(hstu), P[:7] + [ctypes.c_void_p(FAKE + 2)]) == E  # misaligned out
    assert call(_shape(hstu), P[:7] + [P[6]]) == E                      # out aliases X
    assert call(_shape(hstu, num_seqs=0, total_tokens=0)) == hstu.HSTU_OK
