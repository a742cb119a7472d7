"""The C-ABI library loads, exports every symbol include/mk.h declares, and
validates arguments on the host (no device needed)."""
import ctypes as C

import pytest

import attention_decode_megakernel_b200 as mk
from attention_decode_megakernel_b200 import build, synth


@pytest.fixture(scope="module")
def L():
    build.build()
    return mk.lib()


def test_every_declared_symbol_is_exported(L):
    names = mk.header_symbols()
    assert "mk_create" in names and "mk_decode_step" in names and "mk_delta_step" in names
    for n in names:
        assert hasattr(L, n), n


def test_workspace_bytes_and_config_validation(L):
    tiny = mk.mk_workspace_bytes(synth.tiny_config(max_ctx=256))
    big = mk.mk_workspace_bytes(synth.hybrid_08b_config(max_ctx=4096))
    assert 0 < tiny < big
    # 9 state buffers of 18.9 MB + a 4096-position bf16 KV cache dominate
    assert big > 9 * 18 * 16 * 128 * 128 * 4 + 6 * 2 * 2 * 4096 * 256 * 2
    c = mk.make_config(synth.tiny_config())
    c.n_layers = 0
    assert L.mk_workspace_bytes(C.byref(c)) == 0
    c = mk.make_config(synth.tiny_config())
    c.max_verify = 9
    assert L.mk_workspace_bytes(C.byref(c)) == 0


def test_host_side_argument_errors(L):
    h = C.c_void_p()
    assert L.mk_create(None, None, None, 0, None, C.byref(h)) == mk.MK_ERR_ARG
    assert L.mk_create(C.byref(mk.make_config(synth.tiny_config())), None, None, 0, None,
                       None) == mk.MK_ERR_ARG
    assert L.mk_reset(None) == mk.MK_ERR_ARG
    assert L.mk_decode_step(None, 0, None) == mk.MK_ERR_ARG
    assert L.mk_accept(None, 1) == mk.MK_ERR_ARG
    assert L.mk_position(None) == -1
    assert L.mk_delta_step(None, None, None, None, None, None, None, 1, 16, 128, 128,
                           None) == mk.MK_ERR_ARG


def test_strerror_covers_every_status(L):
    seen = set()
    for code in range(8):
        s = mk.mk_strerror(code)
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 8
    assert mk.mk_strerror(99) == "unknown status"
