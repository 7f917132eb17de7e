"""The C-ABI library loads and exports every entry point include/kvq.h declares
(CPU only: no kernel is launched)."""
import ctypes
import os
import re

import pytest

from quantized_kv_cache_20_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    path = kbuild.build()
    import torch  # noqa: F401  (loads the shared CUDA runtime first, as the binding does)
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("kvq_write", "kvq_decode_attn", "kvq_prefill_attn", "kvq_sink_plan", "kvq_sink_mask",
              "kvq_decode_workspace_bytes", "kvq_strerror", "kvq_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_declares_the_same_symbols():
    from quantized_kv_cache_20_b200 import kvq
    assert sorted(kvq.EXPORTS) == _declared()


def test_host_only_calls(lib):
    lib.kvq_strerror.restype = ctypes.c_char_p
    assert lib.kvq_strerror(0) == b"ok"
    assert b"invalid" in lib.kvq_strerror(-1)
    assert lib.kvq_version() >= 100


def test_argument_checks_reject_before_any_launch(lib):
    P = ctypes.c_void_p
    lib.kvq_write.argtypes = [ctypes.c_int, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_int, P, P, ctypes.c_int64, P, P, P, P, P]
    strides = (ctypes.c_int64 * 4)(8, 8, 8, 1)
    fake = P(16)
    # unknown mode
    assert lib.kvq_write(9, 1, fake, 1, 1, 1, 64, strides, fake, 8, fake, fake, fake, None, None) == -1
    # round_scale is one of the three scale rules
    assert lib.kvq_write(2, 3, fake, 1, 1, 1, 64, strides, fake, 8, fake, fake, fake, None, None) == -1
    assert lib.kvq_write(3, -1, fake, 1, 1, 1, 64, strides, fake, 8, fake, fake, fake, None, None) == -1
    # int8 mode needs D in {64, 128, 256}
    assert lib.kvq_write(0, 1, fake, 1, 1, 1, 96, strides, fake, 8, fake, fake, fake, None, None) == -2
    # block modes need d % 32 == 0 and d <= 8192
    assert lib.kvq_write(1, 1, fake, 1, 1, 1, 48, strides, fake, 8, fake, fake, None, None, None) == -2
    assert lib.kvq_write(1, 1, fake, 1, 1, 1, 8224, strides, fake, 8, fake, fake, None, None, None) == -2
    # float-scale modes (1, 4, 6) need 4-byte aligned scales
    for m in (1, 4, 6):
        assert lib.kvq_write(m, 1, fake, 1, 1, 1, 64, strides, fake, 8, fake, P(17), None, None, None) == -1
    # the new modes take the block-mode size rules
    for m in (4, 5, 6):
        assert lib.kvq_write(m, 1, fake, 1, 1, 1, 48, strides, fake, 8, fake, fake, None, None, None) == -2
    # null x
    assert lib.kvq_write(0, 1, None, 1, 1, 1, 64, strides, fake, 8, fake, fake, fake, None, None) == -1
    # misaligned x
    assert lib.kvq_write(0, 1, P(18), 1, 1, 1, 64, strides, fake, 8, fake, fake, fake, None, None) == -1
    # empty work is a no-op
    assert lib.kvq_write(0, 1, fake, 0, 1, 1, 64, strides, fake, 8, fake, fake, fake, None, None) == 0


def test_write_kv_argument_checks_reject_before_any_launch(lib):
    """kvq_write_kv checks both tensors and the shared arguments on the host."""
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.kvq_write_kv.argtypes = [I, I, P, P, I, I, I, I, P, P, P, I64, P, P, P, P, P, P, P, P]
    st = (ctypes.c_int64 * 4)(8, 8, 8, 1)
    f = P(16)

    def call(mode=0, k=f, v=f, D=64, B=1, ks=st, vs=st, sm=f, kc=f, ksc=f, kz=f, vc=f, vsc=f, vz=f):
        return lib.kvq_write_kv(mode, 1, k, v, B, 1, 1, D, ks, vs, sm, 8, kc, ksc, kz, vc, vsc, vz, None, None)

    assert call(mode=9) == -1                      # unknown mode
    assert call(D=96) == -2                        # int8 affine needs D in {64, 128, 256}
    assert call(v=None) == -1                      # null v
    assert call(v=P(24)) == -1                     # misaligned v
    assert call(vs=(ctypes.c_int64 * 4)(8, 8, 4, 1)) == -1   # V row stride not a multiple of 8 elements
    assert call(vz=None) == -1                     # int8 affine needs the V zero points
    assert call(sm=None) == -1                     # null slot_mapping
    assert call(mode=1, ksc=P(17), kz=None, vz=None) == -1  # float scales 4-byte aligned
    assert call(B=0) == 0                          # empty work is a no-op
