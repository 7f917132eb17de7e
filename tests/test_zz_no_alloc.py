"""The decode entry point that allocates nothing (kvq_decode_attn_static).

Some callers cannot hand the library a workspace: runtimes that own all device
memory from start-up, plain C hosts without a device allocator, decode loops
that must not allocate.  For them the library keeps its own scratch buffer in
its image.  This file checks, through the C ABI, that two calls in a row give
the same results as the workspace entry point, within the attention tolerance
the other tests use.  It is collected last, and passes alone in a fresh
process (the first call sets up the buffer's device address) as well as after
the other tests.
"""
import ctypes
import math

import pytest
import torch

from quantized_kv_cache_20_b200 import kvq
from quantized_kv_cache_20_b200 import workloads as wl
from tests.helpers import DEV, assert_attn_close, int32_scalar

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Hq, Hkv, D, S):
    g = wl.generator(seed)
    K = [t.to(DEV) for t in wl.int8_cache_like(B, Hkv, S, D, g)]
    V = [t.to(DEV) for t in wl.int8_cache_like(B, Hkv, S, D, g)]
    q = wl.bf16_normal((B, Hq, 1, D), g).to(DEV)
    return q, K, V


@pytest.mark.parametrize("shape", [(8, 32, 8, 128, 8192, (4096, 1500)), (2, 8, 2, 256, 2048, (2048, 77))])
def test_static_scratch_decode_matches_workspace_decode(shape):
    B, Hq, Hkv, D, S, kvs = shape
    q, K, V = _inputs(1234 + D, B, Hq, Hkv, D, S)
    lib = kvq.load()
    for n in kvs:  # two calls in a row on the shared buffer
        kv = int32_scalar(n)
        ref = kvq.decode_attn(q, *K, *V, kv)
        got = torch.empty_like(q)
        st = lib.kvq_decode_attn_static(
            ctypes.c_void_p(q.data_ptr()), B, Hq, Hkv, D, *[ctypes.c_void_p(t.data_ptr()) for t in K],
            *[ctypes.c_void_p(t.data_ptr()) for t in V], S, ctypes.c_void_p(kv.data_ptr()), None,
            ctypes.c_float(1.0 / math.sqrt(D)), ctypes.c_void_p(got.data_ptr()), None,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == kvq.KVQ_OK, kvq.strerror(st)
        torch.cuda.synchronize()
        assert_attn_close(got.float().cpu().double().numpy(), ref.float().cpu().double().numpy(),
                          f"static scratch kv_len={n}")


def test_static_scratch_rejects_problems_that_do_not_fit():
    # the workspace holds one merge counter per (batch row, kv head, head chunk):
    # 40000 x 64 x 2 of them take 20 MB, more than the 8 MiB buffer
    B, Hq, Hkv, D, S = 40000, 512, 64, 256, 16
    assert kvq.decode_workspace_bytes(B, Hq, Hkv, D, S) > kvq.STATIC_SCRATCH_BYTES
    lib = kvq.load()
    fake = ctypes.c_void_p(256)
    st = lib.kvq_decode_attn_static(fake, B, Hq, Hkv, D, fake, fake, fake, fake, fake, fake, S, fake, None,
                                    ctypes.c_float(0.1), fake, None, None)
    assert st == kvq.KVQ_ESCRATCH
