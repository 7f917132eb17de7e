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


@pytest.mark.parametrize("shape", [(8, 32, 8, 128, 8192, (4096, 1500)), (2, 4, 2, 256, 2048, (2048, 77))])
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


def _static_call(q, K, V, kv, out, B, Hq, Hkv, D, S):
    lib = kvq.load()
    return lib.kvq_decode_attn_static(
        ctypes.c_void_p(q.data_ptr()), B, Hq, Hkv, D, *[ctypes.c_void_p(t.data_ptr()) for t in K],
        *[ctypes.c_void_p(t.data_ptr()) for t in V], S, ctypes.c_void_p(kv.data_ptr()), None,
        ctypes.c_float(1.0 / math.sqrt(D)), ctypes.c_void_p(out.data_ptr()), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# (B, Hq, Hkv, D, S, kv_len): D 256 -> 64 -> 128, then the q heads per kv head
# change, then the batch, then D 256 again.  Each shape moves the partial
# records to other offsets of the one shared buffer; the merge counters must not.
SEQUENCE = [(2, 4, 2, 256, 2048, 2048), (3, 8, 2, 64, 2048, 1999), (2, 16, 4, 128, 1024, 1024),
            (2, 12, 4, 128, 2048, 1537), (5, 4, 2, 64, 1024, 1000), (1, 6, 2, 256, 4096, 3000)]


def test_static_scratch_serves_a_sequence_of_shapes():
    """Calls of different shapes one after another on the one static buffer, each
    checked against the fp64 oracle (and, for good measure, the workspace path)."""
    import numpy as np
    import oracle
    for i, (B, Hq, Hkv, D, S, n) in enumerate(SEQUENCE):
        g = wl.generator(4321 + i)
        Kc = wl.int8_cache_like(B, Hkv, S, D, g)
        Vc = wl.int8_cache_like(B, Hkv, S, D, g)
        qc = wl.bf16_normal((B, Hq, 1, D), g)
        K = [t.to(DEV) for t in Kc]
        V = [t.to(DEV) for t in Vc]
        q = qc.to(DEV)
        kv = int32_scalar(n)
        got = torch.empty_like(q)
        st = _static_call(q, K, V, kv, got, B, Hq, Hkv, D, S)
        assert st == kvq.KVQ_OK, kvq.strerror(st)
        torch.cuda.synchronize()
        ref = oracle.sdpa(wl.u16(qc), *[t.numpy() for t in Kc], *[t.numpy() for t in Vc], kv_len=n,
                          sm_scale=1 / math.sqrt(D))
        assert_attn_close(got.float().cpu().double().numpy(), ref, f"static scratch call {i} {B, Hq, Hkv, D}")
        assert torch.equal(got, kvq.decode_attn(q, *K, *V, kv)), f"call {i}: static and workspace paths differ"
        assert np.isfinite(ref).all()


def test_static_scratch_rejects_problems_that_do_not_fit():
    # D = 256 with 4 q heads per kv head: two partial records of 4 x 256 floats
    # per CTA take 1.2 MB, more than the 1 MiB buffer
    B, Hq, Hkv, D, S = 1, 8, 2, 256, 1024
    assert kvq.decode_workspace_bytes(B, Hq, Hkv, D, S) > kvq.STATIC_SCRATCH_BYTES
    lib = kvq.load()
    fake = ctypes.c_void_p(256)
    st = lib.kvq_decode_attn_static(fake, B, Hq, Hkv, D, fake, fake, fake, fake, fake, fake, S, fake, None,
                                    ctypes.c_float(0.1), fake, None, None)
    assert st == kvq.KVQ_ESCRATCH
