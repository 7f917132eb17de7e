"""The bounded-wait timeout path of the decode and prefill kernels, run on the
GPU without withholding any copy or tensor-core commit: with the main-loop wait
bound set below 1 us every wait gives up at once.  The kernel must report
KVQ_ERR_TIMEOUT, drain what it issued (with the full 1 s bound), leave the
decode merge counters at zero, and the next call with the default bound must be
correct."""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_20_b200 import kvq
from quantized_kv_cache_20_b200 import workloads as wl
from tests.helpers import DEV, assert_attn_close, bf16_to_f64, err_word, int32_scalar

pytestmark = pytest.mark.gpu


def test_decode_timeout_is_reported_and_the_next_call_is_correct():
    w = wl.DECODE
    g = wl.generator(31337)
    B, Hq, Hkv, D, S, n = w.B, w.Hq, w.Hkv, w.D, w.S, w.kv_len
    K = wl.int8_cache_like(B, Hkv, S, D, g)
    V = wl.int8_cache_like(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    Kd = [t.to(DEV) for t in K]
    Vd = [t.to(DEV) for t in V]
    qd = q.to(DEV)
    kv = int32_scalar(n)
    ws = kvq.decode_workspace(B, Hq, Hkv, D, S, DEV)
    lib = kvq.load()
    err = err_word()
    try:
        lib.kvq_set_wait_limit_ns(1)
        kvq.decode_attn(qd, *Kd, *Vd, kv, workspace=ws, err_word=err)
        torch.cuda.synchronize()
    finally:
        lib.kvq_set_wait_limit_ns(0)
    assert err.item() & kvq.KVQ_ERR_TIMEOUT, "the waits did not give up with a 1 ns bound"
    assert torch.count_nonzero(ws[:1024]).item() == 0, "merge counters left set after the aborted call"
    err = err_word()
    out = kvq.decode_attn(qd, *Kd, *Vd, kv, workspace=ws, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    rows = [(b, h, 0) for b in (0, 3, 7) for h in (0, 13, 31)]
    ref = oracle.sdpa_rows(wl.u16(q), *[t.numpy() for t in K], *[t.numpy() for t in V], kv_len=n,
                           sm_scale=1 / math.sqrt(D), rows=rows)
    got = bf16_to_f64(out)
    assert_attn_close(np.stack([got[b, h, i] for b, h, i in rows]), ref, "decode after a timeout")


@pytest.mark.parametrize("block_mode", [0, 2])
def test_prefill_timeout_is_reported_and_the_next_call_is_correct(block_mode):
    """The prefill roles (softmax, converters, MMA issuer) all give up at their
    first wait; the MMA thread still drains its commits before TMEM is freed."""
    g = wl.generator(31338 + block_mode)
    B, Hq, Hkv, D, S, Lq, n = 1, 8, 2, 128, 1024, 256, 1000
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    qd = q.to(DEV)
    kv = int32_scalar(n)
    if block_mode == 0:
        K = [t.to(DEV) for t in wl.int8_cache_like(B, Hkv, S, D, g)]
        V = [t.to(DEV) for t in wl.int8_cache_like(B, Hkv, S, D, g)]
        run = lambda e: kvq.prefill_attn(qd, *K, *V, kv, is_causal=True, mask_is_causal=True, err_word=e)
    else:
        K, V = [], []
        for c in (K, V):  # a cache written by kvq_write (valid codes only)
            x = wl.bf16_normal((B, Hkv, S, D), g)
            c += [torch.zeros((B, Hkv, S, D), dtype=torch.uint8, device=DEV),
                  torch.zeros((B, Hkv, S, D // 32), dtype=torch.uint8, device=DEV)]
            kvq.write(block_mode, x.to(DEV), torch.arange(S, dtype=torch.int32, device=DEV), *c)
        run = lambda e: kvq.prefill_attn_block(block_mode, qd, *K, *V, kv, is_causal=True, mask_is_causal=True,
                                               err_word=e)
    lib = kvq.load()
    err = err_word()
    try:
        lib.kvq_set_wait_limit_ns(1)
        run(err)
        torch.cuda.synchronize()
    finally:
        lib.kvq_set_wait_limit_ns(0)
    assert err.item() & kvq.KVQ_ERR_TIMEOUT, "the waits did not give up with a 1 ns bound"
    err = err_word()
    out = run(err)
    torch.cuda.synchronize()
    assert err.item() == 0
    rows = [(0, h, i) for h in (0, 3, 7) for i in (0, 100, 255)]
    if block_mode == 0:
        ref = oracle.sdpa_rows(wl.u16(q), *[t.cpu().numpy() for t in K], *[t.cpu().numpy() for t in V], kv_len=n,
                               sm_scale=1 / math.sqrt(D), rows=rows, is_causal=True)
    else:
        Kf = oracle.dequant_block(block_mode, K[0].cpu().numpy(), K[1].cpu().numpy())
        Vf = oracle.dequant_block(block_mode, V[0].cpu().numpy(), V[1].cpu().numpy())
        ref = oracle.sdpa_dense_rows(wl.u16(q), Kf, Vf, n, 1 / math.sqrt(D), rows, is_causal=True)
    got = bf16_to_f64(out)
    assert_attn_close(np.stack([got[b, h, i] for b, h, i in rows]), ref, "prefill after a timeout")
