"""GPU parity of kvq_decode_attn / kvq_prefill_attn against the fp64 oracle:
|gpu - oracle| <= 2e-3 + 1e-2 |oracle| element by element, plus the
bit-identities the pages fix (per-tile causal skip on/off, kv_len = S)."""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_20_b200 import kvq
from quantized_kv_cache_20_b200 import workloads as wl
from tests.helpers import DEV, assert_attn_close, bf16_to_f64, err_word, int32_scalar

pytestmark = pytest.mark.gpu


def _cache(B, Hkv, S, D, g):
    K = wl.int8_cache_like(B, Hkv, S, D, g)
    V = wl.int8_cache_like(B, Hkv, S, D, g)
    return K, V


def _np(c):
    return [t.numpy() for t in c]


def _decode_gpu(q, K, V, kv_len, mask=None, sm=None, err=None):
    Kd = [t.to(DEV) for t in K]
    Vd = [t.to(DEV) for t in V]
    out = kvq.decode_attn(q.to(DEV), *Kd, *Vd, int32_scalar(kv_len) if isinstance(kv_len, int) else kv_len,
                          mask=None if mask is None else mask.to(DEV), sm_scale=sm, err_word=err)
    torch.cuda.synchronize()
    return out


# ---------------------------------------------------------------------------- decode

def test_tiny_write_then_decode():
    """16 tokens x 2 kv heads, D=64, written at random slots of a 64-slot cache;
    4 q heads (GQA 2:1) attend at kv_len 40.  The oracle writes its own cache."""
    w = wl.TINY
    g = wl.generator(w.seed)
    k = wl.bf16_normal((w.B, w.Hkv, w.T, w.D), g)
    v = wl.bf16_normal((w.B, w.Hkv, w.T, w.D), g)
    sm = wl.slot_mapping_random(w.T, w.S, 3, g)
    K0 = wl.int8_cache_like(w.B, w.Hkv, w.S, w.D, g)
    V0 = wl.int8_cache_like(w.B, w.Hkv, w.S, w.D, g)
    q = wl.bf16_normal((w.B, w.Hq, 1, w.D), g)
    Kd = [t.to(DEV) for t in K0]
    Vd = [t.to(DEV) for t in V0]
    kvq.write(0, k.to(DEV), sm.to(DEV), *Kd)
    kvq.write(0, v.to(DEV), sm.to(DEV), *Vd)
    out = kvq.decode_attn(q.to(DEV), *Kd, *Vd, int32_scalar(w.kv_len))
    Ko = [t.numpy().copy() for t in K0]
    Vo = [t.numpy().copy() for t in V0]
    oracle.write(0, wl.u16(k), sm.numpy(), w.S, *Ko)
    oracle.write(0, wl.u16(v), sm.numpy(), w.S, *Vo)
    ref = oracle.sdpa(wl.u16(q), *Ko, *Vo, kv_len=w.kv_len, sm_scale=1 / math.sqrt(w.D))
    assert_attn_close(bf16_to_f64(out), ref, "tiny")


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (6, 2), (8, 2), (16, 2), (10, 2)])
@pytest.mark.parametrize("kv_len", [1, 37, 200, 512])
def test_decode_shapes(D, Hq, Hkv, kv_len):
    g = wl.generator(D * 7 + Hq * 3 + kv_len)
    B, S = 2, 512
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    out = _decode_gpu(q, K, V, kv_len)
    ref = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=kv_len, sm_scale=1 / math.sqrt(D))
    assert_attn_close(bf16_to_f64(out), ref, f"D={D} Hq={Hq} Hkv={Hkv} kv={kv_len}")


def test_decode_with_additive_mask():
    g = wl.generator(77)
    B, Hq, Hkv, D, S = 1, 8, 2, 128, 256
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    rng = np.random.default_rng(1)
    m = np.where(rng.random(S) < 0.4, -np.inf, rng.normal(size=S) * 2).astype(np.float32)
    m[5] = 0.0
    mask = torch.from_numpy(m).reshape(1, S)
    out = _decode_gpu(q, K, V, 230, mask=mask)
    ref = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=230, sm_scale=1 / math.sqrt(D), mask=m.reshape(1, S))
    assert_attn_close(bf16_to_f64(out), ref, "mask")


def test_decode_config_full_size():
    """batch 8, 32 q / 8 kv heads, D=128, 8192 slots, kv_len 4096 read on device."""
    w = wl.DECODE
    g = wl.generator(w.seed)
    K, V = _cache(w.B, w.Hkv, w.S, w.D, g)
    q = wl.bf16_normal((w.B, w.Hq, 1, w.D), g)
    out = _decode_gpu(q, K, V, w.kv_len)
    ref = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=w.kv_len, sm_scale=1 / math.sqrt(w.D))
    assert_attn_close(bf16_to_f64(out), ref, "decode config")


@pytest.mark.parametrize("B,Hkv,G,D,kv_len", [
    (12, 8, 4, 128, 1000),   # 96 units: one CTA a unit (k = 1), no merge
    (5, 8, 4, 128, 1500),    # 40 units: three CTAs a unit (k = 3), counter merge
    (8, 8, 4, 128, 50),      # 64 units of one chunk: the second CTA of every pair has none
    (8, 8, 4, 128, 8000),    # 64 units of 125 chunks: the flattened split takes fewer rounds
    (37, 2, 4, 128, 700),    # 74 units: every CTA streams, as cluster pairs
    (4, 8, 8, 64, 3000),     # 32 units (one head chunk of 8): four CTAs a unit
    (16, 4, 2, 256, 760),    # D = 256 (two buffers a warp), 64 units of 24 chunks in pairs
])
def test_decode_split_choices(B, Hkv, G, D, kv_len):
    """The kernel picks its split from the shape and the kv_len it reads: the
    flattened cut over every CTA, or U k CTAs that each take a k-th of one unit
    (merged in pairs through distributed shared memory when k = 2)."""
    g = wl.generator(B * 7 + Hkv * 13 + G + D + kv_len)
    S = (kv_len + 63) // 64 * 64 + 64
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hkv * G, 1, D), g)
    out = _decode_gpu(q, K, V, kv_len)
    ref = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=kv_len, sm_scale=1 / math.sqrt(D))
    assert_attn_close(bf16_to_f64(out), ref, f"decode split B={B} Hkv={Hkv} G={G} D={D} kv={kv_len}")


def test_long_config_decode_full_size():
    """batch 1, 32 q / 16 kv heads, D=256, kv_len = 131072 (the whole cache)."""
    w = wl.LONG
    g = wl.generator(w.seed + 100)
    K, V = _cache(w.B, w.Hkv, w.S, w.D, g)
    q = wl.bf16_normal((w.B, w.Hq, 1, w.D), g)
    out = _decode_gpu(q, K, V, w.kv_len)
    rows = [(0, h, 0) for h in range(w.Hq)]
    ref = oracle.sdpa_rows(wl.u16(q), *_np(K), *_np(V), kv_len=w.kv_len, sm_scale=1 / math.sqrt(w.D), rows=rows)
    assert_attn_close(bf16_to_f64(out)[0, :, 0], ref, "long decode")


def test_sink_config_decode_steps():
    """4 sink + 2044 ring slots: plan -> write K/V -> mask -> decode for positions
    0 .. 10000, checked around the first wrap (2048), the second (4096), the
    third (6143) and at the end (10000); the oracle keeps its own cache and plan."""
    w = wl.SINK
    g = wl.generator(w.seed)
    S, D = w.S, w.D
    K0 = wl.int8_cache_random(1, w.Hkv, S, D, g)
    V0 = wl.int8_cache_random(1, w.Hkv, S, D, g)
    Kd = [t.to(DEV) for t in K0]
    Vd = [t.to(DEV) for t in V0]
    Ko = [t.numpy().copy() for t in K0]
    Vo = [t.numpy().copy() for t in V0]
    sp_d = torch.full((S,), -1, dtype=torch.int32, device=DEV)
    sp_o = np.full(S, -1, np.int32)
    ip = torch.zeros(1, dtype=torch.int32, device=DEV)
    sm_d = torch.empty(1, dtype=torch.int32, device=DEV)
    kv_d = torch.empty(1, dtype=torch.int32, device=DEV)
    mask_d = torch.empty((1, S), dtype=torch.float32, device=DEV)
    ws = kvq.decode_workspace(1, w.Hq, w.Hkv, D, S, DEV)
    checks = {0, 3, 4, 5, 2047, 2048, 2049, 2300, 4095, 4096, 6143, 10000}
    last = max(checks)
    gen = wl.generator(w.seed + 1)
    for p in range(last + 1):
        k = wl.bf16_normal((1, w.Hkv, 1, D), gen)
        v = wl.bf16_normal((1, w.Hkv, 1, D), gen)
        ip.fill_(p)
        kvq.sink_plan(ip, 1, 1, w.sink, sp_d, sm_d, kv_d)
        kvq.write(0, k.to(DEV), sm_d, *Kd)
        kvq.write(0, v.to(DEV), sm_d, *Vd)
        sm_o, kv_o = oracle.sink_plan(p, 1, 1, w.sink, S, sp_o)
        oracle.write(0, wl.u16(k), sm_o, S, *Ko)
        oracle.write(0, wl.u16(v), sm_o, S, *Vo)
        if p in checks:
            q = wl.bf16_normal((1, w.Hq, 1, D), gen)
            kvq.sink_mask(ip, 1, sp_d, mask_d)
            out = kvq.decode_attn(q.to(DEV), *Kd, *Vd, kv_d, mask=mask_d, workspace=ws)
            mask_o = oracle.sink_mask(p, 1, sp_o)
            ref = oracle.sdpa(wl.u16(q), *Ko, *Vo, kv_len=kv_o, sm_scale=1 / math.sqrt(D), mask=mask_o)
            assert_attn_close(bf16_to_f64(out), ref, f"sink decode p={p}")


def test_kv_len_is_read_on_device_each_call():
    g = wl.generator(91)
    B, Hq, Hkv, D, S = 1, 4, 1, 128, 1024
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g).to(DEV)
    Kd = [t.to(DEV) for t in K]
    Vd = [t.to(DEV) for t in V]
    kv = int32_scalar(1)
    ws = kvq.decode_workspace(B, Hq, Hkv, D, S, DEV)
    for n in (1, 100, 1024, 513):
        kv.fill_(n)  # only device memory changes; the launch arguments do not
        out = kvq.decode_attn(q, *Kd, *Vd, kv, workspace=ws)
        ref = oracle.sdpa(wl.u16(q.cpu()), *_np(K), *_np(V), kv_len=n, sm_scale=1 / math.sqrt(D))
        assert_attn_close(bf16_to_f64(out), ref, f"kv_len {n}")


def test_kv_len_full_equals_bound_at_s_and_out_of_range_is_clamped():
    g = wl.generator(92)
    B, Hq, Hkv, D, S = 2, 8, 2, 64, 256
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    a = _decode_gpu(q, K, V, S)
    err = err_word()
    b = _decode_gpu(q, K, V, S + 50, err=err)
    assert torch.equal(a, b)
    assert err.item() & kvq.KVQ_ERR_KV_LEN_RANGE
    err2 = err_word()
    z = _decode_gpu(q, K, V, -5, err=err2)
    assert err2.item() & kvq.KVQ_ERR_KV_LEN_RANGE
    assert torch.all(z == 0)


def test_decode_is_deterministic():
    g = wl.generator(93)
    B, Hq, Hkv, D, S = 4, 16, 4, 128, 2048
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    a = _decode_gpu(q, K, V, 2000)
    b = _decode_gpu(q, K, V, 2000)
    assert torch.equal(a, b)


def test_decode_workspace_reused_across_shapes_keeps_counters_at_zero():
    """One caller workspace, zero-filled once, serves calls of changing D, q heads
    per kv head and batch in stream order.  Each call is checked against the
    oracle, and after each the merge counters (the first 1 KiB) are zero again."""
    seq = [(2, 4, 2, 256, 2048, 2048), (3, 8, 2, 64, 2048, 1999), (2, 16, 4, 128, 1024, 1024),
           (2, 12, 4, 128, 2048, 1537), (5, 4, 2, 64, 1024, 1000), (1, 8, 2, 256, 4096, 3000)]
    size = max(kvq.decode_workspace_bytes(B, Hq, Hkv, D, S) for B, Hq, Hkv, D, S, _ in seq)
    ws = torch.zeros(size, dtype=torch.uint8, device=DEV)
    for i, (B, Hq, Hkv, D, S, n) in enumerate(seq):
        g = wl.generator(5150 + i)
        K, V = _cache(B, Hkv, S, D, g)
        q = wl.bf16_normal((B, Hq, 1, D), g)
        out = kvq.decode_attn(q.to(DEV), *[t.to(DEV) for t in K], *[t.to(DEV) for t in V], int32_scalar(n),
                              workspace=ws)
        torch.cuda.synchronize()
        ref = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=n, sm_scale=1 / math.sqrt(D))
        assert_attn_close(bf16_to_f64(out), ref, f"reused workspace call {i}")
        assert torch.count_nonzero(ws[:1024]).item() == 0, f"merge counters left set after call {i}"


# ---------------------------------------------------------------------------- prefill

def _prefill_gpu(q, K, V, kv_len, **kw):
    Kd = [t.to(DEV) for t in K]
    Vd = [t.to(DEV) for t in V]
    if "mask" in kw and kw["mask"] is not None:
        kw["mask"] = kw["mask"].to(DEV)
    out = kvq.prefill_attn(q.to(DEV), *Kd, *Vd, int32_scalar(kv_len), **kw)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (4, 4), (6, 3)])
@pytest.mark.parametrize("Lq,kv_len", [(1, 50), (5, 50), (33, 160), (128, 128), (70, 300)])
def test_prefill_causal_shapes(D, Hq, Hkv, Lq, kv_len):
    g = wl.generator(D + Hq * 11 + Lq * 13 + kv_len)
    B, S = 2, 320
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = _prefill_gpu(q, K, V, kv_len, is_causal=True, mask_is_causal=True)
    ref = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=kv_len, sm_scale=1 / math.sqrt(D), is_causal=True)
    assert_attn_close(bf16_to_f64(out), ref, f"prefill D={D} G={Hq // Hkv} Lq={Lq} kv={kv_len}")


@pytest.mark.parametrize("D", [64, 128, 256])
def test_prefill_tile_skip_is_bit_identical(D):
    g = wl.generator(500 + D)
    B, Hq, Hkv, S, Lq, kv_len = 1, 8, 2, 640, 200, 600
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    a = _prefill_gpu(q, K, V, kv_len, is_causal=True, mask_is_causal=False)
    b = _prefill_gpu(q, K, V, kv_len, is_causal=True, mask_is_causal=True)
    assert torch.equal(a, b)
    # at Lq = 1 the bound is the whole kv_len: the causal and plain settings agree bit for bit
    q1 = wl.bf16_normal((B, Hq, 1, D), g)
    c = _prefill_gpu(q1, K, V, kv_len, is_causal=True, mask_is_causal=True)
    d = _prefill_gpu(q1, K, V, kv_len, is_causal=False, mask_is_causal=False)
    assert torch.equal(c, d)


def test_sink_config_prefill_chunks():
    """128-token chunks through the 4 + 2044 ring over positions 0 .. 10111 (79
    chunks), checked on the chunks that span positions 2048, 4096, 6144 and 8192,
    on an early one and on the last (masked attention, no causal flag)."""
    w = wl.SINK
    g = wl.generator(w.seed + 7)
    S, D, Lq = w.S, w.D, w.Lq
    K0 = wl.int8_cache_random(1, w.Hkv, S, D, g)
    V0 = wl.int8_cache_random(1, w.Hkv, S, D, g)
    Kd = [t.to(DEV) for t in K0]
    Vd = [t.to(DEV) for t in V0]
    Ko = [t.numpy().copy() for t in K0]
    Vo = [t.numpy().copy() for t in V0]
    sp_d = torch.full((S,), -1, dtype=torch.int32, device=DEV)
    sp_o = np.full(S, -1, np.int32)
    ip = torch.zeros(1, dtype=torch.int32, device=DEV)
    sm_d = torch.empty(Lq, dtype=torch.int32, device=DEV)
    kv_d = torch.empty(1, dtype=torch.int32, device=DEV)
    mask_d = torch.empty((Lq, S), dtype=torch.float32, device=DEV)
    for c in range(79):
        p = c * Lq
        k = wl.bf16_normal((1, w.Hkv, Lq, D), g)
        v = wl.bf16_normal((1, w.Hkv, Lq, D), g)
        ip.fill_(p)
        kvq.sink_plan(ip, 1, Lq, w.sink, sp_d, sm_d, kv_d)
        kvq.write(0, k.to(DEV), sm_d, *Kd)
        kvq.write(0, v.to(DEV), sm_d, *Vd)
        sm_o, kv_o = oracle.sink_plan(p, 1, Lq, w.sink, S, sp_o)
        oracle.write(0, wl.u16(k), sm_o, S, *Ko)
        oracle.write(0, wl.u16(v), sm_o, S, *Vo)
        if any(p <= x < p + Lq for x in (2048, 4096, 6144, 8192)) or c in (3, 78):
            q = wl.bf16_normal((1, w.Hq, Lq, D), g)
            kvq.sink_mask(ip, Lq, sp_d, mask_d)
            out = kvq.prefill_attn(q.to(DEV), *Kd, *Vd, kv_d, mask=mask_d)
            mask_o = oracle.sink_mask(p, Lq, sp_o)
            rows = [(0, h, i) for h in (0, 5, 31) for i in range(0, Lq, 9)] + [(0, 17, Lq - 1)]
            ref = oracle.sdpa_rows(wl.u16(q), *Ko, *Vo, kv_len=kv_o, sm_scale=1 / math.sqrt(D), rows=rows,
                                   mask=mask_o)
            got = bf16_to_f64(out)
            assert_attn_close(np.stack([got[b, h, i] for b, h, i in rows]), ref, f"sink prefill p={p}")


def test_long_config_prefill_sampled_rows():
    """Lq = 2048 causal chunk at kv_len 131072 (32 q / 16 kv heads, D=256),
    checked on the first and the last row of every 64-row block (a CTA takes 128
    rows = 2 q heads x 64 positions here, and the per-tile causal bound moves at
    each block edge; the 128-row tile edges are among them), across heads."""
    w = wl.LONG
    g = wl.generator(w.seed + 200)
    K, V = _cache(w.B, w.Hkv, w.S, w.D, g)
    q = wl.bf16_normal((w.B, w.Hq, w.Lq, w.D), g)
    out = _prefill_gpu(q, K, V, w.kv_len, is_causal=True, mask_is_causal=True)
    rows = [(0, (5 * t + e) % w.Hq, 64 * t + 63 * e) for t in range(w.Lq // 64) for e in (0, 1)]
    ref = oracle.sdpa_rows(wl.u16(q), *_np(K), *_np(V), kv_len=w.kv_len, sm_scale=1 / math.sqrt(w.D),
                           rows=rows, is_causal=True)
    got = bf16_to_f64(out)
    assert_attn_close(np.stack([got[b, h, i] for b, h, i in rows]), ref, "long prefill")


# ---------------------------------------------------------------------------- per-row kv_len

def _slice(c, b):
    return [t[b:b + 1] for t in c]


@pytest.mark.parametrize("D", [64, 128, 256])
def test_decode_varlen_rows_match_the_oracle_per_row(D):
    """Rows of one decode batch at different context lengths (0 .. 4000 of
    4096 slots): each row equals the oracle run at its own kv_len."""
    g = wl.generator(700 + D)
    B, Hq, Hkv, S = 6, 8, 2, 4096
    lens = [0, 1, 37, 352, 1000, 4000]
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    err = err_word()
    out = kvq.decode_attn_varlen(q.to(DEV), *[t.to(DEV) for t in K], *[t.to(DEV) for t in V],
                                 torch.tensor(lens, dtype=torch.int32, device=DEV), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = bf16_to_f64(out)
    for b in range(B):
        ref = oracle.sdpa(wl.u16(q[b:b + 1]), *_np(_slice(K, b)), *_np(_slice(V, b)), kv_len=lens[b],
                          sm_scale=1 / math.sqrt(D))
        assert_attn_close(got[b:b + 1], ref, f"varlen decode D={D} row {b} kv={lens[b]}")
    assert torch.all(out[0] == 0)


@pytest.mark.parametrize("D", [64, 128])
def test_decode_varlen_many_short_rows_with_empty_ones(D):
    """64 rows of 0..200 slots, a fifth of them empty: CTA ranges, flattened by
    each row's own length, span up to several rows (empty rows in between own
    no chunks and must still come out zero)."""
    g = wl.generator(760 + D)
    B, Hq, Hkv, S = 64, 8, 2, 256
    rng = torch.Generator().manual_seed(761 + D)
    lens = torch.randint(1, 201, (B,), generator=rng)
    lens[torch.randperm(B, generator=rng)[: B // 5]] = 0
    lens = lens.tolist()
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    err = err_word()
    out = kvq.decode_attn_varlen(q.to(DEV), *[t.to(DEV) for t in K], *[t.to(DEV) for t in V],
                                 torch.tensor(lens, dtype=torch.int32, device=DEV), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = bf16_to_f64(out)
    for b in range(B):
        if lens[b] == 0:
            assert torch.all(out[b] == 0), f"row {b} (kv 0) is not zero"
            continue
        ref = oracle.sdpa(wl.u16(q[b:b + 1]), *_np(_slice(K, b)), *_np(_slice(V, b)), kv_len=lens[b],
                          sm_scale=1 / math.sqrt(D))
        assert_attn_close(got[b:b + 1], ref, f"varlen decode D={D} row {b} kv={lens[b]}")


@pytest.mark.parametrize("D,lens", [
    (128, [512, 1024, 2048, 3072, 4096, 5120, 6144, 8192]),  # the ragged bench batch: 144 CTAs, 1-4 a unit
    (256, [100, 3000, 0, 7000, 64, 2500]),                     # D = 256, an empty row, a one-chunk row
])
def test_decode_varlen_row_aligned_split(D, lens):
    """A few rows of different lengths: each row's units get their own CTAs (more for
    longer rows), so no CTA spans two units; every row equals the oracle at its length."""
    g = wl.generator(790 + D + len(lens))
    B, Hkv, G = len(lens), 8 if D == 128 else 4, 4 if D == 128 else 2
    S = 8192
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hkv * G, 1, D), g)
    err = err_word()
    out = kvq.decode_attn_varlen(q.to(DEV), *[t.to(DEV) for t in K], *[t.to(DEV) for t in V],
                                 torch.tensor(lens, dtype=torch.int32, device=DEV), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = bf16_to_f64(out)
    for b in range(B):
        if lens[b] == 0:
            assert torch.all(out[b] == 0)
            continue
        ref = oracle.sdpa(wl.u16(q[b:b + 1]), *_np(_slice(K, b)), *_np(_slice(V, b)), kv_len=lens[b],
                          sm_scale=1 / math.sqrt(D))
        assert_attn_close(got[b:b + 1], ref, f"row-aligned varlen decode D={D} row {b} kv={lens[b]}")


def test_decode_varlen_equal_rows_is_the_scalar_path():
    g = wl.generator(777)
    B, Hq, Hkv, D, S = 4, 16, 4, 128, 2048
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    Kd = [t.to(DEV) for t in K]
    Vd = [t.to(DEV) for t in V]
    a = kvq.decode_attn(q.to(DEV), *Kd, *Vd, int32_scalar(1500))
    b = kvq.decode_attn_varlen(q.to(DEV), *Kd, *Vd, torch.full((B,), 1500, dtype=torch.int32, device=DEV))
    assert torch.equal(a, b)


def test_decode_varlen_out_of_range_rows_are_clamped_and_flagged():
    g = wl.generator(778)
    B, Hq, Hkv, D, S = 3, 4, 2, 64, 512
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    Kd = [t.to(DEV) for t in K]
    Vd = [t.to(DEV) for t in V]
    err = err_word()
    out = kvq.decode_attn_varlen(q.to(DEV), *Kd, *Vd, torch.tensor([-3, 9999, 100], dtype=torch.int32, device=DEV),
                                 err_word=err)
    torch.cuda.synchronize()
    assert err.item() & kvq.KVQ_ERR_KV_LEN_RANGE
    ref = kvq.decode_attn_varlen(q.to(DEV), *Kd, *Vd, torch.tensor([0, S, 100], dtype=torch.int32, device=DEV))
    assert torch.equal(out, ref)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_prefill_varlen_rows_match_the_oracle_per_row(D):
    g = wl.generator(800 + D)
    B, Hq, Hkv, S, Lq = 3, 4, 2, 320, 70
    lens = [70, 171, 320]
    K, V = _cache(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = kvq.prefill_attn_varlen(q.to(DEV), *[t.to(DEV) for t in K], *[t.to(DEV) for t in V],
                                  torch.tensor(lens, dtype=torch.int32, device=DEV), is_causal=True,
                                  mask_is_causal=True)
    torch.cuda.synchronize()
    got = bf16_to_f64(out)
    for b in range(B):
        ref = oracle.sdpa(wl.u16(q[b:b + 1]), *_np(_slice(K, b)), *_np(_slice(V, b)), kv_len=lens[b],
                          sm_scale=1 / math.sqrt(D), is_causal=True)
        assert_attn_close(got[b:b + 1], ref, f"varlen prefill D={D} row {b} kv={lens[b]}")


# ---------------------------------------------------------------------------- TQ4 cache

@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("Hq,Hkv,kv_len", [(4, 2, 40), (8, 2, 1000), (6, 3, 777), (32, 8, 4096)])
def test_tq4_decode_matches_the_oracle(D, Hq, Hkv, kv_len):
    g = wl.generator(900 + D + Hq + kv_len)
    B, S = 2, 4096
    K = wl.int4_cache_random(B, Hkv, S, D, g)
    V = wl.int4_cache_random(B, Hkv, S, D, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    err = err_word()
    out = kvq.decode_attn_tq4(q.to(DEV), *[t.to(DEV) for t in K], *[t.to(DEV) for t in V], int32_scalar(kv_len),
                              err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=kv_len, sm_scale=1 / math.sqrt(D))
    assert_attn_close(bf16_to_f64(out), ref, f"tq4 decode D={D} Hq={Hq} Hkv={Hkv} kv={kv_len}")


def test_tq4_decode_with_mask_and_written_cache():
    """Write K/V through kvq_write mode 7, then attend with an additive mask."""
    g = wl.generator(950)
    B, Hq, Hkv, D, S, T = 1, 8, 2, 128, 512, 300
    x_k = wl.bf16_normal((B, Hkv, T, D), g)
    x_v = wl.bf16_normal((B, Hkv, T, D), g)
    sm = torch.arange(T, dtype=torch.int32)
    K = [t.to(DEV) for t in wl.int4_cache_random(B, Hkv, S, D, g)]
    V = [t.to(DEV) for t in wl.int4_cache_random(B, Hkv, S, D, g)]
    kvq.write(7, x_k.to(DEV), sm.to(DEV), *K)
    kvq.write(7, x_v.to(DEV), sm.to(DEV), *V)
    mask = torch.zeros(S, dtype=torch.float32)
    mask[torch.randperm(T, generator=torch.Generator().manual_seed(3))[:90]] = -float("inf")
    q = wl.bf16_normal((B, Hq, 1, D), g)
    out = kvq.decode_attn_tq4(q.to(DEV), *K, *V, int32_scalar(T), mask=mask.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.sdpa(wl.u16(q), *[t.cpu().numpy() for t in K], *[t.cpu().numpy() for t in V], kv_len=T,
                      sm_scale=1 / math.sqrt(D), mask=mask.numpy()[None, :])
    assert_attn_close(bf16_to_f64(out), ref, "tq4 decode, written cache, masked")


# ---------------------------------------------------------------------------- block caches (modes 1-6)

def _block_cache_from_writer(mode, B, Hkv, S, D, kv, g, round_scale=True):
    """A block cache filled by kvq_write from bf16 N(0, 1) rows (1% x10 outliers):
    slots [0, kv) written, the rest left at zero codes."""
    x = wl.bf16_normal((B, Hkv, kv, D), g, outlier_p=0.01, outlier_scale=10.0)
    row = D // 2 if mode == 3 else D
    f32 = mode in (1, 4, 6)
    codes = torch.zeros((B, Hkv, S, row), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((B, Hkv, S, D // 32), dtype=torch.float32 if f32 else torch.uint8, device=DEV)
    sm = torch.arange(kv, dtype=torch.int32).repeat(B)
    kvq.write(mode, x.to(DEV), sm.to(DEV), codes, scales, round_scale=round_scale)
    return codes, scales


@pytest.mark.parametrize("mode", [1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_block_cache_decode_matches_the_oracle(mode, D):
    g = wl.generator(1100 + 10 * mode + D)
    B, Hq, Hkv, S, kv = 2, 8, 2, 1024, 777
    Kc, Ks = _block_cache_from_writer(mode, B, Hkv, S, D, kv, g)
    Vc, Vs = _block_cache_from_writer(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    err = err_word()
    out = kvq.decode_attn_block(mode, q.to(DEV), Kc, Ks, Vc, Vs, int32_scalar(kv), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.sdpa_block(mode, wl.u16(q), Kc.cpu().numpy(), Ks.cpu().numpy(), Vc.cpu().numpy(),
                            Vs.cpu().numpy(), kv_len=kv, sm_scale=1 / math.sqrt(D))
    assert_attn_close(bf16_to_f64(out), ref, f"block-cache decode mode {mode} D={D}")


@pytest.mark.parametrize("mode", [1, 3])
@pytest.mark.parametrize("Hq,Hkv,kv", [(4, 4, 1), (8, 1, 300), (32, 8, 4096)])
def test_block_cache_decode_shapes_and_mask(mode, Hq, Hkv, kv):
    g = wl.generator(1200 + mode + Hq + kv)
    B, D, S = 1, 128, 4096
    Kc, Ks = _block_cache_from_writer(mode, B, Hkv, S, D, kv, g)
    Vc, Vs = _block_cache_from_writer(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    mask = torch.zeros(S, dtype=torch.float32)
    mask[torch.randperm(kv, generator=torch.Generator().manual_seed(kv))[: kv // 3]] = -float("inf")
    mask[0] = 0.0
    out = kvq.decode_attn_block(mode, q.to(DEV), Kc, Ks, Vc, Vs, int32_scalar(kv), mask=mask.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.sdpa_block(mode, wl.u16(q), Kc.cpu().numpy(), Ks.cpu().numpy(), Vc.cpu().numpy(),
                            Vs.cpu().numpy(), kv_len=kv, sm_scale=1 / math.sqrt(D), mask=mask.numpy()[None, :])
    assert_attn_close(bf16_to_f64(out), ref, f"block-cache decode mode {mode} Hq={Hq} Hkv={Hkv} kv={kv}")


def test_block_cache_decode_empty_and_out_of_range():
    g = wl.generator(1300)
    B, Hq, Hkv, D, S = 1, 4, 2, 64, 512
    Kc, Ks = _block_cache_from_writer(1, B, Hkv, S, D, 100, g)
    Vc, Vs = _block_cache_from_writer(1, B, Hkv, S, D, 100, g)
    q = wl.bf16_normal((B, Hq, 1, D), g).to(DEV)
    z = kvq.decode_attn_block(1, q, Kc, Ks, Vc, Vs, int32_scalar(0))
    assert torch.all(z == 0)
    err = err_word()
    a = kvq.decode_attn_block(1, q, Kc, Ks, Vc, Vs, int32_scalar(99999), err_word=err)
    b = kvq.decode_attn_block(1, q, Kc, Ks, Vc, Vs, int32_scalar(S))
    torch.cuda.synchronize()
    assert err.item() & kvq.KVQ_ERR_KV_LEN_RANGE and torch.equal(a, b)


@pytest.mark.parametrize("mode", [1, 3])
@pytest.mark.parametrize("D", [64, 256])
def test_block_cache_decode_several_tiles_per_warp(mode, D):
    """64 (b, kv head) units split about 5 ways give every warp two or three
    32-slot tiles: the staged-tile ring (two buffers at D 64, one at D 256) is
    reused within a split."""
    g = wl.generator(1400 + mode + D)
    B, Hq, Hkv, S, kv = 8, 32, 8, 4096, 3000
    Kc, Ks = _block_cache_from_writer(mode, B, Hkv, S, D, kv, g)
    Vc, Vs = _block_cache_from_writer(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, 1, D), g)
    out = kvq.decode_attn_block(mode, q.to(DEV), Kc, Ks, Vc, Vs, int32_scalar(kv))
    torch.cuda.synchronize()
    ref = oracle.sdpa_block(mode, wl.u16(q), Kc.cpu().numpy(), Ks.cpu().numpy(), Vc.cpu().numpy(),
                            Vs.cpu().numpy(), kv_len=kv, sm_scale=1 / math.sqrt(D))
    assert_attn_close(bf16_to_f64(out), ref, f"block-cache decode mode {mode} D={D}, several tiles per warp")
