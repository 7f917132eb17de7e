"""Pins for the oracle's fp64 attention over the int8 cache (CPU only).

abaddon src/attention_cache/mod.rs, trait KvCache (forward_attention shapes,
GQA through repeat_kv, scale typically 1/sqrt(head_dim)); ExecuTorch PR 20351
commit notes (kv_len bounds the loop; causal row i sees kv_len - Lq + i; at
Lq = 1 the causal bound is the whole kv_len); ExecuTorch PR 24473, Summary
(additive float mask).  Checked against torch's scaled_dot_product_attention
in float64 (an independent library routine), closed forms and invariances.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from quantized_kv_cache_20_b200 import workloads as wl


def _case(seed, B=2, Hq=4, Hkv=2, Lq=3, D=16, S=24):
    g = wl.generator(seed)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    k, ks, kz = wl.int8_cache_like(B, Hkv, S, D, g)
    v, vs, vz = wl.int8_cache_like(B, Hkv, S, D, g)
    return q, (k, ks, kz), (v, vs, vz)


def _np(c):
    return [t.numpy() for t in c]


def _torch_ref(q, K, V, kv_len, sm_scale, mask=None, is_causal=False):
    k, ks, kz = K
    v, vs, vz = V
    kd = (k.double() - kz.double()[..., None]) * ks.double()[..., None]
    vd = (v.double() - vz.double()[..., None]) * vs.double()[..., None]
    kd, vd = kd[:, :, :kv_len], vd[:, :, :kv_len]
    G = q.shape[1] // k.shape[1]
    kd = kd.repeat_interleave(G, dim=1)      # contiguous GQA groups (repeat_kv)
    vd = vd.repeat_interleave(G, dim=1)
    Lq = q.shape[2]
    bias = torch.zeros(Lq, kv_len, dtype=torch.float64)
    if mask is not None:
        bias = bias + torch.from_numpy(mask[:, :kv_len]).double()
    if is_causal:
        i = torch.arange(Lq)[:, None]
        j = torch.arange(kv_len)[None, :]
        bias = bias.masked_fill(j > kv_len - Lq + i, -math.inf)
    # the oracle takes sm_scale as binary32, as the C ABI does
    sm_scale = float(np.float32(sm_scale))
    return F.scaled_dot_product_attention(q.double(), kd, vd, attn_mask=bias, scale=sm_scale).numpy()


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (4, 4), (8, 1)])
@pytest.mark.parametrize("is_causal", [False, True])
def test_matches_torch_sdpa_fp64(Hq, Hkv, is_causal):
    q, K, V = _case(1, Hq=Hq, Hkv=Hkv)
    kv_len, sm = 19, 1 / math.sqrt(16)
    ours = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=kv_len, sm_scale=sm, is_causal=is_causal)
    ref = _torch_ref(q, K, V, kv_len, sm, is_causal=is_causal)
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-12)


def test_matches_torch_with_additive_mask():
    q, K, V = _case(2, Lq=2)
    rng = np.random.default_rng(3)
    mask = np.where(rng.random((2, 24)) < 0.3, -np.inf, rng.normal(size=(2, 24))).astype(np.float32)
    mask[:, 0] = 0.0
    ours = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=24, sm_scale=0.3, mask=mask)
    ref = _torch_ref(q, K, V, 24, 0.3, mask=mask)
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-12)


def test_uniform_keys_give_mean_of_values():
    q, K, V = _case(3, B=1, Lq=1)
    k, ks, kz = K
    k[:] = k[:, :, :1]
    ks[:] = ks[:, :, :1]
    kz[:] = kz[:, :, :1]
    kv_len = 11
    out = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=kv_len, sm_scale=0.25)
    vd = oracle.dequant_int8(*_np(V))[:, :, :kv_len].mean(axis=2)     # [B, Hkv, D]
    G = q.shape[1] // k.shape[1]
    for h in range(q.shape[1]):
        np.testing.assert_allclose(out[0, h, 0], vd[0, h // G], rtol=1e-12, atol=1e-12)


def test_single_visible_slot_returns_its_value():
    q, K, V = _case(4, B=1, Lq=1)
    mask = np.full((1, 24), -np.inf, np.float32)
    mask[0, 7] = 0.0
    out = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=20, sm_scale=0.25, mask=mask)
    vd = oracle.dequant_int8(*_np(V))
    for h in range(4):
        np.testing.assert_allclose(out[0, h, 0], vd[0, h // 2, 7], rtol=0, atol=1e-12)


def test_causal_at_lq1_equals_unbounded_and_kv_len_truncates():
    q, K, V = _case(5, Lq=1)
    a = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=17, sm_scale=0.2, is_causal=True)
    b = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=17, sm_scale=0.2)
    assert np.array_equal(a, b)
    # kv_len = n over a cache equals attention over a cache that only has n slots
    K17 = [t[:, :, :17].contiguous() for t in K]
    V17 = [t[:, :, :17].contiguous() for t in V]
    c = oracle.sdpa(wl.u16(q), *_np(K17), *_np(V17), kv_len=17, sm_scale=0.2)
    assert np.array_equal(b, c)


def test_constant_mask_shift_changes_nothing_and_empty_row_is_zero():
    q, K, V = _case(6, Lq=2)
    m0 = np.zeros((2, 24), np.float32)
    a = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=24, sm_scale=0.2, mask=m0)
    b = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=24, sm_scale=0.2, mask=m0 + 3.5)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    m1 = np.full((2, 24), -np.inf, np.float32)
    z = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=24, sm_scale=0.2, mask=m1)
    assert np.all(z == 0)


def test_rows_helper_matches_full():
    q, K, V = _case(7, Lq=3)
    full = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=21, sm_scale=0.2, is_causal=True)
    rows = [(0, 0, 0), (1, 3, 2), (0, 2, 1)]
    part = oracle.sdpa_rows(wl.u16(q), *_np(K), *_np(V), kv_len=21, sm_scale=0.2, rows=rows,
                            is_causal=True)
    for n, (b, h, i) in enumerate(rows):
        assert np.array_equal(part[n], full[b, h, i])


def _unpack4(packed):
    t = torch.from_numpy(packed.astype(np.int64))
    return torch.stack([t & 15, t >> 4], dim=-1).reshape(*t.shape[:-1], -1)


@pytest.mark.parametrize("is_causal", [False, True])
def test_tq4_cache_matches_torch_sdpa_fp64(is_causal):
    # the TQ4 (nibble-packed) cache: unpacked here independently of the oracle
    g = wl.generator(61)
    B, Hq, Hkv, Lq, D, S = 2, 4, 2, 3, 16, 24
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    K = wl.int4_cache_random(B, Hkv, S, D, g)
    V = wl.int4_cache_random(B, Hkv, S, D, g)
    kv_len, sm = 19, 1 / math.sqrt(D)
    ours = oracle.sdpa(wl.u16(q), *_np(K), *_np(V), kv_len=kv_len, sm_scale=sm, is_causal=is_causal)
    Ku = (_unpack4(K[0].numpy()), K[1], K[2])
    Vu = (_unpack4(V[0].numpy()), V[1], V[2])
    ref = _torch_ref(q, Ku, Vu, kv_len, sm, is_causal=is_causal)
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------- block caches

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP MX FP4 E2M1 magnitudes


def _dequant_independent(mode, codes, scales):
    """Block-cache values computed here with torch's float8 decoders (modes 1, 2, 4, 5),
    the OCP E2M1 magnitudes (mode 3), int8 (mode 6) and 2^(e-127) for E8M0."""
    c = torch.from_numpy(np.ascontiguousarray(codes))
    if mode == 3:
        lo, hi = (c & 15).long(), (c >> 4).long()
        nib = torch.stack([lo, hi], dim=-1).reshape(*c.shape[:-1], -1)
        mag = torch.tensor(E2M1_VALUES, dtype=torch.float64)[nib & 7]
        val = torch.where(nib >= 8, -mag, mag)
    elif mode in (1, 2):
        val = c.view(torch.float8_e4m3fn).double()
    elif mode in (4, 5):
        val = c.view(torch.float8_e5m2).double()
    else:
        val = c.view(torch.int8).double()
    sc = torch.from_numpy(np.ascontiguousarray(scales))
    sc = sc.double() if mode in (1, 4, 6) else torch.exp2(sc.double() - 127)
    return (val.reshape(*val.shape[:-1], -1, 32) * sc[..., None]).reshape(val.shape).numpy()


@pytest.mark.parametrize("mode", [1, 2, 3, 4, 5, 6])
def test_block_dequant_matches_independent_decode(mode):
    g = wl.generator(70 + mode)
    codes, scales = wl.block_cache_random(2, 3, 5, 64, mode, g)
    ours = oracle.dequant_block(mode, codes.numpy(), scales.numpy())
    ref = _dequant_independent(mode, codes.numpy(), scales.numpy())
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(ours))          # NaN codes stay NaN
    assert np.array_equal(ours[fin], ref[fin])


@pytest.mark.parametrize("mode", [1, 2, 3, 4, 5, 6])
def test_block_dequant_inverts_the_quantizer_within_its_bound(mode):
    g = wl.generator(80 + mode)
    x = wl.bf16_normal((16, 128), g, outlier_p=0.02, outlier_scale=10.0)
    for r in range(x.shape[0]):
        codes, scales = oracle.block_row(mode, wl.u16(x[r]))
        deq = oracle.dequant_block(mode, codes[None], scales[None])[0]
        xv = x[r].double().numpy()
        amax = np.abs(xv.reshape(-1, 32)).max(axis=1).repeat(32)
        # relative half-steps: E4M3 2^-4, E5M2 2^-3, E2M1 up to 1/6 of amax... bound by a step of the grid
        step = {1: 2.0 ** -3, 2: 2.0 ** -3, 4: 2.0 ** -2, 5: 2.0 ** -2, 3: 1.0 / 3, 6: 1.0 / 127}[mode]
        assert np.all(np.abs(deq - xv) <= step * amax + 1e-30), (mode, r)


def test_dense_sdpa_matches_torch_fp64():
    g = torch.Generator().manual_seed(91)
    B, Hq, Hkv, Lq, D, S = 2, 6, 3, 3, 16, 24
    q = wl.bf16_normal((B, Hq, Lq, D), wl.generator(92))
    K = torch.randn((B, Hkv, S, D), generator=g, dtype=torch.float64)
    V = torch.randn((B, Hkv, S, D), generator=g, dtype=torch.float64)
    kv_len, sm = 21, 0.3
    for is_causal in (False, True):
        ours = oracle.sdpa_dense(wl.u16(q), K.numpy(), V.numpy(), kv_len, sm, is_causal=is_causal)
        G = Hq // Hkv
        kd, vd = K[:, :, :kv_len].repeat_interleave(G, 1), V[:, :, :kv_len].repeat_interleave(G, 1)
        bias = torch.zeros(Lq, kv_len, dtype=torch.float64)
        if is_causal:
            i, j = torch.arange(Lq)[:, None], torch.arange(kv_len)[None, :]
            bias = bias.masked_fill(j > kv_len - Lq + i, -math.inf)
        ref = F.scaled_dot_product_attention(q.double(), kd, vd, attn_mask=bias, scale=float(np.float32(sm)))
        np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-12, atol=1e-12)
