"""GPU parity of kvq_prefill_attn_block (chunked-prefill attention over the per-32
block caches of kvq_write modes 1-6) against the fp64 oracle: the cache is
dequantized by the oracle's own codecs (IndexerQuantCache, 计算公式) and attended
in fp64; |gpu - oracle| <= 2e-3 + 1e-2 |oracle| element by element."""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_20_b200 import kvq
from quantized_kv_cache_20_b200 import workloads as wl
from tests.helpers import DEV, assert_attn_close, bf16_to_f64, err_word, int32_scalar

pytestmark = pytest.mark.gpu

F32_MODES = (1, 4, 6)


def _written_cache(mode, B, Hkv, S, D, kv, g):
    """A block cache filled by kvq_write from bf16 N(0, 1) rows with 1% x10
    outliers: slots [0, kv) written, the rest zero codes and zero scales."""
    x = wl.bf16_normal((B, Hkv, kv, D), g, outlier_p=0.01, outlier_scale=10.0)
    row = D // 2 if mode == 3 else D
    codes = torch.zeros((B, Hkv, S, row), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((B, Hkv, S, D // 32), dtype=torch.float32 if mode in F32_MODES else torch.uint8,
                         device=DEV)
    kvq.write(mode, x.to(DEV), torch.arange(kv, dtype=torch.int32).repeat(B).to(DEV), codes, scales)
    return codes, scales


def _run(mode, q, K, V, kv, **kw):
    out = kvq.prefill_attn_block(mode, q.to(DEV), *K, *V, int32_scalar(kv) if isinstance(kv, int) else kv, **kw)
    torch.cuda.synchronize()
    return out


def _ref(mode, q, K, V, kv, **kw):
    Kc, Ks = (t.cpu().numpy() for t in K)
    Vc, Vs = (t.cpu().numpy() for t in V)
    return oracle.sdpa_block(mode, wl.u16(q), Kc, Ks, Vc, Vs, kv_len=kv, sm_scale=1 / math.sqrt(q.shape[-1]),
                             **kw)


@pytest.mark.parametrize("mode", [1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_block_prefill_causal_matches_the_oracle(mode, D):
    """Two CTAs of query rows (the second ragged) over four 128-slot tiles (the
    last ragged), causal with the per-tile bound."""
    g = wl.generator(2000 + 10 * mode + D)
    B, Hq, Hkv, S, Lq, kv = 1, 4, 2, 512, 150, 420
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    err = err_word()
    out = _run(mode, q, K, V, kv, is_causal=True, mask_is_causal=True, err_word=err)
    assert err.item() == 0
    ref = _ref(mode, q, K, V, kv, is_causal=True)
    assert_attn_close(bf16_to_f64(out), ref, f"block prefill mode {mode} D={D}")


@pytest.mark.parametrize("mode", [1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("Hq,Hkv,Lq,kv", [(8, 1, 33, 200), (6, 2, 5, 50), (4, 4, 128, 128), (16, 2, 64, 700)])
def test_block_prefill_gqa_shapes(mode, Hq, Hkv, Lq, kv):
    """Four, two and one q heads per CTA (the GQA head chunks), a single row,
    a chunk equal to the cache length."""
    g = wl.generator(2100 + 7 * mode + Hq + Lq + kv)
    B, D, S = 2, 128, 768
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = _run(mode, q, K, V, kv, is_causal=True, mask_is_causal=True)
    ref = _ref(mode, q, K, V, kv, is_causal=True)
    assert_attn_close(bf16_to_f64(out), ref, f"block prefill mode {mode} Hq={Hq} Hkv={Hkv} Lq={Lq} kv={kv}")


@pytest.mark.parametrize("mode", [2, 3, 6])
def test_block_prefill_with_additive_mask(mode):
    """A sink/ring-style additive mask (no causal flag): random -inf holes, slot 0
    always visible."""
    g = wl.generator(2200 + mode)
    B, Hq, Hkv, D, S, Lq, kv = 1, 8, 2, 64, 384, 100, 384
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    mask = torch.zeros((Lq, S), dtype=torch.float32)
    hide = torch.rand((Lq, S), generator=g) < 0.3
    mask[hide] = -float("inf")
    mask[:, 0] = 0.0
    mask[:, 5] = -1.5  # a finite additive term
    out = _run(mode, q, K, V, kv, mask=mask.to(DEV))
    ref = _ref(mode, q, K, V, kv, mask=mask.numpy())
    assert_attn_close(bf16_to_f64(out), ref, f"block prefill mode {mode} masked")


def _spread_scales(mode, cache, lo, hi, g):
    """Multiply each group scale by 2^k, k uniform in [lo, hi], and zero 5% of
    the groups (E8M0: shift the exponent byte, code 0 for the zeroed groups)."""
    _, s = cache
    shift = torch.randint(lo, hi + 1, s.shape, generator=g)
    zero = torch.rand(s.shape, generator=g) < 0.05
    if mode in F32_MODES:
        f = torch.pow(2.0, shift.float())
        f[zero] = 0.0
        s.mul_(f.to(DEV))
    else:
        e = (s.cpu().to(torch.int32) + shift).clamp_(1, 254)
        e[zero] = 0
        s.copy_(e.to(torch.uint8).to(DEV))


@pytest.mark.parametrize("mode", [1, 2, 3, 4, 5, 6])
def test_block_prefill_wide_scale_spread_within_a_slot(mode):
    """Group scales of one slot that differ by up to 2^24 (and all-zero groups):
    the per-slot power of two factored out by the converters must keep the
    largest groups exact and lose only what lies below fp16's range."""
    g = wl.generator(2300 + mode)
    B, Hq, Hkv, D, S, Lq, kv = 1, 4, 2, 256, 256, 64, 256
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    _spread_scales(mode, K, -24, 0, g)
    _spread_scales(mode, V, -24, 0, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = _run(mode, q, K, V, kv, is_causal=True, mask_is_causal=True)
    ref = _ref(mode, q, K, V, kv, is_causal=True)
    assert_attn_close(bf16_to_f64(out), ref, f"block prefill mode {mode}, wide scale spread")


@pytest.mark.parametrize("mode", [2, 3, 5])
def test_block_prefill_e8m0_large_scores_stay_exact(mode):
    """K groups scaled up by as much as 2^8 drive the scores into the hundreds:
    with E8M0 scales K reaches the tensor cores exactly and the scores are fp32
    sums of exact products, so the strict tolerance holds however peaked the
    softmax becomes.  (V keeps O(1) values: P is rounded to fp16, which costs up
    to 2^-11 sum_j p_j |V_jd| whatever the cache format.)"""
    g = wl.generator(2350 + mode)
    B, Hq, Hkv, D, S, Lq, kv = 1, 4, 2, 256, 256, 64, 256
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    _spread_scales(mode, K, -4, 8, g)
    _spread_scales(mode, V, -4, 0, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = _run(mode, q, K, V, kv, is_causal=True, mask_is_causal=True)
    ref = _ref(mode, q, K, V, kv, is_causal=True)
    assert_attn_close(bf16_to_f64(out), ref, f"block prefill mode {mode}, large scores")


@pytest.mark.parametrize("mode", F32_MODES)
def test_block_prefill_float_scales_large_scores_within_the_rounding_bound(mode):
    """With float group scales each K and V element is rounded to fp16 once
    (unit roundoff u = 2^-11) and, below fp16's normal range, by at most 2^-25
    times its slot's power of two 2^E.  A score s_j then moves by at most
    d_i = sm_scale * max_j sum_d |q_d| (u |K_jd| + 2^-25 2^E_j), each softmax
    weight by a factor within e^(+-2 d_i), and the output by at most
    (e^(2 d_i) - 1) max_j |V_jd - out_d| + 2u max_j |V_jd| beyond the strict
    tolerance (the second term: the V rounding and the fp16 rounding of P).
    Scores in the hundreds (groups scaled up by 2^8) exercise it."""
    g = wl.generator(2380 + mode)
    B, Hq, Hkv, D, S, Lq, kv = 1, 4, 2, 256, 256, 64, 256
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    _spread_scales(mode, K, -4, 8, g)
    _spread_scales(mode, V, -4, 8, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = bf16_to_f64(_run(mode, q, K, V, kv, is_causal=True, mask_is_causal=True))
    ref = _ref(mode, q, K, V, kv, is_causal=True)
    Kf = oracle.dequant_block(mode, K[0].cpu().numpy(), K[1].cpu().numpy())[0]  # [Hkv, S, D]
    Vf = oracle.dequant_block(mode, V[0].cpu().numpy(), V[1].cpu().numpy())[0]
    ks = K[1].cpu().numpy()[0].astype(np.float64)  # [Hkv, S, D/32]
    smax = ks.max(axis=-1)
    E = np.where(smax > 0, np.ceil(np.log2(np.where(smax > 0, smax, 1.0))), 0.0)  # [Hkv, S]
    u = 2.0 ** -11
    qf = q.to(torch.float64).numpy()[0]  # [Hq, Lq, D], exact
    G = Hq // Hkv
    sm = 1 / math.sqrt(D)
    for h in range(Hq):
        hk = h // G
        elem = u * np.abs(Kf[hk, :kv]) + 2.0 ** -25 * np.exp2(E[hk, :kv])[:, None]  # [kv, D]
        d = sm * (np.abs(qf[h]) @ elem.T).max(axis=1)  # [Lq]
        spread = np.abs(Vf[hk, :kv][None, :, :] - ref[0, h][:, None, :]).max(axis=1)  # [Lq, D]
        extra = np.expm1(2 * d)[:, None] * spread + 2 * u * np.abs(Vf[hk, :kv]).max(axis=0)[None, :]
        err = np.abs(out[0, h] - ref[0, h])
        bound = 2e-3 + 1e-2 * np.abs(ref[0, h]) + extra
        assert (err <= bound).all(), f"mode {mode} head {h}: worst excess {(err - bound).max()}"


@pytest.mark.parametrize("mode", [1, 3])
def test_block_prefill_tile_skip_is_bit_identical(mode):
    g = wl.generator(2400 + mode)
    B, Hq, Hkv, D, S, Lq, kv = 1, 8, 2, 128, 640, 200, 600
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    a = _run(mode, q, K, V, kv, is_causal=True, mask_is_causal=False)
    b = _run(mode, q, K, V, kv, is_causal=True, mask_is_causal=True)
    assert torch.equal(a, b)


def test_block_prefill_kv_len_out_of_range_is_clamped_and_flagged():
    g = wl.generator(2500)
    B, Hq, Hkv, D, S, Lq = 1, 4, 2, 64, 256, 16
    K = _written_cache(2, B, Hkv, S, D, S, g)
    V = _written_cache(2, B, Hkv, S, D, S, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    err = err_word()
    a = _run(2, q, K, V, 99999, is_causal=True, err_word=err)
    b = _run(2, q, K, V, S, is_causal=True)
    assert err.item() & kvq.KVQ_ERR_KV_LEN_RANGE and torch.equal(a, b)


@pytest.mark.parametrize("mode", [2, 3])
def test_block_prefill_long_chunk_sampled_rows(mode):
    """A 1024-row causal chunk at the end of 16384 filled slots (16 q / 2 kv
    heads, D = 256): the first and the last row of every 64-row block, across
    heads, against the oracle one row at a time."""
    g = wl.generator(2600 + mode)
    B, Hq, Hkv, D, S, Lq = 1, 16, 2, 256, 16384, 1024
    kv = S
    K = _written_cache(mode, B, Hkv, S, D, kv, g)
    V = _written_cache(mode, B, Hkv, S, D, kv, g)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = _run(mode, q, K, V, kv, is_causal=True, mask_is_causal=True)
    rows = [(0, (5 * t + e) % Hq, 64 * t + 63 * e) for t in range(Lq // 64) for e in (0, 1)]
    Kf = oracle.dequant_block(mode, K[0].cpu().numpy(), K[1].cpu().numpy())
    Vf = oracle.dequant_block(mode, V[0].cpu().numpy(), V[1].cpu().numpy())
    ref = oracle.sdpa_dense_rows(wl.u16(q), Kf, Vf, kv, 1 / math.sqrt(D), rows, is_causal=True)
    got = bf16_to_f64(out)
    assert_attn_close(np.stack([got[b, h, i] for b, h, i in rows]), ref, f"long block prefill mode {mode}")


def test_block_prefill_rejects_bad_arguments():
    g = wl.generator(2700)
    K = _written_cache(1, 1, 1, 64, 64, 16, g)
    V = _written_cache(1, 1, 1, 64, 64, 16, g)
    q = wl.bf16_normal((1, 1, 4, 64), g).to(DEV)
    lib = kvq.load()
    out = torch.empty_like(q)
    kv = int32_scalar(16)
    args = (q.data_ptr(), 1, 1, 1, 4, 64, K[0].data_ptr(), K[1].data_ptr(), V[0].data_ptr(), V[1].data_ptr(), 64,
            kv.data_ptr(), None, 1, 1, 0.125, out.data_ptr(), None, None)
    assert lib.kvq_prefill_attn_block(1, *args) == kvq.KVQ_OK
    assert lib.kvq_prefill_attn_block(0, *args) == kvq.KVQ_EINVAL  # int8 affine has its own entry point
    assert lib.kvq_prefill_attn_block(7, *args) == kvq.KVQ_EINVAL
    bad_d = list(args)
    bad_d[5] = 96
    assert lib.kvq_prefill_attn_block(1, *bad_d) == kvq.KVQ_EUNSUPPORTED
    torch.cuda.synchronize()
