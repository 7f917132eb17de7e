"""GPU parity of kvq_write against the oracle: codes, scales, zero points and
every untouched byte must match exactly (bit-exact integer/byte work)."""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_20_b200 import kvq
from quantized_kv_cache_20_b200 import workloads as wl
from tests.helpers import DEV, err_word

pytestmark = pytest.mark.gpu


def _prefill(mode, B, H, S, D, g):
    if mode == 0:
        c, s, z = wl.int8_cache_random(B, H, S, D, g)
        return [c, s, z]
    if mode == 7:
        c, s, z = wl.int4_cache_random(B, H, S, D, g)
        return [c, s, z]
    c, s = wl.block_cache_random(B, H, S, D, mode, g)
    return [c, s, None]


def _run_both(mode, x, sm, cache0, S, round_scale=1):
    """Write x on the GPU and in the oracle over identical pre-filled caches."""
    gpu = [None if c is None else c.to(DEV) for c in cache0]
    err = err_word()
    kvq.write(mode, x.to(DEV) if not x.is_cuda else x, sm.to(DEV), gpu[0], gpu[1], gpu[2], err_word=err,
              round_scale=round_scale)
    torch.cuda.synchronize()
    ref = [None if c is None else c.numpy().copy() for c in cache0]
    xc = x.cpu()
    oerr = oracle.write(mode, wl.u16(xc), sm.numpy(), S, ref[0], ref[1], ref[2], round_scale=round_scale)
    return [None if c is None else c.cpu().numpy() for c in gpu], ref, int(err.item()), oerr


def _assert_equal(gpu, ref, what):
    for name, a, b in zip(("codes", "scales", "zero_points"), gpu, ref):
        if a is None:
            continue
        if a.dtype == np.float32:
            a, b = a.view(np.uint32), b.view(np.uint32)   # bit patterns
        bad = np.argwhere(a != b)
        assert bad.size == 0, f"{what} {name}: {len(bad)} mismatches, first at {bad[:3].tolist()}"


def test_tiny_int8_write():
    w = wl.TINY
    g = wl.generator(w.seed)
    k = wl.bf16_normal((w.B, w.Hkv, w.T, w.D), g)
    sm = wl.slot_mapping_random(w.T, w.S, 3, g)
    cache0 = _prefill(0, w.B, w.Hkv, w.S, w.D, g)
    gpu, ref, err, oerr = _run_both(0, k, sm, cache0, w.S)
    assert err == 0 and oerr == 0
    _assert_equal(gpu, ref, "tiny")


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 37), (2, 8, 129)])
def test_int8_ragged_shapes_and_strides(D, shape):
    B, H, T = shape
    S = 160
    g = wl.generator(1000 + D + T)
    # K/V as a strided view of a [B, T, H, D] projection output
    x = wl.bf16_normal((B, T, H, D), g, outlier_p=0.02, outlier_scale=20.0).permute(0, 2, 1, 3)
    sm = torch.stack([wl.slot_mapping_random(T, S, T // 5, g) for _ in range(B)]).reshape(-1)
    cache0 = _prefill(0, B, H, S, D, g)
    xd = x.to(DEV)  # keeps the permuted strides
    assert xd.stride(3) == 1
    gpu, ref, err, oerr = _run_both(0, xd, sm, cache0, S)
    assert err == 0
    _assert_equal(gpu, ref, f"int8 D={D} {shape}")


def _special_rows(d, g):
    rows = []
    rows.append(torch.zeros(d))                                   # all zero
    r = torch.zeros(d); r[::3] = -0.0; rows.append(r)             # signed zeros
    rows.append(torch.full((d,), 3.0))                            # constant
    rows.append(wl.bf16_normal((d,), g).float() * 1e-20)          # tiny
    rows.append(wl.bf16_normal((d,), g).float() * 1e30)           # huge
    rows.append(-wl.bf16_normal((d,), g).float().abs())           # non-positive
    # exact E4M3 / E2M1 midpoints at scale 1 (amax 448 or 6 -> scale 1)
    e4 = torch.arange(0, 0x7E, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    mids = (e4[:-1] + e4[1:]) / 2
    r = torch.cat([mids, -mids]); r = r[: d - 1]; r = torch.cat([torch.tensor([448.0]), r])
    rows.append(torch.nn.functional.pad(r, (0, d - r.numel())))
    fp4 = torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0,
                        5.5, 0.1, 0.3, 0.8, 2.2, 2.9, 4.9, -6.0, 7.0, 100.0, -100.0, 0.0, -0.0, 1.0, 3.0, 4.0,
                        -0.5])
    rows.append(fp4.repeat(d // 32))
    # exact E5M2 midpoints at scale 1 (amax 57344)
    e5 = torch.arange(0, 0x7C, dtype=torch.uint8).view(torch.float8_e5m2).float()
    mids5 = (e5[:-1] + e5[1:]) / 2
    r = torch.cat([torch.tensor([57344.0]), mids5, -mids5])[:d]
    rows.append(torch.nn.functional.pad(r, (0, d - r.numel())))
    # exact int8 half-integers at scale 1 (amax 127)
    halves = torch.arange(-126, 127, dtype=torch.float32) + 0.5
    r = torch.cat([torch.tensor([127.0, -127.0]), halves])[:d]
    rows.append(torch.nn.functional.pad(r, (0, d - r.numel())))
    return torch.stack([r.to(torch.bfloat16) for r in rows])


# (mode, round_scale): the IndexerQuantCache quant modes and cache types built;
# round_scale (1 ceil, 0 floor, 2 the OCP MX rule) matters for the E8M0 modes 2, 3, 5
BLOCK_CASES = [(1, 1), (2, 1), (3, 1), (4, 1), (5, 1), (6, 1), (2, 0), (5, 0), (3, 0), (2, 2), (3, 2), (5, 2)]


@pytest.mark.parametrize("mode,round_scale", BLOCK_CASES)
@pytest.mark.parametrize("d", [32, 96, 512, 8192])
def test_block_modes_small(mode, round_scale, d):
    g = wl.generator(2000 + mode * 10 + d + (0 if round_scale == 1 else 7 + round_scale))
    bs = 300 if d <= 512 else 24
    S = 2 * bs
    x = wl.bf16_normal((bs, d), g, outlier_p=0.01, outlier_scale=10.0)
    sp = _special_rows(d, g)
    x[: sp.shape[0]] = sp
    sm = wl.slot_mapping_random(bs, S, bs // 10, g)
    cache0 = _prefill(mode, 1, 1, S, d, g)
    gpu, ref, err, oerr = _run_both(mode, x.view(1, 1, bs, d), sm, cache0, S, round_scale)
    assert err == 0
    _assert_equal(gpu, ref, f"mode {mode} round_scale={round_scale} d={d}")


@pytest.mark.parametrize("mode,round_scale", BLOCK_CASES)
def test_block_config_full_size(mode, round_scale):
    """x [16384, 512] (1% x10 outliers) into 65536 slots, 10% skipped."""
    w = wl.BLOCK
    g = wl.generator(w.seed)
    x = wl.bf16_normal((w.tokens, w.d), g, outlier_p=w.outlier_p, outlier_scale=w.outlier_scale)
    sm = wl.slot_mapping_random(w.tokens, w.num_slots, int(w.tokens * w.skip_frac), g)
    cache0 = _prefill(mode, 1, 1, w.num_slots, w.d, g)
    gpu, ref, err, oerr = _run_both(mode, x.view(1, 1, w.tokens, w.d), sm, cache0, w.num_slots, round_scale)
    assert err == 0
    _assert_equal(gpu, ref, f"block mode {mode} round_scale={round_scale}")


def test_decode_config_bulk_fill_full_size():
    """batch 8, 8 kv heads, D=128: positions 0..4094 into 8192 slots (slot = position)."""
    w = wl.DECODE
    g = wl.generator(w.seed)
    T = w.kv_len - 1
    x = wl.bf16_normal((w.B, w.Hkv, T, w.D), g)
    sm = torch.arange(T, dtype=torch.int32).repeat(w.B)
    cache0 = _prefill(0, w.B, w.Hkv, w.S, w.D, g)
    gpu, ref, err, _ = _run_both(0, x, sm, cache0, w.S)
    assert err == 0
    _assert_equal(gpu, ref, "decode fill")


def test_long_config_chunk_write():
    """batch 1, 16 kv heads, D=256: one 2048-token chunk at positions 129024..131071."""
    w = wl.LONG
    g = wl.generator(w.seed)
    x = wl.bf16_normal((w.B, w.Hkv, w.T, w.D), g)
    sm = torch.arange(w.S - w.T, w.S, dtype=torch.int32)
    S = w.S
    cache0 = _prefill(0, w.B, w.Hkv, S, w.D, wl.generator(99))
    gpu, ref, err, _ = _run_both(0, x, sm, cache0, S)
    _assert_equal(gpu, ref, "long chunk")


@pytest.mark.parametrize("mode", [0, 1, 3, 4, 6])
def test_second_identical_write_is_a_no_op_on_gpu(mode):
    g = wl.generator(3000 + mode)
    B, H, T, D, S = 2, 4, 33, 128, 96
    x = wl.bf16_normal((B, H, T, D), g).to(DEV)
    sm = torch.stack([wl.slot_mapping_random(T, S, 4, g) for _ in range(B)]).reshape(-1).to(DEV)
    cache = [None if c is None else c.to(DEV) for c in _prefill(mode, B, H, S, D, g)]
    kvq.write(mode, x, sm, cache[0], cache[1], cache[2])
    once = [None if c is None else c.clone() for c in cache]
    kvq.write(mode, x, sm, cache[0], cache[1], cache[2])
    for a, b in zip(cache, once):
        if a is not None:
            assert torch.equal(a.view(torch.uint8) if a.dtype != torch.float32 else a.view(torch.int32),
                               b.view(torch.uint8) if b.dtype != torch.float32 else b.view(torch.int32))


def test_out_of_range_slots_are_skipped_and_flagged():
    g = wl.generator(4000)
    B, H, T, D, S = 1, 2, 16, 64, 32
    x = wl.bf16_normal((B, H, T, D), g)
    sm = wl.slot_mapping_random(T, S, 2, g)
    sm[3] = S + 5
    sm[4] = -9
    cache0 = _prefill(0, B, H, S, D, g)
    gpu, ref, err, oerr = _run_both(0, x, sm, cache0, S)
    assert err & kvq.KVQ_ERR_SLOT_RANGE and oerr & 1
    _assert_equal(gpu, ref, "bad slots")


def test_empty_and_all_skipped():
    g = wl.generator(5000)
    D, S = 128, 16
    cache = [c.to(DEV) for c in _prefill(0, 1, 1, S, D, g)]
    before = [c.clone() for c in cache]
    x = wl.bf16_normal((1, 1, 4, D), g).to(DEV)
    sm = torch.full((4,), -1, dtype=torch.int32, device=DEV)
    kvq.write(0, x, sm, *cache)
    x0 = torch.empty((1, 1, 0, D), dtype=torch.bfloat16, device=DEV)
    kvq.write(0, x0, torch.empty(0, dtype=torch.int32, device=DEV), *cache)
    for a, b in zip(cache, before):
        assert torch.equal(a, b)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 37), (2, 8, 129)])
def test_tq4_write_ragged_shapes(D, shape):
    """Mode 7 (TQ4: 4-bit affine per token and head, two codes per byte):
    codes, scales and zero points bit-exact, untouched slots byte-equal."""
    B, H, T = shape
    g = wl.generator(4000 + D + 7 * T)
    S = 2 * T + 3
    x = wl.bf16_normal((B, H, T, D), g, outlier_p=0.02, outlier_scale=8.0)
    sp = _special_rows(D, g)
    n = min(T, sp.shape[0])
    x[0, 0, :n] = sp[:n]
    sm = torch.stack([wl.slot_mapping_random(T, S, T // 5, g) for _ in range(B)]).reshape(-1)
    cache0 = _prefill(7, B, H, S, D, g)
    gpu, ref, err, oerr = _run_both(7, x, sm, cache0, S)
    assert err == 0 and oerr == 0
    _assert_equal(gpu, ref, f"tq4 D={D} shape={shape}")


@pytest.mark.parametrize("mode", [0, 1, 3, 7])
@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 37), (8, 8, 1)])
def test_write_kv_matches_two_oracle_writes(mode, shape):
    """kvq_write_kv: K and V written in one launch, each bit-exact against the
    oracle's write of that tensor alone; k is a strided view (a slice of a
    wider tensor), v contiguous; some slots are -1."""
    B, H, T = shape
    D = 128
    g = wl.generator(7000 + mode + 3 * T)
    S = 2 * T + 5
    wide = wl.bf16_normal((B, H, T, 2 * D), g, outlier_p=0.01, outlier_scale=10.0)
    k = wide[..., D:]  # row stride 2D elements: still 16-byte aligned rows
    v = wl.bf16_normal((B, H, T, D), g)
    sm = torch.stack([wl.slot_mapping_random(T, S, T // 4, g) for _ in range(B)]).reshape(-1)
    k0, v0 = _prefill(mode, B, H, S, D, g), _prefill(mode, B, H, S, D, g)
    kg = [None if c is None else c.to(DEV) for c in k0]
    vg = [None if c is None else c.to(DEV) for c in v0]
    err = err_word()
    kvq.write_kv(mode, k.to(DEV), v.to(DEV), sm.to(DEV), kg, vg, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for x, c0, cg, what in ((k, k0, kg, "K"), (v, v0, vg, "V")):
        ref = [None if c is None else c.numpy().copy() for c in c0]
        oerr = oracle.write(mode, wl.u16(x.contiguous()), sm.numpy(), S, ref[0], ref[1], ref[2])
        assert oerr == 0
        _assert_equal([None if c is None else c.cpu().numpy() for c in cg], ref, f"write_kv {what} mode={mode}")


def test_write_kv_rejects_mismatched_arguments():
    g = wl.generator(7100)
    D, S = 64, 16
    kc = [c.to(DEV) for c in _prefill(0, 1, 1, S, D, g)]
    vc = [c.to(DEV) for c in _prefill(0, 1, 1, S, D, g)]
    x = wl.bf16_normal((1, 1, 2, D), g).to(DEV)
    sm = torch.tensor([0, 1], dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError):
        kvq.write_kv(0, x, x[:, :, :1], sm, kc, vc)
    with pytest.raises(RuntimeError):
        kvq.write_kv(0, x, x, sm, kc, (vc[0], vc[1], None))  # mode 0 needs V zero points
