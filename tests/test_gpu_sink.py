"""GPU parity of the attention-sink / ring slot plan and mask (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_20_b200 import kvq
from quantized_kv_cache_20_b200 import workloads as wl
from tests.helpers import DEV, err_word, int32_scalar

pytestmark = pytest.mark.gpu


def _step(pos, T, B, sink, S, slot_pos_d, slot_pos_o, mask_rows):
    ip = int32_scalar(pos)
    sm = torch.empty(B * T, dtype=torch.int32, device=DEV)
    kv = torch.empty(1, dtype=torch.int32, device=DEV)
    kvq.sink_plan(ip, B, T, sink, slot_pos_d, sm, kv)
    mask = torch.empty((mask_rows, S), dtype=torch.float32, device=DEV)
    kvq.sink_mask(ip, mask_rows, slot_pos_d, mask)
    sm_o, kv_o = oracle.sink_plan(pos, B, T, sink, S, slot_pos_o)
    mask_o = oracle.sink_mask(pos, mask_rows, slot_pos_o)
    assert np.array_equal(sm.cpu().numpy(), sm_o)
    assert int(kv.item()) == kv_o
    assert np.array_equal(slot_pos_d.cpu().numpy(), slot_pos_o)
    assert np.array_equal(mask.cpu().numpy().view(np.uint32), mask_o.view(np.uint32))


@pytest.mark.parametrize("sink", [0, 4])
def test_small_ring_with_mixed_chunks(sink):
    S, B = 32, 2
    sp_d = torch.full((S,), -1, dtype=torch.int32, device=DEV)
    sp_o = np.full(S, -1, np.int32)
    pos = 0
    for step in range(60):
        T = [1, 3, 7, S - sink][step % 4]
        _step(pos, T, B, sink, S, sp_d, sp_o, T)
        pos += T


def test_sink_config_decode_positions():
    """4 sink + 2044 ring slots, positions stepped 0..10000 one at a time."""
    w = wl.SINK
    checks = {0, 3, 4, 5, 2047, 2048, 2049, 4095, 4096, 6143, 10000}
    sp_d = torch.full((w.S,), -1, dtype=torch.int32, device=DEV)
    sp_o = np.full(w.S, -1, np.int32)
    ip = torch.zeros(1, dtype=torch.int32, device=DEV)
    sm = torch.empty(1, dtype=torch.int32, device=DEV)
    kv = torch.empty(1, dtype=torch.int32, device=DEV)
    for p in range(10001):
        if p in checks:
            _step(p, 1, 1, w.sink, w.S, sp_d, sp_o, 1)
        else:
            ip.fill_(p)
            kvq.sink_plan(ip, 1, 1, w.sink, sp_d, sm, kv)
            oracle.sink_plan(p, 1, 1, w.sink, w.S, sp_o)


def test_sink_config_prefill_chunks_across_the_wrap():
    w = wl.SINK
    sp_d = torch.full((w.S,), -1, dtype=torch.int32, device=DEV)
    sp_o = np.full(w.S, -1, np.int32)
    for c in range(40):
        _step(c * w.Lq, w.Lq, 1, w.sink, w.S, sp_d, sp_o, w.Lq)


def test_negative_position_is_flagged():
    S = 16
    sp = torch.full((S,), -1, dtype=torch.int32, device=DEV)
    sm = torch.zeros(2, dtype=torch.int32, device=DEV)
    kv = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    err = err_word()
    kvq.sink_plan(int32_scalar(-3), 1, 2, 2, sp, sm, kv, err_word=err)
    assert err.item() & kvq.KVQ_ERR_INPUT_POS
    assert sm.tolist() == [-1, -1] and kv.item() == 0
    assert torch.all(sp == -1)


def test_host_rejects_oversized_chunk():
    S = 16
    sp = torch.full((S,), -1, dtype=torch.int32, device=DEV)
    sm = torch.zeros(16, dtype=torch.int32, device=DEV)
    kv = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(kvq.KvqError) as e:
        kvq.sink_plan(int32_scalar(0), 1, 13, 4, sp, sm, kv)
    assert e.value.status == kvq.KVQ_EUNSUPPORTED


# ---------------------------------------------------------------------------- per-row positions

def _rows_step(pos, T, sink, S, sp_d, sp_o, Lq):
    """One per-row plan + mask on the GPU and in the oracle; bit-exact comparison."""
    B = len(pos)
    ip = torch.tensor(pos, dtype=torch.int32, device=DEV)
    sm = torch.empty(B * T, dtype=torch.int32, device=DEV)
    kv = torch.empty(B, dtype=torch.int32, device=DEV)
    err = err_word()
    kvq.sink_plan_rows(ip, T, sink, sp_d, sm, kv, err_word=err)
    mask = torch.empty((B, Lq, S), dtype=torch.float32, device=DEV)
    kvq.sink_mask_rows(ip, Lq, sp_d, mask)
    sm_o, kv_o = oracle.sink_plan_rows(np.array(pos, np.int32), T, sink, S, sp_o)
    mask_o = oracle.sink_mask_rows(np.array(pos, np.int32), Lq, sp_o)
    assert np.array_equal(sm.cpu().numpy(), sm_o)
    assert np.array_equal(kv.cpu().numpy(), kv_o)
    assert np.array_equal(sp_d.cpu().numpy(), sp_o)
    assert np.array_equal(mask.cpu().numpy().view(np.uint32), mask_o.view(np.uint32))
    assert (err.item() & kvq.KVQ_ERR_INPUT_POS) == (kvq.KVQ_ERR_INPUT_POS if min(pos) < 0 else 0)
    return ip, sm, kv, mask, sm_o, kv_o, mask_o


@pytest.mark.parametrize("sink", [0, 4])
def test_rows_plan_and_mask_ragged_positions(sink):
    """Five rows stepping from different positions (one of them not started,
    input_pos -1, until step 20) through a 64-slot ring, in chunks of 1..5."""
    S = 64
    start = [0, 17, 60, 200, -1]
    sp_d = torch.full((len(start), S), -1, dtype=torch.int32, device=DEV)
    sp_o = np.full((len(start), S), -1, np.int32)
    pos = list(start)
    for step in range(40):
        T = [1, 2, 5][step % 3]
        if step == 20:
            pos[4] = 0
        _rows_step(pos, T, sink, S, sp_d, sp_o, T)
        pos = [p + T if p >= 0 else p for p in pos]


def test_ragged_sink_batch_decode_and_prefill():
    """A batch of three sequences at different positions of 4 + 2044 sink/ring
    caches: each row is brought to its position through the single-row API
    (chunks of up to 2044), then decoded together for a few steps (per-row
    plan -> write -> per-row mask -> varlen decode with one mask row per batch
    row) and once as a 64-token chunk (varlen prefill, mask [B, Lq, S])."""
    w = wl.SINK
    S, D, sink, Hq, Hkv = w.S, w.D, w.sink, w.Hq, w.Hkv
    starts = [100, 2500, 6000]
    B = len(starts)
    g = wl.generator(9090)
    Kc = wl.int8_cache_random(B, Hkv, S, D, g)
    Vc = wl.int8_cache_random(B, Hkv, S, D, g)
    Kd = [t.to(DEV) for t in Kc]
    Vd = [t.to(DEV) for t in Vc]
    Ko = [t.numpy().copy() for t in Kc]
    Vo = [t.numpy().copy() for t in Vc]
    sp_d = torch.full((B, S), -1, dtype=torch.int32, device=DEV)
    sp_o = np.full((B, S), -1, np.int32)

    def write_rows(k, v, sm_d, sm_o, T):
        kvq.write(0, k.to(DEV), sm_d, *Kd)
        kvq.write(0, v.to(DEV), sm_d, *Vd)
        oracle.write(0, wl.u16(k), sm_o, S, *Ko)
        oracle.write(0, wl.u16(v), sm_o, S, *Vo)

    # bring each row to its start through the single-row plan on its own slot table
    for b, p_end in enumerate(starts):
        p = 0
        while p < p_end:
            T = min(S - sink, p_end - p)
            k = wl.bf16_normal((1, Hkv, T, D), g)
            v = wl.bf16_normal((1, Hkv, T, D), g)
            row_d = sp_d[b].clone()
            smd = torch.empty(T, dtype=torch.int32, device=DEV)
            kvd = torch.empty(1, dtype=torch.int32, device=DEV)
            kvq.sink_plan(int32_scalar(p), 1, T, sink, row_d, smd, kvd)
            sp_d[b].copy_(row_d)
            row_o = sp_o[b].copy()
            smo, _ = oracle.sink_plan(p, 1, T, sink, S, row_o)
            sp_o[b] = row_o
            kvq.write(0, k.to(DEV), smd, *[t[b:b + 1] for t in Kd])
            kvq.write(0, v.to(DEV), smd, *[t[b:b + 1] for t in Vd])
            oracle.write(0, wl.u16(k), smo, S, *[t[b:b + 1] for t in Ko])
            oracle.write(0, wl.u16(v), smo, S, *[t[b:b + 1] for t in Vo])
            p += T
    assert np.array_equal(sp_d.cpu().numpy(), sp_o)

    pos = list(starts)
    for step in range(3):  # decode steps
        k = wl.bf16_normal((B, Hkv, 1, D), g)
        v = wl.bf16_normal((B, Hkv, 1, D), g)
        ip, sm, kv, mask, sm_o, kv_o, mask_o = _rows_step(pos, 1, sink, S, sp_d, sp_o, 1)
        write_rows(k, v, sm, sm_o, 1)
        q = wl.bf16_normal((B, Hq, 1, D), g)
        out = kvq.decode_attn_varlen(q.to(DEV), *Kd, *Vd, kv, mask=mask)
        torch.cuda.synchronize()
        got = out.float().cpu().double().numpy()
        for b in range(B):
            ref = oracle.sdpa(wl.u16(q[b:b + 1]), *[t[b:b + 1] for t in Ko], *[t[b:b + 1] for t in Vo],
                              kv_len=int(kv_o[b]), sm_scale=1 / np.sqrt(D), mask=mask_o[b])
            _close(got[b:b + 1], ref, f"ragged sink decode row {b} step {step}")
        pos = [p + 1 for p in pos]

    Lq = 64  # one chunk per row, each at its own position
    k = wl.bf16_normal((B, Hkv, Lq, D), g)
    v = wl.bf16_normal((B, Hkv, Lq, D), g)
    ip, sm, kv, mask, sm_o, kv_o, mask_o = _rows_step(pos, Lq, sink, S, sp_d, sp_o, Lq)
    write_rows(k, v, sm, sm_o, Lq)
    q = wl.bf16_normal((B, Hq, Lq, D), g)
    out = kvq.prefill_attn_varlen(q.to(DEV), *Kd, *Vd, kv, mask=mask)
    torch.cuda.synchronize()
    got = out.float().cpu().double().numpy()
    rows = [(0, h, i) for h in (0, 9, 31) for i in (0, 17, 63)]
    for b in range(B):
        ref = oracle.sdpa_rows(wl.u16(q[b:b + 1]), *[t[b:b + 1] for t in Ko], *[t[b:b + 1] for t in Vo],
                               kv_len=int(kv_o[b]), sm_scale=1 / np.sqrt(D), rows=rows, mask=mask_o[b])
        _close(np.stack([got[b, h, i] for _, h, i in rows]), ref, f"ragged sink prefill row {b}")


def _close(got, ref, what):
    from tests.helpers import assert_attn_close
    assert_attn_close(got, ref, what)
