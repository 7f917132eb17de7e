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
