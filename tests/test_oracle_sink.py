"""Pins for the oracle's attention-sink / ring layout and mask (CPU only).

ExecuTorch PR 24473, Summary: CachePositionsManagerWithSink assigns the write
slots (pinned sink prefix + ring), the ring cache is the sink cache with
sink_size = 0, the mask comes from _create_causal_mask_for_attention_sink and is
an additive float mask; a full-context cache keeps plain causal attention.
The slot formula and the visibility rule are readings; they are pinned by the
special cases they must reduce to and by a hand-derived example.
"""
import os

import numpy as np
import pytest

import oracle


def _rows(path):
    with open(path) as f:
        return [l.split() for l in f if l.strip() and not l.startswith("#")]


def test_golden_single_token_plan(golden_dir):
    sink, S = 2, 6
    slot_pos = np.full(S, -1, np.int32)
    for p, slot, kv in _rows(os.path.join(golden_dir, "sink_plan.txt")):
        sm, kv_len = oracle.sink_plan(int(p), 1, 1, sink, S, slot_pos)
        assert sm[0] == int(slot) and kv_len == int(kv)
    assert slot_pos.tolist() == [0, 1, 10, 11, 8, 9]


def test_golden_chunk_mask(golden_dir):
    sink, S = 2, 6
    slot_pos = np.full(S, -1, np.int32)
    for p in range(6):
        oracle.sink_plan(p, 1, 1, sink, S, slot_pos)
    sm, kv_len = oracle.sink_plan(6, 1, 3, sink, S, slot_pos)
    assert sm.tolist() == [2, 3, 4] and kv_len == 6
    rows = _rows(os.path.join(golden_dir, "sink_mask.txt"))
    assert [int(v) for v in rows[0][1:]] == slot_pos.tolist()
    mask = oracle.sink_mask(6, 3, slot_pos)
    for r, row in enumerate(rows[1:]):
        want = [0.0 if v == "0" else -np.inf for v in row[2:]]
        assert mask[r].tolist() == want


def test_sink_zero_is_plain_ring():
    S = 16
    slot_pos = np.full(S, -1, np.int32)
    for p in range(100):
        sm, _ = oracle.sink_plan(p, 1, 1, 0, S, slot_pos)
        assert sm[0] == p % S


@pytest.mark.parametrize("sink", [0, 4])
def test_before_wrap_slot_is_position_and_mask_is_causal(sink):
    S = 64
    slot_pos = np.full(S, -1, np.int32)
    for p in range(S):
        sm, kv_len = oracle.sink_plan(p, 1, 1, sink, S, slot_pos)
        assert sm[0] == p and kv_len == p + 1
        mask = oracle.sink_mask(p, 1, slot_pos)[0]
        causal = np.where(np.arange(S) <= p, 0.0, -np.inf)
        assert np.array_equal(mask, causal)


def test_filled_count_sinks_visible_and_window():
    sink, S = 4, 32
    ring = S - sink
    slot_pos = np.full(S, -1, np.int32)
    p = 0
    for step in range(40):
        T = [1, 3, 7, 28][step % 4]
        oracle.sink_plan(p, 1, T, sink, S, slot_pos)
        last = p + T - 1
        assert (slot_pos >= 0).sum() == min(last + 1, S)
        mask = oracle.sink_mask(p, T, slot_pos)
        for r in range(T):
            qpos = p + r
            vis = mask[r] == 0
            assert np.all(vis[:min(sink, qpos + 1)])          # sinks always visible
            # the window term (qpos - pos < ring for ring slots) changes nothing
            ring_vis = vis[sink:]
            pos = slot_pos[sink:]
            assert np.all(qpos - pos[ring_vis] < ring)
            # visible count never exceeds what a one-token-at-a-time decode sees
            assert vis.sum() <= min(qpos + 1, S)
        p += T


def test_rows_plan_is_the_single_sequence_plan_per_row():
    """Per-row positions (a ragged batch): each row's slots, slot table, kv_len and
    mask are those of the single-sequence plan run on that row alone; rows with
    the same position agree; a negative position writes nothing."""
    S, sink, T = 64, 4, 3
    pos = np.array([0, 5, 61, 130, 5, -1], np.int32)
    sp = np.full((len(pos), S), -1, np.int32)
    sm, kv = oracle.sink_plan_rows(pos, T, sink, S, sp)
    for b, p in enumerate(pos):
        if p < 0:
            assert np.all(sm[b * T:(b + 1) * T] == -1) and kv[b] == 0 and np.all(sp[b] == -1)
            continue
        alone = np.full(S, -1, np.int32)
        sm1, kv1 = oracle.sink_plan(int(p), 1, T, sink, S, alone)
        assert np.array_equal(sm[b * T:(b + 1) * T], sm1) and kv[b] == kv1 and np.array_equal(sp[b], alone)
        # the ring formula, by hand
        for t in range(T):
            q = int(p) + t
            assert sm[b * T + t] == (q if q < sink else sink + (q - sink) % (S - sink))
    assert np.array_equal(sm[T:2 * T], sm[4 * T:5 * T]) and np.array_equal(sp[1], sp[4])
    m = oracle.sink_mask_rows(np.maximum(pos, 0), T, sp)
    for b in range(len(pos)):
        assert np.array_equal(m[b], oracle.sink_mask(int(max(pos[b], 0)), T, sp[b]))
