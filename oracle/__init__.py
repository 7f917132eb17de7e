"""CPU oracle for the quantized KV-cache hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The CUDA library never routes through
it; it shares no code with ``quantized_kv_cache_20_b200``.

The arithmetic lives in ``kvq_oracle.c`` (plain C, IEEE binary32 for the
quantizers exactly as the formulas are written, fp64 for attention).  This
module builds it on demand with gcc and wraps it with ctypes over numpy arrays.
bf16 tensors travel as their raw ``uint16`` bit patterns.

Sources (page title, section) are cited in ``kvq_oracle.c``; each wrapper below
names the one it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkvq_oracle.so")
_lock = threading.Lock()
_lib = None

MODE_INT8_AFFINE = 0
MODE_FP8_E4M3 = 1
MODE_MXFP8 = 2
MODE_MXFP4 = 3
MODE_FP8_E5M2 = 4
MODE_MXFP8_E5M2 = 5
MODE_INT8_SYM = 6
MODE_INT4_AFFINE = 7
_F32_SCALE_MODES = (MODE_FP8_E4M3, MODE_FP8_E5M2, MODE_INT8_SYM)

_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile ``kvq_oracle.c`` into ``libkvq_oracle.so`` if stale; return its path."""
    stale = force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        lib.kvqo_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.kvqo_e4m3_value.restype = ctypes.c_double
        lib.kvqo_e4m3_encode.argtypes = [f32]
        lib.kvqo_e4m3_encode.restype = ctypes.c_uint8
        lib.kvqo_e5m2_value.argtypes = [ctypes.c_uint8]
        lib.kvqo_e5m2_value.restype = ctypes.c_double
        lib.kvqo_e5m2_encode.argtypes = [f32]
        lib.kvqo_e5m2_encode.restype = ctypes.c_uint8
        lib.kvqo_e8m0_floor.argtypes = [f32]
        lib.kvqo_e8m0_floor.restype = ctypes.c_uint8
        lib.kvqo_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.kvqo_e2m1_value.restype = ctypes.c_double
        lib.kvqo_e2m1_encode.argtypes = [f32]
        lib.kvqo_e2m1_encode.restype = ctypes.c_uint8
        lib.kvqo_e8m0_value.argtypes = [ctypes.c_uint8]
        lib.kvqo_e8m0_value.restype = ctypes.c_double
        lib.kvqo_e8m0_ceil.argtypes = [f32]
        lib.kvqo_e8m0_ceil.restype = ctypes.c_uint8
        lib.kvqo_e8m0_ocp.argtypes = [f32, i32]
        lib.kvqo_e8m0_ocp.restype = ctypes.c_uint8
        lib.kvqo_affine_int8_row.argtypes = [P, i32, P, P, P]
        lib.kvqo_affine_int8_row.restype = None
        lib.kvqo_affine_int4_row.argtypes = [P, i32, P, P, P]
        lib.kvqo_affine_int4_row.restype = None
        lib.kvqo_block_row.argtypes = [i32, i32, P, i32, P, P, P]
        lib.kvqo_block_row.restype = None
        lib.kvqo_write.argtypes = [i32, i32, P, i32, i32, i32, i32, P, P, i64, P, P, P, P]
        lib.kvqo_write.restype = None
        lib.kvqo_sink_plan.argtypes = [i32, i32, i32, i32, i64, P, P, P]
        lib.kvqo_sink_plan.restype = None
        lib.kvqo_sink_mask.argtypes = [i32, i32, P, i64, P]
        lib.kvqo_sink_mask.restype = None
        sdpa_args = [P, i32, i32, i32, i32, i32, P, P, P, P, P, P, i32, i64, i32, P, i32, f32]
        lib.kvqo_sdpa_row.argtypes = sdpa_args + [i32, i32, i32, P]
        lib.kvqo_sdpa_row.restype = None
        lib.kvqo_sdpa.argtypes = sdpa_args + [P]
        lib.kvqo_sdpa.restype = None
        lib.kvqo_dequant_block.argtypes = [i32, P, P, i64, i32, P]
        lib.kvqo_dequant_block.restype = None
        lib.kvqo_sdpa_dense_row.argtypes = [P, i32, i32, i32, i32, P, P, i32, i64, i32, P, i32, f32, i32, i32, i32,
                                             P]
        lib.kvqo_sdpa_dense_row.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype in (np.uint16, np.int16), "bf16 data travels as uint16 bit patterns"
    return x.view(np.uint16)


# --- number formats (OCP FP8 E4M3 "fn" and E5M2, OCP MX E2M1 / E8M0) ----------

def e4m3_value(code: int) -> float:
    return _load().kvqo_e4m3_value(int(code))


def e4m3_encode(v: float) -> int:
    return int(_load().kvqo_e4m3_encode(float(v)))


def e5m2_value(code: int) -> float:
    return _load().kvqo_e5m2_value(int(code))


def e5m2_encode(v: float) -> int:
    return int(_load().kvqo_e5m2_encode(float(v)))


def e2m1_value(code: int) -> float:
    return _load().kvqo_e2m1_value(int(code))


def e2m1_encode(v: float) -> int:
    return int(_load().kvqo_e2m1_encode(float(v)))


def e8m0_value(code: int) -> float:
    return _load().kvqo_e8m0_value(int(code))


def e8m0_ceil(s: float) -> int:
    return int(_load().kvqo_e8m0_ceil(float(s)))


def e8m0_floor(s: float) -> int:
    return int(_load().kvqo_e8m0_floor(float(s)))


def e8m0_ocp(amax: float, emax_elem: int) -> int:
    """OCP MX v1.0 shared exponent floor(log2 amax) - emax_elem, as E8M0."""
    return int(_load().kvqo_e8m0_ocp(float(amax), int(emax_elem)))


# --- quantizers --------------------------------------------------------------

def affine_int8_row(x_bits: np.ndarray):
    """ExecuTorch PR 24473, Summary: per-token-and-head affine int8 of one row.

    Returns (codes int8 [D], scale float32, zero_point int8)."""
    x = _u16(x_bits)
    D = x.shape[-1]
    q = np.zeros(D, np.int8)
    scale = np.zeros(1, np.float32)
    zp = np.zeros(1, np.int8)
    _load().kvqo_affine_int8_row(_ptr(x), D, _ptr(q), _ptr(scale), _ptr(zp))
    return q, scale[0], zp[0]


def affine_int4_row(x_bits: np.ndarray):
    """ExecuTorch PR 20351, commit notes (TQ4 cache: nibble-packed on the last
    dim): the 4-bit affine per-token-and-head reading of one row.

    Returns (packed uint8 [D/2], scale float32, zero_point uint8 in 0..15)."""
    x = _u16(x_bits)
    D = x.shape[-1]
    q = np.zeros(D // 2, np.uint8)
    scale = np.zeros(1, np.float32)
    zp = np.zeros(1, np.uint8)
    _load().kvqo_affine_int4_row(_ptr(x), D, _ptr(q), _ptr(scale), _ptr(zp))
    return q, scale[0], zp[0]


def block_row(mode: int, x_bits: np.ndarray, round_scale: int = 1):
    """IndexerQuantCache, 计算公式: per-32 block quantization of one row.
    round_scale (modes 2, 3, 5): 1 scale rounded up, 0 floor, 2 the OCP MX rule.

    Returns (codes uint8 [d or d/2], scales float32 [d/32] or uint8 E8M0 [d/32])."""
    x = _u16(x_bits)
    d = x.shape[-1]
    codes = np.zeros(d // 2 if mode == MODE_MXFP4 else d, np.uint8)
    sf = np.zeros(d // 32, np.float32)
    se = np.zeros(d // 32, np.uint8)
    _load().kvqo_block_row(mode, int(round_scale), _ptr(x), d, _ptr(codes), _ptr(sf), _ptr(se))
    return codes, (sf if mode in _F32_SCALE_MODES else se)


def write(mode: int, x_bits: np.ndarray, slot_mapping: np.ndarray, num_slots: int,
          codes: np.ndarray, scales: np.ndarray, zero_points: np.ndarray | None = None,
          round_scale: int = 1) -> int:
    """The cache write (quantize + scatter by slot_mapping, -1 = skip), in place.

    x_bits: uint16 [B, H, T, D] (any strides are flattened to contiguous here).
    Returns the error word (bit 0 = a slot outside [0, num_slots) was skipped)."""
    x = _u16(x_bits)
    B, H, T, D = x.shape
    xs = np.array([H * T * D, T * D, D, 1], np.int64)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int32)
    assert sm.size == B * T
    err = np.zeros(1, np.int32)
    _load().kvqo_write(mode, int(round_scale), _ptr(x), B, H, T, D, _ptr(xs), _ptr(sm),
                       int(num_slots), _ptr(codes), _ptr(scales), _ptr(zero_points), _ptr(err))
    return int(err[0])


# --- sink / ring layout --------------------------------------------------------

def sink_plan(input_pos: int, B: int, T: int, sink: int, S: int, slot_pos: np.ndarray):
    """ExecuTorch PR 24473, Summary (CachePositionsManagerWithSink): slots for
    positions input_pos .. input_pos+T-1; updates slot_pos in place.

    Returns (slot_mapping int32 [B*T], kv_len)."""
    assert slot_pos.dtype == np.int32 and slot_pos.size == S
    sm = np.zeros(B * T, np.int32)
    kv = np.zeros(1, np.int32)
    _load().kvqo_sink_plan(int(input_pos), B, T, int(sink), int(S), _ptr(sm), _ptr(slot_pos), _ptr(kv))
    return sm, int(kv[0])


def sink_mask(input_pos: int, Lq: int, slot_pos: np.ndarray) -> np.ndarray:
    """ExecuTorch PR 24473, Summary (_create_causal_mask_for_attention_sink):
    additive float mask [Lq, S]."""
    S = slot_pos.size
    mask = np.zeros((Lq, S), np.float32)
    _load().kvqo_sink_mask(int(input_pos), Lq, _ptr(np.ascontiguousarray(slot_pos, np.int32)), S,
                           _ptr(mask))
    return mask


def sink_plan_rows(input_pos, T: int, sink: int, S: int, slot_pos: np.ndarray):
    """The sink plan per batch row (each row its own sequence, with its own position
    input_pos[b] and its own slot table slot_pos[b]); updates slot_pos [B, S] in place.

    Returns (slot_mapping int32 [B*T], kv_lens int32 [B])."""
    assert slot_pos.dtype == np.int32 and slot_pos.ndim == 2 and slot_pos.shape[1] == S
    B = slot_pos.shape[0]
    sm = np.zeros(B * T, np.int32)
    kv = np.zeros(B, np.int32)
    for b in range(B):
        if int(input_pos[b]) < 0:  # no position: nothing is written, nothing is visible
            sm[b * T:(b + 1) * T] = -1
            continue
        row = np.ascontiguousarray(slot_pos[b])
        sm[b * T:(b + 1) * T], kv[b] = sink_plan(int(input_pos[b]), 1, T, sink, S, row)
        slot_pos[b] = row
    return sm, kv


def sink_mask_rows(input_pos, Lq: int, slot_pos: np.ndarray) -> np.ndarray:
    """The sink mask per batch row: [B, Lq, S], row b from input_pos[b] and slot_pos[b]."""
    return np.stack([sink_mask(int(input_pos[b]), Lq, slot_pos[b]) for b in range(slot_pos.shape[0])])


# --- attention -------------------------------------------------------------------

def _sdpa_common(q_bits, k, ks, kz, v, vs, vz, mask):
    """Codes are int8 [.., D] (kbits 8) or TQ4 nibbles uint8 [.., D/2] (kbits 4)."""
    q = _u16(q_bits)
    arrs = [np.ascontiguousarray(a) for a in (k, ks, kz, v, vs, vz)]
    for i in (0, 2, 3, 5):
        assert arrs[i].dtype in (np.int8, np.uint8)
        arrs[i] = arrs[i].view(np.int8)
    assert arrs[1].dtype == np.float32 and arrs[4].dtype == np.float32
    D = q.shape[-1]
    kbits = 4 if arrs[0].shape[-1] * 2 == D else 8
    assert arrs[0].shape[-1] * 8 == D * kbits and arrs[3].shape == arrs[0].shape
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.float32)
    return q, arrs, m, kbits


def sdpa(q_bits, k, ks, kz, v, vs, vz, kv_len: int, sm_scale: float, mask=None,
         is_causal: bool = False) -> np.ndarray:
    """fp64 attention over the dequantized int8 cache (abaddon KvCache::forward_attention
    shapes; ExecuTorch PR 20351 kv_len bound and causal rule; PR 24473 additive mask).

    q_bits uint16 [B, Hq, Lq, D]; k/v int8 [B, Hkv, S, D] or, for the TQ4 packing,
    uint8 nibbles [B, Hkv, S, D/2]; ks/vs f32 and kz/vz [B, Hkv, S].
    Returns float64 [B, Hq, Lq, D]."""
    q, (k, ks, kz, v, vs, vz), m, kbits = _sdpa_common(q_bits, k, ks, kz, v, vs, vz, mask)
    B, Hq, Lq, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    out = np.zeros((B, Hq, Lq, D), np.float64)
    _load().kvqo_sdpa(_ptr(q), B, Hq, Lq, D, kbits, _ptr(k), _ptr(ks), _ptr(kz), _ptr(v), _ptr(vs), _ptr(vz),
                      Hkv, S, int(kv_len), _ptr(m), int(bool(is_causal)), float(sm_scale), _ptr(out))
    return out


def sdpa_rows(q_bits, k, ks, kz, v, vs, vz, kv_len: int, sm_scale: float, rows, mask=None,
              is_causal: bool = False) -> np.ndarray:
    """Same as ``sdpa`` for selected (b, h, i) rows only; returns float64 [len(rows), D]."""
    q, (k, ks, kz, v, vs, vz), m, kbits = _sdpa_common(q_bits, k, ks, kz, v, vs, vz, mask)
    B, Hq, Lq, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    out = np.zeros((len(rows), D), np.float64)
    lib = _load()
    for n, (b, h, i) in enumerate(rows):
        lib.kvqo_sdpa_row(_ptr(q), B, Hq, Lq, D, kbits, _ptr(k), _ptr(ks), _ptr(kz), _ptr(v), _ptr(vs),
                          _ptr(vz), Hkv, S, int(kv_len), _ptr(m), int(bool(is_causal)), float(sm_scale),
                          int(b), int(h), int(i), out[n].ctypes.data)
    return out


def dequant_int8(codes: np.ndarray, scale: np.ndarray, zp: np.ndarray) -> np.ndarray:
    """(q - zp) * scale in fp64 (the dequantization of the affine int8 reading)."""
    return (codes.astype(np.float64) - zp.astype(np.float64)[..., None]) * scale.astype(np.float64)[..., None]


# --- attention over the per-32 block caches ---------------------------------------

def dequant_block(mode: int, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """IndexerQuantCache, 计算公式 (x ~ code * scale_g): the fp64 values of a block
    cache, codes [.., d] (mode 3: [.., d/2]) and scales [.., d/32]."""
    codes = np.ascontiguousarray(codes).view(np.uint8)
    scales = np.ascontiguousarray(scales)
    d = scales.shape[-1] * 32
    rows = int(np.prod(codes.shape[:-1]))
    out = np.zeros(codes.shape[:-1] + (d,), np.float64)
    _load().kvqo_dequant_block(int(mode), _ptr(codes), _ptr(scales), rows, d, _ptr(out))
    return out


def sdpa_dense(q_bits, K: np.ndarray, V: np.ndarray, kv_len: int, sm_scale: float, mask=None,
               is_causal: bool = False) -> np.ndarray:
    """The same attention as ``sdpa`` over K, V given as fp64 values [B, Hkv, S, D]."""
    q = _u16(q_bits)
    K = np.ascontiguousarray(K, np.float64)
    V = np.ascontiguousarray(V, np.float64)
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.float32)
    B, Hq, Lq, D = q.shape
    Hkv, S = K.shape[1], K.shape[2]
    out = np.zeros((B, Hq, Lq, D), np.float64)
    lib = _load()
    for b in range(B):
        for h in range(Hq):
            for i in range(Lq):
                lib.kvqo_sdpa_dense_row(_ptr(q), B, Hq, Lq, D, _ptr(K), _ptr(V), Hkv, S, int(kv_len), _ptr(m),
                                        int(bool(is_causal)), float(sm_scale), b, h, i, out[b, h, i].ctypes.data)
    return out


def sdpa_dense_rows(q_bits, K: np.ndarray, V: np.ndarray, kv_len: int, sm_scale: float, rows, mask=None,
                    is_causal: bool = False) -> np.ndarray:
    """``sdpa_dense`` for selected (b, h, i) rows only; returns float64 [len(rows), D]."""
    q = _u16(q_bits)
    K = np.ascontiguousarray(K, np.float64)
    V = np.ascontiguousarray(V, np.float64)
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.float32)
    B, Hq, Lq, D = q.shape
    Hkv, S = K.shape[1], K.shape[2]
    out = np.zeros((len(rows), D), np.float64)
    lib = _load()
    for n, (b, h, i) in enumerate(rows):
        lib.kvqo_sdpa_dense_row(_ptr(q), B, Hq, Lq, D, _ptr(K), _ptr(V), Hkv, S, int(kv_len), _ptr(m),
                                int(bool(is_causal)), float(sm_scale), int(b), int(h), int(i), out[n].ctypes.data)
    return out


def sdpa_block(mode: int, q_bits, k_codes, k_scales, v_codes, v_scales, kv_len: int, sm_scale: float,
               mask=None, is_causal: bool = False) -> np.ndarray:
    """fp64 attention over a per-32 block cache: dequantize, then ``sdpa_dense``."""
    return sdpa_dense(q_bits, dequant_block(mode, k_codes, k_scales), dequant_block(mode, v_codes, v_scales),
                      kv_len, sm_scale, mask=mask, is_causal=is_causal)

