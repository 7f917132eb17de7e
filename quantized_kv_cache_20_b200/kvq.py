"""Thin ctypes binding of libkvq.so (the C ABI in include/kvq.h).

Argument marshalling only: shapes, dtypes and devices are read from torch
tensors, pointers and sizes are passed to the library, and every kernel runs
on torch's current CUDA stream.  There is no fallback: if libkvq.so is missing
or a call fails, a RuntimeError is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
KVQ_EINVAL = -1
KVQ_EUNSUPPORTED = -2
KVQ_ECUDA = -3
KVQ_ESCRATCH = -4
STATIC_SCRATCH_BYTES = 1 << 20

KVQ_ERR_SLOT_RANGE = 1
KVQ_ERR_KV_LEN_RANGE = 2
KVQ_ERR_INPUT_POS = 4
KVQ_ERR_TIMEOUT = 8

MODE_INT8_AFFINE = 0
MODE_FP8_E4M3 = 1
MODE_MXFP8 = 2
MODE_MXFP4 = 3
MODE_FP8_E5M2 = 4
MODE_MXFP8_E5M2 = 5
MODE_INT8_SYM = 6
MODE_INT4_AFFINE = 7

SCALE_FLOOR = 0  # round_scale values for the E8M0-scaled modes 2, 3, 5
SCALE_CEIL = 1
SCALE_OCP = 2

EXPORTS = (
    "kvq_write", "kvq_write_kv", "kvq_sink_plan", "kvq_sink_mask", "kvq_sink_plan_rows", "kvq_sink_mask_rows",
    "kvq_decode_workspace_bytes",
    "kvq_decode_attn", "kvq_decode_attn_static", "kvq_decode_static_reset", "kvq_decode_attn_varlen", "kvq_decode_attn_tq4",
    "kvq_decode_block_workspace_bytes", "kvq_decode_attn_block", "kvq_prefill_attn", "kvq_prefill_attn_varlen",
    "kvq_prefill_attn_block",
    "kvq_set_wait_limit_ns", "kvq_strerror", "kvq_version",
)

_lib = None
_lock = threading.Lock()


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libkvq.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:  # loaded: no lock on the call path
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libkvq.so not found at {p}; build it with "
                               "`python -m quantized_kv_cache_20_b200.build`")
        lib = ctypes.CDLL(p)
        P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        lib.kvq_write.argtypes = [I, I, P, I, I, I, I, P, P, I64, P, P, P, P, P]
        lib.kvq_write.restype = I
        lib.kvq_write_kv.argtypes = [I, I, P, P, I, I, I, I, P, P, P, I64, P, P, P, P, P, P, P, P]
        lib.kvq_write_kv.restype = I
        lib.kvq_sink_plan.argtypes = [P, I, I, I, I64, P, P, P, P, P]
        lib.kvq_sink_plan.restype = I
        lib.kvq_sink_mask.argtypes = [P, I, P, I64, P, P]
        lib.kvq_sink_mask.restype = I
        lib.kvq_sink_plan_rows.argtypes = [P, I, I, I, I64, P, P, P, P, P]
        lib.kvq_sink_plan_rows.restype = I
        lib.kvq_sink_mask_rows.argtypes = [P, I, I, P, I64, P, P]
        lib.kvq_sink_mask_rows.restype = I
        lib.kvq_decode_workspace_bytes.argtypes = [I, I, I, I, I64]
        lib.kvq_decode_workspace_bytes.restype = SZ
        lib.kvq_decode_attn.argtypes = [P, I, I, I, I, P, P, P, P, P, P, I64, P, P, F, P, P, SZ, P, P]
        lib.kvq_decode_attn_varlen.argtypes = [P, I, I, I, I, P, P, P, P, P, P, I64, P, P, I64, F, P, P, SZ, P, P]
        lib.kvq_decode_attn_varlen.restype = I
        lib.kvq_decode_attn_tq4.argtypes = lib.kvq_decode_attn.argtypes
        lib.kvq_decode_attn_tq4.restype = I
        lib.kvq_decode_block_workspace_bytes.argtypes = [I, I, I, I, I64]
        lib.kvq_decode_block_workspace_bytes.restype = SZ
        lib.kvq_decode_attn_block.argtypes = [I, P, I, I, I, I, P, P, P, P, I64, P, P, F, P, P, SZ, P, P]
        lib.kvq_decode_attn_block.restype = I
        lib.kvq_decode_attn.restype = I
        lib.kvq_decode_attn_static.argtypes = [P, I, I, I, I, P, P, P, P, P, P, I64, P, P, F, P, P, P]
        lib.kvq_decode_attn_static.restype = I
        lib.kvq_decode_static_reset.argtypes = [P]
        lib.kvq_decode_static_reset.restype = I
        lib.kvq_prefill_attn.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, I64, P, P, I, I, F, P, P, P]
        lib.kvq_prefill_attn_varlen.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, I64, P, P, I64, I, I, F, P, P,
                                                P]
        lib.kvq_prefill_attn_varlen.restype = I
        lib.kvq_prefill_attn.restype = I
        lib.kvq_prefill_attn_block.argtypes = [I, P, I, I, I, I, I, P, P, P, P, I64, P, P, I, I, F, P, P, P]
        lib.kvq_prefill_attn_block.restype = I
        lib.kvq_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.kvq_set_wait_limit_ns.restype = I
        lib.kvq_strerror.argtypes = [I]
        lib.kvq_strerror.restype = ctypes.c_char_p
        lib.kvq_version.argtypes = []
        lib.kvq_version.restype = I
        _lib = lib
        return lib


def strerror(status: int) -> str:
    return load().kvq_strerror(int(status)).decode()


def _check(fn: str, status: int):
    if status != KVQ_OK:
        raise KvqError(fn, status, strerror(status))


def _ptr(t):
    """A tensor's device address as a plain int (ctypes passes it as void*), or None."""
    return None if t is None else t.data_ptr()


# The current stream's raw handle without building a Stream object (the
# binding sits on every decode step's host path); the public call otherwise.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device) -> int:
    if _raw_stream is not None:
        return _raw_stream(device.index if device.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(device).cuda_stream


# The current device index without the lazy-init check of torch.cuda.current_device
# (CUDA is initialised once a CUDA tensor exists); the public call otherwise.
_get_device = getattr(torch._C, "_cuda_getDevice", None) or torch.cuda.current_device


def _on_current_device(t):
    """The library launches on the current device (its SM count, its per-device
    state); a tensor on another device would be read from the wrong context."""
    idx = t.device.index
    if idx is not None and idx != _get_device():
        raise ValueError(f"tensors are on cuda:{idx} but the current device is cuda:{torch.cuda.current_device()}; "
                         "call under torch.cuda.device(...)")


def _cuda(name, t, dtype=None, contiguous=True):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def write(mode: int, x: torch.Tensor, slot_mapping: torch.Tensor, codes: torch.Tensor,
          scales: torch.Tensor, zero_points: torch.Tensor | None = None, *, round_scale: int = SCALE_CEIL,
          err_word: torch.Tensor | None = None) -> None:
    """kvq_write: quantize x [B, H, T, D] (bf16, any strides with unit last stride)
    and scatter into the cache in place.  num_slots is codes.shape[2].  round_scale
    (modes 2, 3, 5): SCALE_CEIL (1 / True), SCALE_FLOOR (0 / False) or SCALE_OCP (2)."""
    _cuda("x", x, torch.bfloat16, contiguous=False)
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("x must be [B, H, T, D] with a unit last stride")
    _cuda("slot_mapping", slot_mapping, torch.int32)
    _cuda("codes", codes)
    _cuda("scales", scales)
    _cuda("zero_points", zero_points)
    _cuda("err_word", err_word, torch.int32)
    _on_current_device(x)
    B, H, T, D = x.shape
    strides = (ctypes.c_int64 * 4)(*x.stride())
    st = load().kvq_write(int(mode), int(round_scale), _ptr(x), B, H, T, D, strides,
                          _ptr(slot_mapping), int(codes.shape[2]), _ptr(codes), _ptr(scales),
                          _ptr(zero_points), _ptr(err_word), _stream(x.device))
    _check("kvq_write", st)


def write_kv(mode: int, k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, k_cache, v_cache, *,
             round_scale: int = SCALE_CEIL, err_word: torch.Tensor | None = None) -> None:
    """kvq_write_kv: kvq_write of k and v (both bf16 [B, H, T, D], unit last stride)
    in one launch.  k_cache / v_cache are (codes, scales, zero_points or None)."""
    for n, t in (("k", k), ("v", v)):
        _cuda(n, t, torch.bfloat16, contiguous=False)
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError(f"{n} must be [B, H, T, D] with a unit last stride")
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    _cuda("slot_mapping", slot_mapping, torch.int32)
    kc, ks, kz = (tuple(k_cache) + (None,))[:3]
    vc, vs, vz = (tuple(v_cache) + (None,))[:3]
    for n, t in (("k_codes", kc), ("k_scales", ks), ("k_zero_points", kz), ("v_codes", vc), ("v_scales", vs),
                 ("v_zero_points", vz)):
        _cuda(n, t)
    if kc.shape[2] != vc.shape[2]:
        raise ValueError("the K and V caches must have the same number of slots")
    _cuda("err_word", err_word, torch.int32)
    _on_current_device(k)
    B, H, T, D = k.shape
    ks_ = (ctypes.c_int64 * 4)(*k.stride())
    vs_ = (ctypes.c_int64 * 4)(*v.stride())
    st = load().kvq_write_kv(int(mode), int(round_scale), _ptr(k), _ptr(v), B, H, T, D, ks_, vs_,
                             _ptr(slot_mapping), int(kc.shape[2]), _ptr(kc), _ptr(ks), _ptr(kz), _ptr(vc), _ptr(vs),
                             _ptr(vz), _ptr(err_word), _stream(k.device))
    _check("kvq_write_kv", st)


def sink_plan(input_pos: torch.Tensor, B: int, T: int, sink_size: int, slot_pos: torch.Tensor,
              slot_mapping: torch.Tensor, kv_len: torch.Tensor,
              err_word: torch.Tensor | None = None) -> None:
    """kvq_sink_plan: slot_mapping [B*T] and kv_len (device scalar) for T tokens
    starting at the device scalar input_pos; updates slot_pos [S] in place."""
    for n, t in (("input_pos", input_pos), ("slot_pos", slot_pos), ("slot_mapping", slot_mapping),
                 ("kv_len", kv_len), ("err_word", err_word)):
        _cuda(n, t, torch.int32)
    _on_current_device(slot_pos)
    st = load().kvq_sink_plan(_ptr(input_pos), B, T, sink_size, slot_pos.numel(), _ptr(slot_mapping),
                              _ptr(slot_pos), _ptr(kv_len), _ptr(err_word), _stream(slot_pos.device))
    _check("kvq_sink_plan", st)


def sink_mask(input_pos: torch.Tensor, Lq: int, slot_pos: torch.Tensor, mask: torch.Tensor) -> None:
    """kvq_sink_mask: additive mask [Lq, S] (float32) from slot_pos."""
    _cuda("input_pos", input_pos, torch.int32)
    _cuda("slot_pos", slot_pos, torch.int32)
    _cuda("mask", mask, torch.float32)
    _on_current_device(mask)
    st = load().kvq_sink_mask(_ptr(input_pos), Lq, _ptr(slot_pos), slot_pos.numel(), _ptr(mask),
                              _stream(mask.device))
    _check("kvq_sink_mask", st)


def sink_plan_rows(input_pos: torch.Tensor, T: int, sink_size: int, slot_pos: torch.Tensor,
                   slot_mapping: torch.Tensor, kv_lens: torch.Tensor,
                   err_word: torch.Tensor | None = None) -> None:
    """kvq_sink_plan_rows: per batch row b, T tokens from input_pos[b] (int32 [B]);
    slot_pos int32 [B, S] in/out, slot_mapping int32 [B*T] and kv_lens int32 [B] out."""
    for n, t in (("input_pos", input_pos), ("slot_pos", slot_pos), ("slot_mapping", slot_mapping),
                 ("kv_lens", kv_lens), ("err_word", err_word)):
        _cuda(n, t, torch.int32)
    if slot_pos.dim() != 2 or slot_pos.shape[0] != input_pos.numel():
        raise ValueError("slot_pos must be [B, S] with B = input_pos.numel()")
    _on_current_device(slot_pos)
    B, S = slot_pos.shape
    st = load().kvq_sink_plan_rows(_ptr(input_pos), B, T, sink_size, S, _ptr(slot_mapping), _ptr(slot_pos),
                                   _ptr(kv_lens), _ptr(err_word), _stream(slot_pos.device))
    _check("kvq_sink_plan_rows", st)


def sink_mask_rows(input_pos: torch.Tensor, Lq: int, slot_pos: torch.Tensor, mask: torch.Tensor) -> None:
    """kvq_sink_mask_rows: additive mask [B, Lq, S] (float32) from slot_pos [B, S]."""
    _cuda("input_pos", input_pos, torch.int32)
    _cuda("slot_pos", slot_pos, torch.int32)
    _cuda("mask", mask, torch.float32)
    if slot_pos.dim() != 2 or mask.shape != (slot_pos.shape[0], Lq, slot_pos.shape[1]):
        raise ValueError("slot_pos must be [B, S] and mask [B, Lq, S]")
    _on_current_device(mask)
    B, S = slot_pos.shape
    st = load().kvq_sink_mask_rows(_ptr(input_pos), B, Lq, _ptr(slot_pos), S, _ptr(mask), _stream(mask.device))
    _check("kvq_sink_mask_rows", st)


def _mask_batch_stride(mask, B, Lq, S):
    """0 for one mask shared by every batch row ([S] / [Lq, S]); Lq * S for a
    per-row mask [B, Lq, S] (decode: [B, 1, S] or [B, S])."""
    if mask is None or mask.numel() == Lq * S:
        return 0
    if mask.numel() == B * Lq * S:
        return Lq * S
    raise ValueError(f"mask must hold Lq*S or B*Lq*S floats, got shape {tuple(mask.shape)}")


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, D: int, S: int) -> int:
    return int(load().kvq_decode_workspace_bytes(B, Hq, Hkv, D, S))


def decode_workspace(B: int, Hq: int, Hkv: int, D: int, S: int, device) -> torch.Tensor:
    """A zero-filled workspace of the size kvq_decode_attn needs (its merge counters,
    the first 1 KiB, start at zero; each completed call leaves them at zero, so it
    can be reused by later calls of any shape that fit it)."""
    with torch.cuda.device(device):
        n = decode_workspace_bytes(B, Hq, Hkv, D, S)
    if n == 0:
        raise ValueError("unsupported decode configuration")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _attn_common(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, mask, out, err_word):
    _cuda("q", q, torch.bfloat16)
    for n, t in (("k", k), ("k_zp", k_zp), ("v", v), ("v_zp", v_zp)):
        _cuda(n, t, torch.int8)
    _cuda("k_scale", k_scale, torch.float32)
    _cuda("v_scale", v_scale, torch.float32)
    _cuda("kv_len", kv_len, torch.int32)
    _cuda("mask", mask, torch.float32)
    _cuda("out", out, torch.bfloat16)
    _cuda("err_word", err_word, torch.int32)
    if k.dim() != 4 or q.dim() != 4:
        raise ValueError("q must be [B, Hq, Lq, D] and k/v [B, Hkv, S, D]")
    _on_current_device(q)


def decode_attn(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, *, out=None, mask=None, sm_scale=None,
                workspace=None, err_word=None) -> torch.Tensor:
    """kvq_decode_attn: q [B, Hq, 1, D] bf16 over the int8 cache [B, Hkv, S, D].
    kv_len: int32 device scalar.  (decode_attn_varlen takes one per batch row.)"""
    return _decode(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, out, mask, sm_scale, workspace, err_word,
                   varlen=False)


def decode_attn_varlen(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_lens, *, out=None, mask=None, sm_scale=None,
                       workspace=None, err_word=None) -> torch.Tensor:
    """kvq_decode_attn_varlen: as decode_attn with kv_lens int32 [B] on the device."""
    if kv_lens.numel() != q.shape[0]:
        raise ValueError("kv_lens must hold one entry per batch row")
    return _decode(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_lens, out, mask, sm_scale, workspace, err_word,
                   varlen=True)


def decode_attn_block(mode: int, q, k_codes, k_scales, v_codes, v_scales, kv_len, *, out=None, mask=None,
                      sm_scale=None, workspace=None, err_word=None) -> torch.Tensor:
    """kvq_decode_attn_block: q [B, Hq, 1, D] bf16 over a per-32 block cache written by
    kvq_write mode 1..6: codes uint8 [B, Hkv, S, D] (mode 3: D/2), scales [B, Hkv, S, D/32]
    (float32 for modes 1, 4, 6, E8M0 uint8 otherwise)."""
    _cuda("q", q, torch.bfloat16)
    _block_cache_args(mode, k_codes, k_scales, v_codes, v_scales)
    _cuda("kv_len", kv_len, torch.int32)
    _cuda("mask", mask, torch.float32)
    _cuda("err_word", err_word, torch.int32)
    _on_current_device(q)
    B, Hq, Lq, D = q.shape
    Hkv, S = k_codes.shape[1], k_codes.shape[2]
    if Lq != 1:
        raise ValueError("decode takes one query row")
    if out is None:
        out = torch.empty_like(q)
    _cuda("out", out, torch.bfloat16)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if workspace is None:
        nbytes = int(load().kvq_decode_block_workspace_bytes(B, Hq, Hkv, D, S))
        with torch.cuda.device(q.device):
            workspace = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    st = load().kvq_decode_attn_block(int(mode), _ptr(q), B, Hq, Hkv, D, _ptr(k_codes), _ptr(k_scales),
                                      _ptr(v_codes), _ptr(v_scales), S, _ptr(kv_len), _ptr(mask),
                                      float(sm_scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                      _ptr(err_word), _stream(q.device))
    _check("kvq_decode_attn_block", st)
    return out


def _block_cache_args(mode, k_codes, k_scales, v_codes, v_scales):
    for n, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        _cuda(n, t, torch.uint8)
    f32 = mode in (MODE_FP8_E4M3, MODE_FP8_E5M2, MODE_INT8_SYM)
    for n, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _cuda(n, t, torch.float32 if f32 else torch.uint8)


def prefill_attn_block(mode: int, q, k_codes, k_scales, v_codes, v_scales, kv_len, *, out=None, mask=None,
                       is_causal=False, mask_is_causal=False, sm_scale=None, err_word=None) -> torch.Tensor:
    """kvq_prefill_attn_block: q [B, Hq, Lq, D] bf16 (rows at positions kv_len - Lq + i) over a
    per-32 block cache written by kvq_write mode 1..6 (layouts as for decode_attn_block)."""
    _cuda("q", q, torch.bfloat16)
    _block_cache_args(mode, k_codes, k_scales, v_codes, v_scales)
    _cuda("kv_len", kv_len, torch.int32)
    _cuda("mask", mask, torch.float32)
    _cuda("err_word", err_word, torch.int32)
    _on_current_device(q)
    B, Hq, Lq, D = q.shape
    Hkv, S = k_codes.shape[1], k_codes.shape[2]
    if out is None:
        out = torch.empty_like(q)
    _cuda("out", out, torch.bfloat16)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    st = load().kvq_prefill_attn_block(int(mode), _ptr(q), B, Hq, Hkv, Lq, D, _ptr(k_codes), _ptr(k_scales),
                                       _ptr(v_codes), _ptr(v_scales), S, _ptr(kv_len), _ptr(mask),
                                       int(bool(is_causal)), int(bool(mask_is_causal)), float(sm_scale), _ptr(out),
                                       _ptr(err_word), _stream(q.device))
    _check("kvq_prefill_attn_block", st)
    return out


def decode_attn_tq4(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, *, out=None, mask=None, sm_scale=None,
                    workspace=None, err_word=None) -> torch.Tensor:
    """kvq_decode_attn_tq4: q [B, Hq, 1, D] bf16 over the TQ4 cache: k/v uint8 nibbles
    [B, Hkv, S, D/2], scales float32 and zero points (0..15, uint8 or int8) [B, Hkv, S]."""
    for n, t in (("k", k), ("v", v)):
        _cuda(n, t, torch.uint8)
    if k.shape[-1] * 2 != q.shape[-1]:
        raise ValueError("a TQ4 cache holds D/2 bytes per slot")
    kz = k_zp.view(torch.int8) if k_zp.dtype == torch.uint8 else k_zp
    vz = v_zp.view(torch.int8) if v_zp.dtype == torch.uint8 else v_zp
    return _decode(q, k.view(torch.int8), k_scale, kz, v.view(torch.int8), v_scale, vz, kv_len, out, mask,
                   sm_scale, workspace, err_word, varlen=False, tq4=True)


def _decode(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, out, mask, sm_scale, workspace, err_word, varlen,
            tq4=False):
    if out is None:
        out = torch.empty_like(q)
    _attn_common(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, mask, out, err_word)
    B, Hq, Lq, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if Lq != 1:
        raise ValueError("decode takes one query row (use prefill_attn)")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, D, S, q.device)
    if varlen:
        name = "kvq_decode_attn_varlen"
        st = load().kvq_decode_attn_varlen(_ptr(q), B, Hq, Hkv, D, _ptr(k), _ptr(k_scale), _ptr(k_zp), _ptr(v),
                                           _ptr(v_scale), _ptr(v_zp), S, _ptr(kv_len), _ptr(mask),
                                           _mask_batch_stride(mask, B, 1, S), float(sm_scale), _ptr(out),
                                           _ptr(workspace), workspace.numel(), _ptr(err_word), _stream(q.device))
    else:
        if mask is not None and mask.numel() != S:
            raise ValueError("decode_attn takes one mask row [S] (per-row masks: decode_attn_varlen)")
        name = "kvq_decode_attn_tq4" if tq4 else "kvq_decode_attn"
        st = getattr(load(), name)(_ptr(q), B, Hq, Hkv, D, _ptr(k), _ptr(k_scale), _ptr(k_zp), _ptr(v),
                                   _ptr(v_scale), _ptr(v_zp), S, _ptr(kv_len), _ptr(mask), float(sm_scale),
                                   _ptr(out), _ptr(workspace), workspace.numel(), _ptr(err_word),
                                   _stream(q.device))
    _check(name, st)
    return out


def decode_attn_static(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, *, out=None, mask=None, sm_scale=None,
                       err_word=None) -> torch.Tensor:
    """kvq_decode_attn_static: decode attention that allocates nothing; its scratch
    is the library's own per-device buffer (for callers that cannot allocate)."""
    if out is None:
        out = torch.empty_like(q)
    _attn_common(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, mask, out, err_word)
    B, Hq, Lq, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if Lq != 1:
        raise ValueError("decode takes one query row (use prefill_attn)")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    st = load().kvq_decode_attn_static(_ptr(q), B, Hq, Hkv, D, _ptr(k), _ptr(k_scale), _ptr(k_zp), _ptr(v),
                                       _ptr(v_scale), _ptr(v_zp), S, _ptr(kv_len), _ptr(mask),
                                       float(sm_scale), _ptr(out), _ptr(err_word), _stream(q.device))
    _check("kvq_decode_attn_static", st)
    return out


def decode_static_reset(device=None):
    """kvq_decode_static_reset: zero the static decode buffer on `device` (needed only
    after a call that reported KVQ_ERR_TIMEOUT)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check("kvq_decode_static_reset", load().kvq_decode_static_reset(_stream(dev)))


def prefill_attn(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, *, out=None, mask=None, is_causal=False,
                 mask_is_causal=False, sm_scale=None, err_word=None) -> torch.Tensor:
    """kvq_prefill_attn: q [B, Hq, Lq, D] bf16 (rows at positions kv_len - Lq + i)."""
    return _prefill(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, out, mask, is_causal, mask_is_causal,
                    sm_scale, err_word, varlen=False)


def prefill_attn_varlen(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_lens, *, out=None, mask=None,
                        is_causal=False, mask_is_causal=False, sm_scale=None, err_word=None) -> torch.Tensor:
    """kvq_prefill_attn_varlen: as prefill_attn with kv_lens int32 [B] on the device."""
    if kv_lens.numel() != q.shape[0]:
        raise ValueError("kv_lens must hold one entry per batch row")
    return _prefill(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_lens, out, mask, is_causal, mask_is_causal,
                    sm_scale, err_word, varlen=True)


def _prefill(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, out, mask, is_causal, mask_is_causal, sm_scale,
             err_word, varlen):
    if out is None:
        out = torch.empty_like(q)
    _attn_common(q, k, k_scale, k_zp, v, v_scale, v_zp, kv_len, mask, out, err_word)
    B, Hq, Lq, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if varlen:
        name = "kvq_prefill_attn_varlen"
        st = load().kvq_prefill_attn_varlen(_ptr(q), B, Hq, Hkv, Lq, D, _ptr(k), _ptr(k_scale), _ptr(k_zp),
                                            _ptr(v), _ptr(v_scale), _ptr(v_zp), S, _ptr(kv_len), _ptr(mask),
                                            _mask_batch_stride(mask, B, Lq, S), int(bool(is_causal)),
                                            int(bool(mask_is_causal)), float(sm_scale), _ptr(out), _ptr(err_word),
                                            _stream(q.device))
    else:
        if mask is not None and mask.numel() != Lq * S:
            raise ValueError("prefill_attn takes one mask [Lq, S] (per-row masks: prefill_attn_varlen)")
        name = "kvq_prefill_attn"
        st = load().kvq_prefill_attn(_ptr(q), B, Hq, Hkv, Lq, D, _ptr(k), _ptr(k_scale), _ptr(k_zp), _ptr(v),
                                     _ptr(v_scale), _ptr(v_zp), S, _ptr(kv_len), _ptr(mask), int(bool(is_causal)),
                                     int(bool(mask_is_causal)), float(sm_scale), _ptr(out), _ptr(err_word),
                                     _stream(q.device))
    _check(name, st)
    return out
