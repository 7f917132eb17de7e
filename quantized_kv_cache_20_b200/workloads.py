"""Seeded synthetic inputs for the five workloads (shapes, sizes and value
distributions only; none of the quantization or attention arithmetic).

Every tensor is drawn on the CPU from a ``torch.Generator`` with a fixed seed,
so the CUDA library and the CPU oracle can be fed bit-identical inputs.  bf16
activations are fp32 N(0, 1) draws rounded to nearest-even by ``.to(bfloat16)``.

Workloads (sizes follow the configurations the pages' workloads imply):
  tiny   -- 16 tokens x 2 kv heads x D=64 into a 64-slot cache, 3 skipped slots;
            decode with 4 q heads (GQA 2:1) at kv_len 40.
  decode -- batch 8, 32 q / 8 kv heads, D=128, 8192 slots, 4096 filled;
            one token written per step, then decode attention at kv_len 4096.
  sink   -- batch 1, 32 q / 8 kv heads, D=128, 4 sink + 2044 ring slots,
            positions 0..10000 (decode) and 128-token prefill chunks.
  block  -- x [16384, 512] with 1% of elements x10, 65536 slots, 10% skipped;
            FP8 E4M3 / MX-FP8 / MX-FP4 block writes.
  long   -- batch 1, 32 q / 16 kv heads, D=256, 131072 slots; 2048-token
            causal prefill chunk at kv_len 131072, then decode.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    S: int
    kv_len: int = 0
    T: int = 1
    sink: int = 0
    Lq: int = 1


TINY = Workload("tiny", seed=0, B=1, Hq=4, Hkv=2, D=64, S=64, kv_len=40, T=16)
DECODE = Workload("decode", seed=1, B=8, Hq=32, Hkv=8, D=128, S=8192, kv_len=4096, T=1)
SINK = Workload("sink", seed=2, B=1, Hq=32, Hkv=8, D=128, S=2048, T=1, sink=4, Lq=128)
LONG = Workload("long", seed=4, B=1, Hq=32, Hkv=16, D=256, S=131072, kv_len=131072, T=2048, Lq=2048)


@dataclass(frozen=True)
class BlockWorkload:
    name: str
    seed: int
    tokens: int
    d: int
    num_slots: int
    skip_frac: float
    outlier_p: float
    outlier_scale: float


BLOCK = BlockWorkload("block", seed=3, tokens=16384, d=512, num_slots=65536, skip_frac=0.10,
                      outlier_p=0.01, outlier_scale=10.0)

WORKLOADS = {w.name: w for w in (TINY, DECODE, SINK, LONG)}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def bf16_normal(shape, gen: torch.Generator, outlier_p: float = 0.0,
                outlier_scale: float = 1.0) -> torch.Tensor:
    """fp32 N(0,1) draws, optionally scaled by ``outlier_scale`` with probability
    ``outlier_p`` (seeded Bernoulli), rounded to bf16."""
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if outlier_p > 0:
        hit = torch.rand(shape, generator=gen) < outlier_p
        x = torch.where(hit, x * outlier_scale, x)
    return x.to(torch.bfloat16)


def slot_mapping_random(tokens: int, num_slots: int, n_skip: int, gen: torch.Generator) -> torch.Tensor:
    """``tokens`` distinct slots drawn without replacement from [0, num_slots),
    then ``n_skip`` of them (chosen at random) replaced by -1."""
    sm = torch.randperm(num_slots, generator=gen)[:tokens].to(torch.int32)
    if n_skip:
        idx = torch.randperm(tokens, generator=gen)[:n_skip]
        sm[idx] = -1
    return sm


def int8_cache_random(B: int, H: int, S: int, D: int, gen: torch.Generator):
    """Arbitrary cache contents (uniform codes, scales U(0.01, 0.1), zero points
    uniform over int8), used as a pre-fill so untouched slots have content."""
    codes = torch.randint(-128, 128, (B, H, S, D), generator=gen, dtype=torch.int8)
    scales = torch.rand((B, H, S), generator=gen) * 0.09 + 0.01
    zps = torch.randint(-128, 128, (B, H, S), generator=gen, dtype=torch.int8)
    return codes, scales, zps


def int8_cache_like(B: int, H: int, S: int, D: int, gen: torch.Generator):
    """Cache contents shaped like a quantized N(0,1) cache: codes ~ round(N(0,1) * 42)
    clipped to int8, zero points in [-6, 6], scales U(0.018, 0.030), so the
    dequantized values are O(1) and attention scores are well spread."""
    codes = (torch.randn((B, H, S, D), generator=gen) * 42.0).round().clamp_(-128, 127).to(torch.int8)
    zps = torch.randint(-6, 7, (B, H, S), generator=gen, dtype=torch.int8)
    scales = torch.rand((B, H, S), generator=gen) * 0.012 + 0.018
    return codes, scales, zps


def block_cache_random(B: int, H: int, S: int, d: int, mode: int, gen: torch.Generator):
    """Arbitrary pre-fill for a block-mode cache: random code bytes and either
    float32 scales U(0.01, 0.1) (modes 1, 4, 6) or random E8M0 bytes in [100, 140]."""
    row = d // 2 if mode == 3 else d
    codes = torch.randint(0, 256, (B, H, S, row), generator=gen, dtype=torch.uint8)
    if mode in (1, 4, 6):
        scales = torch.rand((B, H, S, d // 32), generator=gen) * 0.09 + 0.01
    else:
        scales = torch.randint(100, 141, (B, H, S, d // 32), generator=gen, dtype=torch.uint8)
    return codes, scales


def int4_cache_random(B: int, H: int, S: int, D: int, gen: torch.Generator):
    """Arbitrary pre-fill / content for a TQ4 (4-bit, nibble-packed) cache: random
    code bytes [B, H, S, D/2], scales U(0.3, 0.5), zero points in [5, 10]."""
    codes = torch.randint(0, 256, (B, H, S, D // 2), generator=gen, dtype=torch.uint8)
    scales = torch.rand((B, H, S), generator=gen) * 0.2 + 0.3
    zps = torch.randint(5, 11, (B, H, S), generator=gen, dtype=torch.int8)
    return codes, scales, zps


def u16(t: torch.Tensor):
    """Raw bit patterns of a CPU bf16 tensor as a numpy uint16 array."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
