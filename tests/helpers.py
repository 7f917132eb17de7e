"""Shared helpers for the GPU parity tests (inputs come from the seeded
generators; expected values come from the oracle only)."""
import math

import numpy as np
import torch

import oracle
from quantized_kv_cache_20_b200 import kvq
from quantized_kv_cache_20_b200 import workloads as wl

DEV = "cuda"

# Attention tolerance: |gpu - fp64 oracle| <= ATOL + RTOL * |oracle|.
ATOL = 2e-3
RTOL = 1e-2


def assert_attn_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} outside tolerance; worst at {i}: "
                             f"got {got[i]}, ref {ref[i]}")


def bf16_to_f64(t):
    return t.float().cpu().double().numpy()


def dev(*ts):
    return [t.to(DEV) for t in ts]


def int32_scalar(v):
    return torch.tensor([v], dtype=torch.int32, device=DEV)


def err_word():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def cache_np(c):
    return [t.cpu().numpy() for t in c]
