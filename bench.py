"""Benchmark of the quantized KV-cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

A step is one decode step of the `decode` workload on one GPU: write one new
token's K and V (int8 affine per token and head) for batch 8 x 8 kv heads into
slot 4095, then run decode attention for 32 q heads at kv_len 4096 (read from
device memory) over the 8192-slot cache.  Eight independent layer caches are
rotated step by step, so each step reads a cache that is not in L2 (8 x 66.6
MiB > 126 MB).  Steps are replayed from CUDA graphs.  With N > 1 (torchrun),
every rank runs its own replica (weak scaling, no collective on the data path);
the time is the max over ranks.

Printed (rank 0): one JSON line with the headline metric (tokens/s), the
roofline of the dominant kernel (decode attention, HBM-bound), the end-to-end
number through the Python binding with host buffers, the CPU oracle baseline
(all host cores, and one core), the GPU clocks (sampled from the warm-up to the
end of the detail workloads, and read just before and after the timed region),
and per-kernel detail lines for the bulk fill write, the block-quantized writes,
the long-context decode, and the chunked prefills on the tensor cores, with
bounded oracle timings beside some of them.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KV-write GB/s + int8-KV decode attn tokens/s, % of B200 HBM roofline"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one decode_kernel launch on
# the decode workload, from one ncu capture, and the SHA-256 of the decode source it was
# taken on: the line reports the figure only while the source is unchanged (else null).
DECODE_TRAFFIC_BYTES = 70691328  # 69,872,384 read + 818,944 written; algorithmic 69,861,376
DECODE_TRAFFIC_SRC_SHA256 = "07319a2aab83d131daf76006a29d6c7d5a2d2a9e02764c2c769c529e1ed9ae82"
DECODE_SRC = ("quantized_kv_cache_20_b200/csrc/kvq_decode.cu", "quantized_kv_cache_20_b200/csrc/kvq_decode_kernel.cuh",
              "quantized_kv_cache_20_b200/csrc/kvq_common.cuh")


def decode_source_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in DECODE_SRC:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=65536)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--no-detail", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--kernel", choices=["decode", "fill", "block1", "block2", "block3", "long_decode",
                                         "long_prefill", "sink_prefill"],
                    help="profiling aid: launch only this kernel on its workload --steps times, print nothing")
    ap.add_argument("--kv-len", type=int, default=0,
                    help="with --kernel long_prefill: cache length and kv_len (default: the full 131072)")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (kernels here are timed alone)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def causal_prefill_flops(Hq, D, Lq, kv_len):
    """Algorithmic FLOPs of a causal chunk: 2 D (q.k) + 2 D (p.v) per visible (row, key) pair;
    row i sees kv_len - Lq + i + 1 keys."""
    pairs = Lq * (kv_len - Lq) + Lq * (Lq + 1) // 2
    return 4 * D * Hq * pairs


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 200 ms) of this GPU's SM clock and throttle reasons."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def once(self):
        """One reading: {sm_mhz, sm_max_mhz, reasons} (None fields when nvidia-smi is missing)."""
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                  "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                 timeout=10).stdout
        except Exception:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        r = self._parse(out)
        return {"sm_mhz": r["sm_mhz"], "sm_max_mhz": r["sm_max_mhz"], "reasons": r["reasons"]}

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return self._parse(out)

    @staticmethod
    def _parse(out):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- dist
class Dist:
    def __init__(self, n_req: int):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if n_req != self.world and self.world != 1:
            raise SystemExit(f"--gpus {n_req} but WORLD_SIZE={self.world}")
        self.torch = torch
        self.device = None
        self.pg = False

    def setup_cuda(self):
        torch = self.torch
        self.device = torch.device("cuda", self.local)
        torch.cuda.set_device(self.device)
        if self.world > 1:
            import torch.distributed as td
            td.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=self.device)
            self.pg = True

    def setup_cpu(self):
        if self.world > 1:
            import torch.distributed as td
            td.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as td
            if self.device is not None:
                td.barrier(device_ids=[self.local])
            else:
                td.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch.distributed as td
        t = self.torch.tensor([x], dtype=self.torch.float64, device=self.device or "cpu")
        td.all_reduce(t, op=td.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as td
            td.destroy_process_group()


# ---------------------------------------------------------------------------- CPU oracle
def _oracle_decode_steps(seconds: float, min_steps: int = 1, max_steps: int | None = None,
                         rows_per_step: int | None = None):
    """Time the CPU oracle on the decode workload.  A step writes one token's K
    and V (64 rows each) and computes `rows_per_step` of the 256 (b, h)
    attention rows at kv_len 4096 (all of them by default; a sample cycles
    through the rows).  Returns (steps, seconds, full_step_seconds): the last
    is the time a step with all 256 rows takes, estimated from the sample."""
    import numpy as np
    import oracle
    from quantized_kv_cache_20_b200 import workloads as wl

    w = wl.DECODE
    g = wl.generator(w.seed)
    S = w.kv_len  # only the first kv_len slots take part in a step
    K = [t.numpy().copy() for t in wl.int8_cache_like(w.B, w.Hkv, S, w.D, g)]
    V = [t.numpy().copy() for t in wl.int8_cache_like(w.B, w.Hkv, S, w.D, g)]
    k = wl.u16(wl.bf16_normal((w.B, w.Hkv, 1, w.D), g))
    v = wl.u16(wl.bf16_normal((w.B, w.Hkv, 1, w.D), g))
    q = wl.u16(wl.bf16_normal((w.B, w.Hq, 1, w.D), g))
    sm = np.full(w.B, S - 1, np.int32)
    rows = [(b, h, 0) for b in range(w.B) for h in range(w.Hq)]
    r = len(rows) if rows_per_step is None else max(1, min(len(rows), rows_per_step))
    oracle.build()
    steps, t_write, t_attn = 0, 0.0, 0.0
    t0 = time.perf_counter()
    while True:
        ta = time.perf_counter()
        oracle.write(0, k, sm, S, *K)
        oracle.write(0, v, sm, S, *V)
        tb = time.perf_counter()
        if r == len(rows):
            oracle.sdpa(q, *K, *V, kv_len=w.kv_len, sm_scale=1 / math.sqrt(w.D))
        else:
            sel = [rows[(steps * r + j) % len(rows)] for j in range(r)]
            oracle.sdpa_rows(q, *K, *V, kv_len=w.kv_len, sm_scale=1 / math.sqrt(w.D), rows=sel)
        tc = time.perf_counter()
        t_write += tb - ta
        t_attn += tc - tb
        steps += 1
        el = tc - t0
        if (steps >= min_steps and el >= seconds) or (max_steps is not None and steps >= max_steps):
            break
    full = (t_write + t_attn * len(rows) / r) / steps
    return steps, el, full


def _oracle_decode_steps_threads(seconds: float, cores: int, min_steps: int = 1, max_steps: int | None = None,
                                 rows_per_step: int | None = None):
    """The decode workload's steps on the CPU oracle, called unchanged from `cores`
    threads (ctypes releases the GIL inside each call): the write of the step's 64 K
    and 64 V rows split by batch row, the attention rows by row.  A step computes
    `rows_per_step` of the 256 (b, h) rows (all by default; a sample cycles through
    them).  Returns (steps, seconds, full_step_seconds), the last estimated from the
    sample as for _oracle_decode_steps."""
    import concurrent.futures as cf
    import numpy as np
    import oracle
    from quantized_kv_cache_20_b200 import workloads as wl

    w = wl.DECODE
    g = wl.generator(w.seed)
    S = w.kv_len
    K = [t.numpy().copy() for t in wl.int8_cache_like(w.B, w.Hkv, S, w.D, g)]
    V = [t.numpy().copy() for t in wl.int8_cache_like(w.B, w.Hkv, S, w.D, g)]
    k = wl.u16(wl.bf16_normal((w.B, w.Hkv, 1, w.D), g))
    v = wl.u16(wl.bf16_normal((w.B, w.Hkv, 1, w.D), g))
    q = wl.u16(wl.bf16_normal((w.B, w.Hq, 1, w.D), g))
    sm = np.full(1, S - 1, np.int32)
    rows = [(b, h, 0) for b in range(w.B) for h in range(w.Hq)]
    r = len(rows) if rows_per_step is None else max(1, min(len(rows), rows_per_step))
    oracle.build()

    def write_row(b):  # batch row b's token, into batch row b of the caches
        oracle.write(0, k[b:b + 1], sm, S, *[t[b:b + 1] for t in K])
        oracle.write(0, v[b:b + 1], sm, S, *[t[b:b + 1] for t in V])

    def attend(part):
        if part:
            oracle.sdpa_rows(q, *K, *V, kv_len=w.kv_len, sm_scale=1 / math.sqrt(w.D), rows=part)

    steps, t_write, t_attn = 0, 0.0, 0.0
    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        t0 = time.perf_counter()
        while True:
            ta = time.perf_counter()
            list(ex.map(write_row, range(w.B)))
            tb = time.perf_counter()
            sel = rows if r == len(rows) else [rows[(steps * r + j) % len(rows)] for j in range(r)]
            list(ex.map(attend, [sel[i::cores] for i in range(cores)]))
            tc = time.perf_counter()
            t_write += tb - ta
            t_attn += tc - tb
            steps += 1
            el = tc - t0
            if (steps >= min_steps and el >= seconds) or (max_steps is not None and steps >= max_steps):
                break
    full = (t_write + t_attn * len(rows) / r) / steps
    return steps, el, full


def _cpu_detail(detail, cores):
    """Bounded oracle timings beside the detail lines, on all host cores (the
    unchanged C oracle from `cores` threads over independent tokens / rows)."""
    import concurrent.futures as cf
    import numpy as np
    import oracle
    from quantized_kv_cache_20_b200 import workloads as wl

    def timed(fn, units, scale, label):
        t0 = time.perf_counter()
        with cf.ThreadPoolExecutor(max_workers=cores) as ex:
            list(ex.map(fn, units))
        el = time.perf_counter() - t0
        return {"kind": "oracle", "cores": cores, "sample": label, "sample_s": el, "us_full": 1e6 * el * scale}

    # int8 fill write: 8 x 8 heads x 4095 tokens; sample: batch row 0 (1/8), split by head
    w = wl.DECODE
    g = wl.generator(11)
    x = wl.u16(wl.bf16_normal((1, w.Hkv, w.kv_len - 1, w.D), g))
    Kc = [np.zeros((1, w.Hkv, w.kv_len, w.D), np.int8), np.zeros((1, w.Hkv, w.kv_len), np.float32),
          np.zeros((1, w.Hkv, w.kv_len), np.int8)]
    sm = np.arange(w.kv_len - 1, dtype=np.int32)

    def fill_head(h):
        oracle.write(0, x[:, h:h + 1], sm, w.kv_len, *[t[:, h:h + 1] for t in Kc])
    if "int8_fill_write" in detail:
        c = timed(fill_head, range(w.Hkv), 8 * 2, "K of batch row 0 (1/16 of the fill: 8 heads x 4095 tokens)")
        c["GB/s"] = detail["int8_fill_write"]["bytes"] / (c["us_full"] / 1e6) / 1e9
        detail["int8_fill_write"]["cpu"] = c
    # block writes: x [16384, 512]; sample 2048 tokens, split in chunks of 128
    bw = wl.BLOCK
    xb = wl.u16(wl.bf16_normal((1, 1, 2048, bw.d), g, outlier_p=bw.outlier_p, outlier_scale=bw.outlier_scale))
    for mode, name in ((1, "fp8_e4m3"), (2, "mxfp8"), (3, "mxfp4")):
        key = f"block_write_{name}"
        if key not in detail:
            continue
        row = bw.d // 2 if mode == 3 else bw.d
        codes = np.zeros((1, 1, 2048, row), np.uint8)
        scales = np.zeros((1, 1, 2048, bw.d // 32), np.float32 if mode == 1 else np.uint8)

        def blk(i, mode=mode, codes=codes, scales=scales):
            sl = slice(128 * i, 128 * i + 128)
            oracle.write(mode, xb[:, :, sl], np.arange(128, dtype=np.int32), 128, codes[:, :, sl], scales[:, :, sl])
        c = timed(blk, range(16), bw.tokens / 2048, "2048 of the 16384 tokens (no skipped rows), scaled")
        c["GB/s"] = detail[key]["bytes"] / (c["us_full"] / 1e6) / 1e9
        detail[key]["cpu"] = c
    # long prefill: 64 rows of the 2048-row causal chunk (the first and the last row of every
    # 128-row tile, over the heads), fp64 over a 131072-slot cache, scaled to 2048 x 32 rows
    if "long_prefill" in detail:
        lw = wl.LONG
        Hk = 1  # one kv head's cache holds the sample's rows (the cost per row does not depend on the head)
        Kl = [t.numpy() for t in wl.int8_cache_like(1, Hk, lw.kv_len, lw.D, g)]
        Vl = [t.numpy() for t in wl.int8_cache_like(1, Hk, lw.kv_len, lw.D, g)]
        ql = wl.u16(wl.bf16_normal((1, 2, lw.Lq, lw.D), g))
        rows = [(0, e % 2, 128 * t + 127 * e) for t in range(lw.Lq // 128) for e in (0, 1)]
        rows += [(0, 1, 64 * t + 63) for t in range(32)]  # 64 rows in all
        rows = rows[:64]

        def att(r):
            oracle.sdpa_rows(ql, *Kl, *Vl, kv_len=lw.kv_len, sm_scale=1 / math.sqrt(lw.D), rows=[r], is_causal=True)
        c = timed(att, rows, lw.Lq * lw.Hq / len(rows), "64 rows of the causal chunk (first and last row of every "
                                                         "128-row tile), scaled to the 2048 x 32 rows")
        c["TFLOP/s"] = detail["long_prefill"]["flops"] / (c["us_full"] / 1e6) / 1e12
        detail["long_prefill"]["cpu"] = c


REFERENCE_BUDGET_S = 120.0  # the timed part of --impl reference stays near this


def run_reference(args, dist: Dist):
    """The oracle arm: rank 0 alone times the C oracle on the host cores (other
    ranks exit at once).  Each step attends a bounded sample of the 256 rows,
    sized so that --steps K stays within about REFERENCE_BUDGET_S seconds; the
    metric is scaled to full steps."""
    if dist.rank != 0:
        return
    from quantized_kv_cache_20_b200 import workloads as wl
    w = wl.DECODE
    cores = _cpu_cores()
    _, _, full = _oracle_decode_steps_threads(0.0, cores, min_steps=1, max_steps=1)  # calibration (and build)
    rows_total = w.B * w.Hq
    per_row = full / rows_total
    r = int(max(1, min(rows_total, REFERENCE_BUDGET_S / max(1, args.steps) / per_row)))
    _oracle_decode_steps_threads(0.0, cores, min_steps=args.warmup, max_steps=args.warmup, rows_per_step=r)
    steps, el, full = _oracle_decode_steps_threads(0.0, cores, min_steps=args.steps, max_steps=args.steps,
                                                   rows_per_step=r)
    value = w.B / full
    sample = (f"{steps} decode steps, each writing 1 token K/V for 8x8 rows and computing {r} of the 256 "
              f"attention rows at kv_len 4096 (rows cycle); tokens/s scaled to full 256-row steps; the unchanged "
              f"C oracle called from {cores} threads, {el:.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * full,
        "measured_ms_per_sampled_step": 1000 * el / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": _config(args),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(args):
    return {
        "workload": "decode step: batch 8, 32 q / 8 kv heads (GQA 4:1), D=128, int8 per-token-head KV cache of "
                    "8192 slots with 4096 filled; write 1 token K/V then decode attention at kv_len 4096 "
                    "read on device",
        "global_batch": 8 * args.gpus,
        "seq_len": 4096,
        "l2": f"{args.layers} independent layer caches rotated per step ({args.layers} x 66.6 MiB read > 126 MB L2)",
        "graphs": "each step replayed from a CUDA graph",
        "parallelism": f"replicas x{args.gpus} (weak scaling, no collective on the data path)",
    }


# ---------------------------------------------------------------------------- GPU arm
def run_kvq(args, dist: Dist):
    import torch
    from quantized_kv_cache_20_b200 import build as kbuild
    from quantized_kv_cache_20_b200 import kvq
    from quantized_kv_cache_20_b200 import workloads as wl

    dist.setup_cuda()
    if dist.local == 0:
        kbuild.build()
    dist.barrier()
    kvq.load()
    dev = dist.device
    w = wl.DECODE
    B, Hq, Hkv, D, S, KV = w.B, w.Hq, w.Hkv, w.D, w.S, w.kv_len
    NL = args.layers
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + dist.rank)

    # ---- caches, filled by the write kernel (positions 0..4094, slot = position)
    Tf = KV - 1
    xk = torch.randn((B, Hkv, Tf, D), generator=gen, device=dev).to(torch.bfloat16)
    xv = torch.randn((B, Hkv, Tf, D), generator=gen, device=dev).to(torch.bfloat16)
    sm_fill = torch.arange(Tf, dtype=torch.int32, device=dev).repeat(B)
    layers = []
    for _ in range(NL):
        K = (torch.empty((B, Hkv, S, D), dtype=torch.int8, device=dev),
             torch.empty((B, Hkv, S), dtype=torch.float32, device=dev),
             torch.empty((B, Hkv, S), dtype=torch.int8, device=dev))
        V = (torch.empty_like(K[0]), torch.empty_like(K[1]), torch.empty_like(K[2]))
        kvq.write(0, xk, sm_fill, *K)
        kvq.write(0, xv, sm_fill, *V)
        layers.append((K, V))
    q = torch.randn((B, Hq, 1, D), generator=gen, device=dev).to(torch.bfloat16)
    kn = torch.randn((B, Hkv, 1, D), generator=gen, device=dev).to(torch.bfloat16)
    vn = torch.randn((B, Hkv, 1, D), generator=gen, device=dev).to(torch.bfloat16)
    sm_step = torch.full((B,), KV - 1, dtype=torch.int32, device=dev)
    kv_len = torch.tensor([KV], dtype=torch.int32, device=dev)
    out = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device=dev)
    ws = kvq.decode_workspace(B, Hq, Hkv, D, S, dev)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)

    def step(l):
        K, V = layers[l]
        kvq.write_kv(0, kn, vn, sm_step, K, V)
        kvq.decode_attn(q, *K, *V, kv_len, out=out, workspace=ws)

    def decode_only(l):
        K, V = layers[l]
        kvq.decode_attn(q, *K, *V, kv_len, out=out, workspace=ws)

    # warm the launch path once outside capture, then capture one graph per rotation
    # (NL steps, one per layer) and one of decode launches alone
    with torch.cuda.stream(stream):
        for l in range(NL):
            step(l)
    torch.cuda.synchronize()
    rot_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(rot_graph, stream=stream):
        for l in range(NL):
            step(l)
    dec_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(dec_graph, stream=stream):
        for l in range(NL):
            decode_only(l)
    step_graphs = []
    for l in range(NL):
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph, stream=stream):
            step(l)
        step_graphs.append(gph)
    torch.cuda.synchronize()

    # ---- headline: exactly K steps (whole rotations, then single steps).  nvidia-smi
    # samples every 200 ms from here to the end of the detail workloads (a timed region
    # of a few ms would see no sample), plus one reading right before and after it.
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    reps, rem = divmod(args.steps, NL)
    nsteps = args.steps
    with torch.cuda.stream(stream):
        for i in range(max(1, (args.warmup + NL - 1) // NL)):
            rot_graph.replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    clk_before = clocks.once()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(reps):
            rot_graph.replay()
        for l in range(rem):
            step_graphs[l].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    clk_after = clocks.once()
    dist.barrier()
    ms_local = e0.elapsed_time(e1) / nsteps
    ms = dist.max(ms_local)
    value = dist.world * B / (ms / 1000.0)

    # ---- dominant kernel: decode attention alone, same rotation, events on its stream
    dreps = max(4, reps // 4)
    with torch.cuda.stream(stream):
        dec_graph.replay()
        e0.record(stream)
        for r in range(dreps):
            dec_graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    dec_ms = e0.elapsed_time(e1) / (dreps * NL)
    dec_bytes = 2 * B * Hkv * KV * (D + 4 + 1) + 2 * (B * Hq * D * 2)
    peak, peak_kind = _peaks()
    achieved = dec_bytes / (dec_ms / 1000.0) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS, "peak_kind": peak_kind,
                "kernel": "decode_kernel (split-K int8 decode attention)", "bytes_per_launch": dec_bytes,
                "launch_us": dec_ms * 1000.0}
    same_src = DECODE_TRAFFIC_BYTES is not None and decode_source_sha256() == DECODE_TRAFFIC_SRC_SHA256
    roofline["traffic"] = DECODE_TRAFFIC_BYTES if same_src else None
    roofline["traffic_source"] = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one decode_kernel launch "
                                  "on this workload, captured on the current decode source" if same_src else
                                  "null: the decode source changed since the last ncu capture")

    # ---- end to end through the binding with host buffers
    e2e = _e2e(args, dist, kvq, layers, ws, kv_len, sm_step)

    detail = {}
    if not args.no_detail:
        detail = _detail(args, dist, kvq, wl, layers, xk, xv, sm_fill, stream, peak)
    clk = clocks.stop()
    clk["window"] = ("200 ms samples from the warm-up of the timed steps to the end of the detail workloads "
                     "(continuous GPU load); at_timed_start / at_timed_end bracket the timed region")
    clk["at_timed_start"] = clk_before
    clk["at_timed_end"] = clk_after

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8 x s8 -> s32 (q.K), f16 x f16 -> f32 (P.V), f32 softmax",
        "data": "synthetic", "config": _config(args),
        "roofline": roofline, "e2e": e2e, "gpu_launches": 2 * nsteps, "clocks": clk, "detail": detail,
    }
    if dist.rank == 0 and dist.world == 1:
        cores = _cpu_cores()
        steps_n, el_n, _ = _oracle_decode_steps_threads(args.cpu_seconds, cores)
        line["cpu_baseline"] = {
            "value": B * steps_n / el_n, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{steps_n} full decode steps of the same workload (write 1 token K/V for 8x8 rows + 256 "
                      f"attention rows at kv_len 4096), the unchanged C oracle called from {cores} threads "
                      f"(writes split by token, attention by row), {el_n:.1f} s"}
        steps_c, el_c, _ = _oracle_decode_steps(args.cpu_seconds / 2)
        line["cpu_baseline_1core"] = {
            "value": B * steps_c / el_c, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{steps_c} full decode steps, single-threaded C oracle, {el_c:.1f} s"}
        if detail:
            _cpu_detail(detail, cores)
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    del rot_graph, dec_graph, step_graphs
    dist.close()


def _e2e(args, dist, kvq, layers, ws, kv_len, sm_step):
    import torch
    from quantized_kv_cache_20_b200 import workloads as wl
    w = wl.DECODE
    B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.D
    dev = dist.device
    NL = len(layers)
    steps = max(NL, min(args.steps, 2000))
    g = torch.Generator().manual_seed(7)
    # the step's inputs q, k, v in one pinned host buffer, copied in with one transfer
    nq, nk = B * Hq * D, B * Hkv * D
    hin = torch.randn((nq + 2 * nk,), generator=g).to(torch.bfloat16).pin_memory()
    hout = torch.empty((steps, B, Hq, 1, D), dtype=torch.bfloat16).pin_memory()
    din = torch.empty_like(hin, device=dev)
    dq = din[:nq].view(B, Hq, 1, D)
    dk = din[nq:nq + nk].view(B, Hkv, 1, D)
    dv = din[nq + nk:].view(B, Hkv, 1, D)
    dout = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device=dev)

    def one(i):
        K, V = layers[i % NL]
        din.copy_(hin, non_blocking=True)
        kvq.write_kv(0, dk, dv, sm_step, K, V)
        kvq.decode_attn(dq, *K, *V, kv_len, out=dout, workspace=ws)
        hout[i].copy_(dout, non_blocking=True)

    for i in range(min(NL, steps)):
        one(i)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        one(i)
    e1.record()
    torch.cuda.synchronize()
    ms = dist.max(e0.elapsed_time(e1) / steps)
    h2d = hin.numel() * 2
    return {"value": dist.world * B / (ms / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": dout.numel() * 2, "ms_per_step": ms, "steps": steps,
            "path": "pinned host -> device copy of q, k, v (one buffer), kvq.write_kv + kvq.decode_attn via the Python binding "
                    "(no graph), device -> pinned host copy of the output"}


def _time_graph(stream, fn, reps):
    """Capture fn() into a graph, replay reps times; return mean ms per replay."""
    import torch
    with torch.cuda.stream(stream):
        fn()
    torch.cuda.synchronize()
    gph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gph, stream=stream):
        fn()
    with torch.cuda.stream(stream):
        gph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            gph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del gph
    return ms


def _detail(args, dist, kvq, wl, layers, xk, xv, sm_fill, stream, peak):
    import torch
    dev = dist.device
    res = {}
    # bulk fill write (decode workload): positions 0..4094 of K and V, rotated over the layers
    w = wl.DECODE
    NL = len(layers)
    Tf = xk.shape[2]

    def fill():
        for K, V in layers:
            kvq.write(0, xk, sm_fill, *K)
            kvq.write(0, xv, sm_fill, *V)
    ms = _time_graph(stream, fill, 3) / (2 * NL)
    rows = w.B * w.Hkv * Tf
    fbytes = rows * w.D * 2 + rows * w.D + rows * 5 + w.B * Tf * 4
    res["int8_fill_write"] = {"what": "kvq_write int8, 8x8 heads x 4095 tokens, D=128", "us": ms * 1000,
                              "GB/s": fbytes / (ms / 1000) / 1e9, "frac": fbytes / (ms / 1000) / 1e9 / peak,
                              "bytes": fbytes}
    # block writes: x [16384, 512], 65536 slots, 10% skipped; 6 rotated input/cache sets (> L2)
    bw = wl.BLOCK
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    NB = 6
    sets = []
    for i in range(NB):
        x = torch.randn((1, 1, bw.tokens, bw.d), generator=g, device=dev)
        hit = torch.rand(x.shape, generator=g, device=dev) < bw.outlier_p
        x = torch.where(hit, x * bw.outlier_scale, x).to(torch.bfloat16)
        sm = torch.randperm(bw.num_slots, generator=g, device=dev)[: bw.tokens].to(torch.int32)
        sm[torch.randperm(bw.tokens, generator=g, device=dev)[: int(bw.tokens * bw.skip_frac)]] = -1
        sets.append((x, sm))
    valid = bw.tokens - int(bw.tokens * bw.skip_frac)
    for mode, name, rs in ((1, "fp8_e4m3", True), (2, "mxfp8", True), (3, "mxfp4", True),
                           (4, "fp8_e5m2", True), (5, "mxfp8_e5m2", True), (6, "int8_sym", True),
                           (2, "mxfp8_unrounded_scale", False)):
        code_row = bw.d // 2 if mode == 3 else bw.d
        f32 = mode in (1, 4, 6)
        caches = []
        for i in range(NB):
            c = torch.zeros((1, 1, bw.num_slots, code_row), dtype=torch.uint8, device=dev)
            s = torch.zeros((1, 1, bw.num_slots, bw.d // 32), dtype=torch.float32 if f32 else torch.uint8,
                            device=dev)
            caches.append((c, s))

        def blk():
            for (x, sm), (c, s) in zip(sets, caches):
                kvq.write(mode, x, sm, c, s, round_scale=rs)
        ms = _time_graph(stream, blk, 10) / NB
        sbytes = (bw.d // 32) * (4 if f32 else 1)
        byts = valid * (bw.d * 2 + code_row + sbytes) + bw.tokens * 4
        res[f"block_write_{name}"] = {"what": f"kvq_write mode {mode} (round_scale={int(rs)}), x [16384, 512], "
                                              f"10% skipped", "us": ms * 1000, "GB/s": byts / (ms / 1000) / 1e9,
                                      "frac": byts / (ms / 1000) / 1e9 / peak, "bytes": byts}
        del caches
    del sets
    torch.cuda.empty_cache()
    # TQ4 cache (4-bit affine, two codes per byte) at the decode workload's shape: fill, then decode
    tq = []
    for _ in range(NL):
        Kq = (torch.empty((w.B, w.Hkv, w.S, w.D // 2), dtype=torch.uint8, device=dev),
              torch.empty((w.B, w.Hkv, w.S), dtype=torch.float32, device=dev),
              torch.empty((w.B, w.Hkv, w.S), dtype=torch.int8, device=dev))
        Vq = tuple(torch.empty_like(t) for t in Kq)
        tq.append((Kq, Vq))

    def tq4_fill():
        for Kq, Vq in tq:
            kvq.write(7, xk, sm_fill, *Kq)
            kvq.write(7, xv, sm_fill, *Vq)
    ms = _time_graph(stream, tq4_fill, 3) / (2 * NL)
    qbytes = rows * w.D * 2 + rows * w.D // 2 + rows * 5 + w.B * Tf * 4
    res["tq4_fill_write"] = {"what": "kvq_write mode 7 (TQ4), 8x8 heads x 4095 tokens, D=128", "us": ms * 1000,
                             "GB/s": qbytes / (ms / 1000) / 1e9, "frac": qbytes / (ms / 1000) / 1e9 / peak,
                             "bytes": qbytes}
    kvl4 = torch.tensor([w.kv_len], dtype=torch.int32, device=dev)
    qq = torch.randn((w.B, w.Hq, 1, w.D), device=dev).to(torch.bfloat16)
    oq = torch.empty_like(qq)
    wsq = kvq.decode_workspace(w.B, w.Hq, w.Hkv, w.D, w.S, dev)

    def tq4_dec():
        for Kq, Vq in tq:
            kvq.decode_attn_tq4(qq, *Kq, *Vq, kvl4, out=oq, workspace=wsq)
    ms = _time_graph(stream, tq4_dec, 20) / NL
    dbytes = 2 * w.B * w.Hkv * w.kv_len * (w.D // 2 + 5) + 2 * w.B * w.Hq * w.D * 2
    res["tq4_decode"] = {"what": "kvq_decode_attn_tq4, batch 8, 32 q / 8 kv heads, D=128, kv_len 4096 (TQ4 cache)",
                         "us": ms * 1000, "tokens/s": w.B / (ms / 1000), "GB/s": dbytes / (ms / 1000) / 1e9,
                         "frac": dbytes / (ms / 1000) / 1e9 / peak, "bytes": dbytes}
    del tq, wsq
    torch.cuda.empty_cache()
    # decode over the per-32 block caches (E4M3 + f32 scale, MX-FP8, MX-FP4) at the decode workload's shape
    for mode, name in ((1, "fp8_e4m3"), (2, "mxfp8"), (3, "mxfp4")):
        row = w.D // 2 if mode == 3 else w.D
        f32 = mode == 1
        bl = []
        for _ in range(NL):
            kc = torch.empty((w.B, w.Hkv, w.S, row), dtype=torch.uint8, device=dev)
            ksc = torch.empty((w.B, w.Hkv, w.S, w.D // 32), dtype=torch.float32 if f32 else torch.uint8, device=dev)
            vc, vsc = torch.empty_like(kc), torch.empty_like(ksc)
            kvq.write(mode, xk, sm_fill, kc, ksc)
            kvq.write(mode, xv, sm_fill, vc, vsc)
            bl.append((kc, ksc, vc, vsc))
        qb = torch.randn((w.B, w.Hq, 1, w.D), device=dev).to(torch.bfloat16)
        ob = torch.empty_like(qb)
        kvb = torch.tensor([w.kv_len - 1], dtype=torch.int32, device=dev)
        wsb = torch.empty(max(16, kvq.load().kvq_decode_block_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.S)),
                          dtype=torch.uint8, device=dev)

        def bdec():
            for kc, ksc, vc, vsc in bl:
                kvq.decode_attn_block(mode, qb, kc, ksc, vc, vsc, kvb, out=ob, workspace=wsb)
        ms = _time_graph(stream, bdec, 20) / NL
        sb = (w.D // 32) * (4 if f32 else 1)
        bbytes = 2 * w.B * w.Hkv * (w.kv_len - 1) * (row + sb) + 2 * w.B * w.Hq * w.D * 2
        res[f"block_decode_{name}"] = {"what": f"kvq_decode_attn_block mode {mode}, batch 8, 32 q / 8 kv heads, "
                                               f"D=128, kv_len 4095", "us": ms * 1000, "tokens/s": w.B / (ms / 1000),
                                       "GB/s": bbytes / (ms / 1000) / 1e9,
                                       "frac": bbytes / (ms / 1000) / 1e9 / peak, "bytes": bbytes}
        del bl, wsb
    torch.cuda.empty_cache()
    # the lines below read past position 4095: fill slots 4095..8191 of every layer first
    Tr = w.S - Tf
    xkr = torch.randn((w.B, w.Hkv, Tr, w.D), device=dev).to(torch.bfloat16)
    smr_fill = (torch.arange(Tr, dtype=torch.int32, device=dev) + Tf).repeat(w.B)
    for K, V in layers:
        kvq.write(0, xkr, smr_fill, *K)
        kvq.write(0, xkr, smr_fill, *V)
    del xkr
    # ragged decode batch: the 8 rows of the decode workload at 8 different context lengths
    lens = [512, 1024, 2048, 3072, 4096, 5120, 6144, 8192]
    kvs = torch.tensor(lens, dtype=torch.int32, device=dev)
    qr = torch.randn((w.B, w.Hq, 1, w.D), device=dev).to(torch.bfloat16)
    outr = torch.empty_like(qr)
    wsr = kvq.decode_workspace(w.B, w.Hq, w.Hkv, w.D, w.S, dev)

    def rdec():
        for K, V in layers:
            kvq.decode_attn_varlen(qr, *K, *V, kvs, out=outr, workspace=wsr)
    ms = _time_graph(stream, rdec, 20) / NL
    rbytes = sum(2 * w.Hkv * n * (w.D + 5) for n in lens) + 2 * w.B * w.Hq * w.D * 2
    res["ragged_decode"] = {"what": "kvq_decode_attn_varlen, batch 8 at kv_len 512..8192 (mean 3776), 32 q / 8 kv "
                                    "heads, D=128", "us": ms * 1000, "tokens/s": w.B / (ms / 1000),
                            "GB/s": rbytes / (ms / 1000) / 1e9, "frac": rbytes / (ms / 1000) / 1e9 / peak,
                            "bytes": rbytes}
    # ring cache (sink 0) decode step at the decode workload's scale: the 8192-slot cache has wrapped
    # (position 10000); plan the slot, write K and V, build the mask, attend over all 8192 slots
    ring_pos = torch.tensor([10000], dtype=torch.int32, device=dev)
    slot_pos = torch.arange(w.S, dtype=torch.int32, device=dev) + (10000 - w.S)  # positions 1808..9999 held
    smr = torch.empty(w.B, dtype=torch.int32, device=dev)
    kvr = torch.empty(1, dtype=torch.int32, device=dev)
    maskr = torch.empty((1, w.S), dtype=torch.float32, device=dev)
    knr = torch.randn((w.B, w.Hkv, 1, w.D), device=dev).to(torch.bfloat16)
    vnr = torch.randn((w.B, w.Hkv, 1, w.D), device=dev).to(torch.bfloat16)

    def ring():
        for K, V in layers:
            kvq.sink_plan(ring_pos, w.B, 1, 0, slot_pos, smr, kvr)
            kvq.write_kv(0, knr, vnr, smr, K, V)
            kvq.sink_mask(ring_pos, 1, slot_pos, maskr)
            kvq.decode_attn(qr, *K, *V, kvr, out=outr, mask=maskr, workspace=wsr)
    ms = _time_graph(stream, ring, 20) / NL
    gbytes = 2 * w.B * w.Hkv * w.S * (w.D + 5) + w.S * 4 * 2 + 2 * w.B * w.Hq * w.D * 2
    res["ring_decode_step"] = {"what": "ring cache (sink 0, 8192 slots, wrapped): sink_plan + kvq_write_kv + "
                                       "sink_mask + kvq_decode_attn over 8192 slots, batch 8, 32 q / 8 kv heads",
                               "us": ms * 1000, "tokens/s": w.B / (ms / 1000), "GB/s": gbytes / (ms / 1000) / 1e9,
                               "frac": gbytes / (ms / 1000) / 1e9 / peak, "bytes": gbytes}
    del wsr
    # long-context decode: batch 1, 32 q / 16 kv heads, D=256, kv_len 131072 (1 GiB of codes > L2)
    lw = wl.LONG
    K = (torch.randint(-128, 128, (1, lw.Hkv, lw.S, lw.D), dtype=torch.int8, device=dev),
         torch.rand((1, lw.Hkv, lw.S), device=dev) * 0.012 + 0.018,
         torch.randint(-6, 7, (1, lw.Hkv, lw.S), dtype=torch.int8, device=dev))
    V = (torch.randint(-128, 128, (1, lw.Hkv, lw.S, lw.D), dtype=torch.int8, device=dev),
         torch.rand((1, lw.Hkv, lw.S), device=dev) * 0.012 + 0.018,
         torch.randint(-6, 7, (1, lw.Hkv, lw.S), dtype=torch.int8, device=dev))
    ql = torch.randn((1, lw.Hq, 1, lw.D), device=dev).to(torch.bfloat16)
    ol = torch.empty_like(ql)
    kvl = torch.tensor([lw.kv_len], dtype=torch.int32, device=dev)
    wsl = kvq.decode_workspace(1, lw.Hq, lw.Hkv, lw.D, lw.S, dev)

    def ldec():
        kvq.decode_attn(ql, *K, *V, kvl, out=ol, workspace=wsl)
    ms = _time_graph(stream, ldec, 20)
    lbytes = 2 * lw.Hkv * lw.kv_len * (lw.D + 5) + 2 * lw.Hq * lw.D * 2
    res["long_decode"] = {"what": "kvq_decode_attn, batch 1, 32 q / 16 kv heads, D=256, kv_len 131072",
                          "us": ms * 1000, "tokens/s": 1 / (ms / 1000), "GB/s": lbytes / (ms / 1000) / 1e9,
                          "frac": lbytes / (ms / 1000) / 1e9 / peak, "bytes": lbytes}
    # long-context chunked prefill: the last 2048-row causal chunk at kv_len 131072 (tensor cores)
    tpeak, tkind = _tensor_peak()
    qp = torch.randn((1, lw.Hq, lw.Lq, lw.D), device=dev).to(torch.bfloat16)
    op = torch.empty_like(qp)

    def lpre():
        kvq.prefill_attn(qp, *K, *V, kvl, out=op, is_causal=True, mask_is_causal=True)
    ms = _time_graph(stream, lpre, 5)
    fl = causal_prefill_flops(lw.Hq, lw.D, lw.Lq, lw.kv_len)
    res["long_prefill"] = {"what": "kvq_prefill_attn, causal chunk Lq 2048 at kv_len 131072, 32 q / 16 kv heads, "
                                   "D=256, per-tile causal bound", "us": ms * 1000,
                           "tokens/s": lw.Lq / (ms / 1000), "TFLOP/s": fl / (ms / 1000) / 1e12,
                           "frac": fl / (ms / 1000) / 1e12 / tpeak, "peak_TFLOP/s": tpeak, "peak_kind": tkind,
                           "flops": fl}
    del K, V, qp, op, wsl
    torch.cuda.empty_cache()
    # attention-sink ring: one 128-row chunk over the full 2048-slot ring with the additive mask
    sw = wl.SINK
    NS = 16  # rotated caches (16 x 4.5 MiB K/V codes) so the chunk reads cold-ish data
    rings = []
    for i in range(NS):
        Kr = (torch.randint(-128, 128, (1, sw.Hkv, sw.S, sw.D), dtype=torch.int8, device=dev),
              torch.rand((1, sw.Hkv, sw.S), device=dev) * 0.012 + 0.018,
              torch.randint(-6, 7, (1, sw.Hkv, sw.S), dtype=torch.int8, device=dev))
        Vr = tuple(t.clone() for t in Kr)
        rings.append((Kr, Vr))
    ip = torch.tensor([10000 - sw.Lq], dtype=torch.int32, device=dev)
    spos = torch.full((sw.S,), -1, dtype=torch.int32, device=dev)
    smp = torch.empty(sw.Lq, dtype=torch.int32, device=dev)
    kvs = torch.empty(1, dtype=torch.int32, device=dev)
    mask = torch.empty((sw.Lq, sw.S), dtype=torch.float32, device=dev)
    ipp = torch.zeros(1, dtype=torch.int32, device=dev)
    for p in range(0, 10000 - sw.Lq, sw.Lq):  # step the ring so slot positions wrap as in the workload
        ipp.fill_(p)
        kvq.sink_plan(ipp, 1, sw.Lq, sw.sink, spos, smp, kvs)
    kvq.sink_plan(ip, 1, sw.Lq, sw.sink, spos, smp, kvs)
    kvq.sink_mask(ip, sw.Lq, spos, mask)
    qs = torch.randn((1, sw.Hq, sw.Lq, sw.D), device=dev).to(torch.bfloat16)
    os_ = torch.empty_like(qs)

    def spre():
        for Kr, Vr in rings:
            kvq.prefill_attn(qs, *Kr, *Vr, kvs, out=os_, mask=mask)
    ms = _time_graph(stream, spre, 20) / NS
    fl = 4 * sw.D * sw.Hq * sw.Lq * sw.S
    res["sink_prefill_chunk"] = {"what": "kvq_prefill_attn, 128-row chunk at position 9872 over the 4 + 2044 ring, "
                                         "32 q / 8 kv heads, D=128, additive mask", "us": ms * 1000,
                                 "tokens/s": sw.Lq / (ms / 1000), "TFLOP/s": fl / (ms / 1000) / 1e12,
                                 "frac": fl / (ms / 1000) / 1e12 / tpeak, "flops": fl}
    del rings, mask
    torch.cuda.empty_cache()
    # chunked prefill over a per-32 block cache (MX-FP8): causal 2048-row chunk at kv_len 16384
    Hq_b, Hkv_b, D_b, S_b, Lq_b = 32, 8, 128, 16384, 2048
    cb = []
    for _ in range(2):
        xb = torch.randn((1, Hkv_b, S_b, D_b), device=dev).to(torch.bfloat16)
        c = torch.empty((1, Hkv_b, S_b, D_b), dtype=torch.uint8, device=dev)
        sc = torch.empty((1, Hkv_b, S_b, D_b // 32), dtype=torch.uint8, device=dev)
        kvq.write(2, xb, torch.arange(S_b, dtype=torch.int32, device=dev), c, sc)
        cb.append((c, sc))
        del xb
    qb = torch.randn((1, Hq_b, Lq_b, D_b), device=dev).to(torch.bfloat16)
    ob = torch.empty_like(qb)
    kvb = torch.tensor([S_b], dtype=torch.int32, device=dev)

    def bpre():
        kvq.prefill_attn_block(2, qb, *cb[0], *cb[1], kvb, out=ob, is_causal=True, mask_is_causal=True)
    ms = _time_graph(stream, bpre, 5)
    fl = causal_prefill_flops(Hq_b, D_b, Lq_b, S_b)
    res["block_prefill_mxfp8"] = {"what": "kvq_prefill_attn_block mode 2 (MX-FP8 K/V, E8M0 per 32), causal chunk "
                                          "Lq 2048 at kv_len 16384, 32 q / 8 kv heads, D=128", "us": ms * 1000,
                                  "tokens/s": Lq_b / (ms / 1000), "TFLOP/s": fl / (ms / 1000) / 1e12,
                                  "frac": fl / (ms / 1000) / 1e12 / tpeak, "flops": fl}
    del cb, qb, ob
    torch.cuda.empty_cache()
    return res


def run_kernel(args):
    """Launch one kernel on its workload --steps times (for ncu); no timing, no output."""
    import torch
    from quantized_kv_cache_20_b200 import build as kbuild
    from quantized_kv_cache_20_b200 import kvq
    from quantized_kv_cache_20_b200 import workloads as wl
    kbuild.build()
    kvq.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    if args.kernel in ("decode", "fill", "long_decode", "long_prefill", "sink_prefill"):
        w = {"decode": wl.DECODE, "fill": wl.DECODE, "sink_prefill": wl.SINK}.get(args.kernel, wl.LONG)
        B, Hq, Hkv, D, S, KV = w.B, w.Hq, w.Hkv, w.D, w.S, (w.kv_len or w.S)
        if args.kernel == "long_prefill" and args.kv_len:
            S = KV = args.kv_len
        K = (torch.randint(-128, 128, (B, Hkv, S, D), dtype=torch.int8, device=dev),
             torch.rand((B, Hkv, S), device=dev) * 0.012 + 0.018,
             torch.randint(-6, 7, (B, Hkv, S), dtype=torch.int8, device=dev))
        V = tuple(t.clone() for t in K)
        if args.kernel == "fill":
            x = torch.randn((B, Hkv, KV - 1, D), generator=g, device=dev).to(torch.bfloat16)
            sm = torch.arange(KV - 1, dtype=torch.int32, device=dev).repeat(B)
            for _ in range(args.steps):
                kvq.write(0, x, sm, *K)
        elif args.kernel.endswith("prefill"):
            q = torch.randn((B, Hq, w.Lq, D), generator=g, device=dev).to(torch.bfloat16)
            kv = torch.tensor([KV], dtype=torch.int32, device=dev)
            out = torch.empty_like(q)
            causal = args.kernel == "long_prefill"
            mask = None if causal else torch.zeros((w.Lq, S), dtype=torch.float32, device=dev)
            for _ in range(args.steps):
                kvq.prefill_attn(q, *K, *V, kv, out=out, mask=mask, is_causal=causal, mask_is_causal=causal)
        else:
            q = torch.randn((B, Hq, 1, D), generator=g, device=dev).to(torch.bfloat16)
            kv = torch.tensor([KV], dtype=torch.int32, device=dev)
            ws = kvq.decode_workspace(B, Hq, Hkv, D, S, dev)
            out = torch.empty_like(q)
            for _ in range(args.steps):
                kvq.decode_attn(q, *K, *V, kv, out=out, workspace=ws)
    else:
        mode = int(args.kernel[-1])
        bw = wl.BLOCK
        x = torch.randn((1, 1, bw.tokens, bw.d), generator=g, device=dev).to(torch.bfloat16)
        sm = torch.randperm(bw.num_slots, generator=g, device=dev)[: bw.tokens].to(torch.int32)
        sm[torch.randperm(bw.tokens, generator=g, device=dev)[: int(bw.tokens * bw.skip_frac)]] = -1
        c = torch.zeros((1, 1, bw.num_slots, bw.d // 2 if mode == 3 else bw.d), dtype=torch.uint8, device=dev)
        s = torch.zeros((1, 1, bw.num_slots, bw.d // 32), dtype=torch.float32 if mode == 1 else torch.uint8,
                        device=dev)
        for _ in range(args.steps):
            kvq.write(mode, x, sm, c, s)
    torch.cuda.synchronize()


def main():
    args = _args()
    if args.kernel:
        run_kernel(args)
        return
    dist = Dist(args.gpus)
    if args.impl == "reference":
        run_reference(args, dist)
    else:
        run_kvq(args, dist)


if __name__ == "__main__":
    main()
