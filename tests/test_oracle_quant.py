"""Pins for the oracle's quantizers (CPU only).

The remaining IndexerQuantCache cache types (参数说明: FLOAT8_E5M2 and UINT8
caches, round_scale=false) follow the same formula with Q_MAX 57344 (E5M2) and
127 (symmetric int8 stored as its two's-complement byte); they are pinned the
same way.

int8 affine per token and head: ExecuTorch PR 24473, Summary (affine
asymmetric, float32 scale, int8 zero point) -- the formula is a reading, pinned
by hand-derived rows and by the dequantization error bound.
Per-32 block modes: IndexerQuantCache page, 计算公式 (scale_g = max|x_g| / Q_MAX,
q_i = round(x_i / scale_g)) and the quant_mode list -- pinned by hand-derived
groups, the scale identity and the format error bounds.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_20_b200 import workloads as wl

FLT_EPS = float(np.finfo(np.float32).eps)


def _bits(values):
    t = torch.tensor([float(v) for v in values], dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor([float(v) for v in values], dtype=torch.float32)), \
        "golden inputs must be exact in bf16"
    return wl.u16(t)


def _blocks(path):
    blocks, cur = [], {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line.startswith("#"):
                continue
            if not line:
                if cur:
                    blocks.append(cur)
                cur = {}
                continue
            k, v = line.split(":", 1)
            cur[k.strip()] = v.split()
    if cur:
        blocks.append(cur)
    return blocks


def test_affine_golden_rows(golden_dir):
    blocks = _blocks(os.path.join(golden_dir, "affine_int8_rows.txt"))
    assert len(blocks) == 5
    for b in blocks:
        q, scale, zp = oracle.affine_int8_row(_bits(b["x"]))
        assert q.tolist() == [int(v) for v in b["q"]], b
        assert float(scale) == float(np.float32(b["scale"][0]))
        assert int(zp) == int(b["zp"][0])


def _rows():
    g = wl.generator(21)
    rows = [wl.bf16_normal((64,), g) for _ in range(200)]
    rows += [wl.bf16_normal((128,), g, outlier_p=0.05, outlier_scale=30.0) for _ in range(100)]
    rows += [wl.bf16_normal((128,), g).abs() for _ in range(50)]          # all >= 0
    rows += [-wl.bf16_normal((256,), g).abs() for _ in range(50)]         # all <= 0
    rows += [wl.bf16_normal((64,), g) * 1e-6 for _ in range(20)]          # below the epsilon floor
    rows += [torch.full((64,), 3.0, dtype=torch.bfloat16), torch.zeros(64, dtype=torch.bfloat16)]
    return rows


def test_affine_dequant_error_bound():
    # |(q - zp) * scale - x| <= scale * (1/2 + 2^-13): half a step, plus the
    # binary32 rounding of x / scale (<= 2^-16 of a step for |x/scale| <= 256)
    # and of scale itself at the clamped top code (< 5e-5 of a step).
    for row in _rows():
        q, scale, zp = oracle.affine_int8_row(wl.u16(row))
        x = row.double().numpy()
        deq = (q.astype(np.float64) - float(zp)) * float(scale)
        assert np.all(np.abs(deq - x) <= float(scale) * (0.5 + 2.0 ** -13)), row


def test_affine_range_is_used():
    for row in _rows():
        q, scale, zp = oracle.affine_int8_row(wl.u16(row))
        x = row.float().numpy()
        mn, mx = min(0.0, x.min()), max(0.0, x.max())
        if mn < 0:
            assert q[np.argmin(x)] == -128           # the minimum lands on the lowest code
        else:
            assert int(zp) == -128                    # zero is the lowest value
        if mx > 0 and float(scale) > FLT_EPS:
            assert q[np.argmax(x)] >= 126             # the maximum lands at the top
        assert float(scale) >= FLT_EPS


def test_affine_zero_maps_to_zero_point():
    # an exact 0 dequantizes to exactly 0 (0 is always inside [mn, mx])
    row = torch.tensor([0.0, -1.5, 2.25, 0.0, 0.5, -0.75, 0.0, 1.0], dtype=torch.bfloat16)
    q, scale, zp = oracle.affine_int8_row(wl.u16(row))
    assert q[0] == zp and q[3] == zp and q[6] == zp


def test_block_golden_groups(golden_dir):
    for b in _blocks(os.path.join(golden_dir, "block_groups.txt")):
        mode = int(b["mode"][0])
        xs = [float(v) for v in b["x"]]
        xs += [float(b["fill"][0])] * (32 - len(xs))
        rs = int(b.get("round", ["1"])[0])
        codes, scales = oracle.block_row(mode, _bits(xs), round_scale=rs)
        want = [int(c, 16) for c in b["codes"]]
        nbytes = 16 if mode == 3 else 32
        want += [int(b["codefill"][0], 16)] * (nbytes - len(want))
        assert codes.tolist() == want, (mode, [hex(c) for c in codes], b)
        if mode in (1, 4, 6):
            assert float(scales[0]) == float(np.float32(b["scale"][0]))
        else:
            assert int(scales[0]) == int(b["scale"][0])


def _block_input(rows, d, seed):
    g = wl.generator(seed)
    x = wl.bf16_normal((rows, d), g, outlier_p=0.01, outlier_scale=10.0)
    x[0, :32] = 0                                   # an all-zero group
    x[1, 32:64] = torch.linspace(-1e-30, 1e-30, 32).to(torch.bfloat16)  # tiny group
    return x


def _decode_e4m3(codes):
    table = np.array([oracle.e4m3_value(c) for c in range(256)])
    return table[codes]


def _decode_e2m1(packed):
    table = np.array([oracle.e2m1_value(c) for c in range(16)])
    lo, hi = packed & 0xF, packed >> 4
    return np.stack([table[lo], table[hi]], axis=-1).reshape(*packed.shape[:-1], -1)


@pytest.mark.parametrize("mode", [1, 2, 3])
def test_block_scale_and_error_bounds(mode):
    x = _block_input(64, 512, 31 + mode)
    for r in range(x.shape[0]):
        row = x[r]
        codes, scales = oracle.block_row(mode, wl.u16(row))
        xv = row.double().numpy().reshape(-1, 32)
        amax = np.abs(xv).max(axis=1)
        if mode == 1:
            scale = scales.astype(np.float64)
            # scale_g = max|x_g| / 448 in binary32: within half an ulp of the real quotient
            assert np.all(np.abs(scale - amax / 448) <= np.spacing(scales).astype(np.float64) / 2 + 1e-300)
            deq = _decode_e4m3(codes).reshape(-1, 32) * scale[:, None]
        else:
            scale = np.exp2(scales.astype(np.float64) - 127)
            qmax = 448.0 if mode == 2 else 6.0
            nz = amax > 0
            # the E8M0 scale is the smallest power of two with amax/scale <= Q_MAX
            # (up to the binary32 rounding of amax / Q_MAX)
            r_ = amax[nz] / scale[nz]
            assert np.all(r_ <= qmax * (1 + 2.0 ** -23)) and np.all(r_ > qmax / 2 * (1 - 2.0 ** -23))
            assert np.all(scales[~nz] == 0)
            if mode == 2:
                deq = _decode_e4m3(codes).reshape(-1, 32) * scale[:, None]
            else:
                deq = _decode_e2m1(codes).reshape(-1, 32) * scale[:, None]
        err = np.abs(deq - xv)
        if mode in (1, 2):
            # E4M3: half an ulp is 2^-4 relative for normals; 2^-10 absolute
            # (units of scale) in the subnormal range; + binary32 rounding of x/scale
            bound = 2.0 ** -4 * np.abs(xv) + 2.0 ** -10 * scale[:, None] + 1e-6 * np.abs(xv)
        else:
            bound = 1.0 * scale[:, None] * (1 + 1e-6)   # widest E2M1 gap (4 -> 6) is 2
        assert np.all(err <= bound), (mode, r, err.max())
        # all-zero groups write zero codes
        zero_groups = np.where(amax == 0)[0]
        for gi in zero_groups:
            nb = 16 if mode == 3 else 32
            assert np.all(codes[gi * nb:(gi + 1) * nb] == 0)


def test_block_amax_element_hits_the_top_code():
    x = _block_input(16, 256, 77)
    for r in range(x.shape[0]):
        row = x[r]
        codes, _ = oracle.block_row(1, wl.u16(row))
        xv = row.float().numpy().reshape(-1, 32)
        for gi in range(xv.shape[0]):
            if np.abs(xv[gi]).max() == 0:
                continue
            j = np.argmax(np.abs(xv[gi]))
            assert codes[gi * 32 + j] & 0x7F == 0x7E    # |x| = amax -> 448


def _decode_e5m2(codes):
    table = np.array([oracle.e5m2_value(c) for c in range(256)])
    return table[codes]


@pytest.mark.parametrize("mode,round_scale", [(4, True), (5, True), (5, False), (6, True)])
def test_block_more_modes_scale_and_error_bounds(mode, round_scale):
    x = _block_input(64, 512, 91 + mode + 7 * round_scale)
    for r in range(x.shape[0]):
        row = x[r]
        codes, scales = oracle.block_row(mode, wl.u16(row), round_scale=round_scale)
        xv = row.double().numpy().reshape(-1, 32)
        amax = np.abs(xv).max(axis=1)
        nz = amax > 0
        if mode in (4, 6):
            qmax = 57344.0 if mode == 4 else 127.0
            scale = scales.astype(np.float64)
            assert np.all(np.abs(scale - amax / qmax) <= np.spacing(scales).astype(np.float64) / 2 + 1e-300)
        else:
            scale = np.exp2(scales.astype(np.float64) - 127)
            r_ = amax[nz] / scale[nz]
            if round_scale:   # smallest power of two with amax/scale <= Q_MAX
                assert np.all(r_ <= 57344 * (1 + 2.0 ** -23)) and np.all(r_ > 57344 / 2 * (1 - 2.0 ** -23))
            else:             # largest power of two <= amax / Q_MAX
                assert np.all(r_ >= 57344 * (1 - 2.0 ** -23)) and np.all(r_ < 2 * 57344 * (1 + 2.0 ** -23))
            assert np.all(scales[~nz] == 0)
        if mode == 6:
            q = codes.view(np.int8).astype(np.float64).reshape(-1, 32)
            assert np.all(np.abs(q) <= 127)
            deq = q * scale[:, None]
            # half a step, plus the binary32 rounding of x / scale (<= 127 * 2^-24 of a step)
            bound = scale[:, None] * (0.5 + 2.0 ** -16)
            for gi in np.where(nz)[0]:   # the largest element lands on +-127
                assert abs(q[gi, np.argmax(np.abs(xv[gi]))]) == 127
        else:
            deq = _decode_e5m2(codes).reshape(-1, 32) * scale[:, None]
            # E5M2: half an ulp is 2^-3 relative for normals, 2^-17 absolute (units of
            # scale) in the subnormal range; + binary32 rounding of x / scale
            bound = 2.0 ** -3 * np.abs(xv) + 2.0 ** -17 * scale[:, None] + 1e-6 * np.abs(xv)
            if mode == 5 and not round_scale:   # codes saturate at 57344 * scale
                bound = np.maximum(bound, np.abs(xv) - 57344 * scale[:, None] + 1e-300)
        err = np.abs(deq - xv)
        assert np.all(err <= bound), (mode, round_scale, r, err.max())
        for gi in np.where(~nz)[0]:
            assert np.all(codes[gi * 32:(gi + 1) * 32] == 0)


def test_affine_int4_golden_rows(golden_dir):
    blocks = _blocks(os.path.join(golden_dir, "affine_int4_rows.txt"))
    assert len(blocks) == 5
    for b in blocks:
        packed, scale, zp = oracle.affine_int4_row(_bits(b["x"]))
        q = [int(v) for v in b["q"]]
        assert packed.tolist() == [int(c, 16) for c in b["packed"]], b
        assert packed.tolist() == [q[2 * i] | (q[2 * i + 1] << 4) for i in range(len(q) // 2)]
        assert float(scale) == float(np.float32(b["scale"][0]))
        assert int(zp) == int(b["zp"][0])


def _unpack4(packed):
    return np.stack([packed & 15, packed >> 4], axis=-1).reshape(*packed.shape[:-1], -1)


def test_affine_int4_dequant_error_bound_and_range():
    # |(q - zp) * scale - x| <= scale * (1/2 + 2^-16): half a step plus the binary32
    # rounding of x / scale (<= 15 * 2^-24 of a step) and of scale at the clamped top code
    for row in _rows():
        packed, scale, zp = oracle.affine_int4_row(wl.u16(row))
        q = _unpack4(packed).astype(np.int64)
        x = row.double().numpy()
        deq = (q - int(zp)) * float(scale)
        assert np.all(np.abs(deq - x) <= float(scale) * (0.5 + 2.0 ** -16)), row
        assert 0 <= int(zp) <= 15 and q.min() >= 0 and q.max() <= 15
        mn, mx = min(0.0, x.min()), max(0.0, x.max())
        if mn < 0:
            assert q[np.argmin(x)] == 0               # the minimum lands on the lowest code
        if mx > 0 and float(scale) > FLT_EPS:
            assert q[np.argmax(x)] >= 14              # the maximum lands at the top


def _nearest_saturating(y, table):
    """Brute force: the code whose value is nearest y, saturating at the largest
    magnitude; ties go to the code with an even last bit; the sign follows y."""
    mags = np.array([table[c] for c in range(len(table) // 2)])
    out = np.zeros(y.shape, np.int64)
    for i, v in enumerate(y):
        d = np.abs(mags - min(abs(v), mags.max()))
        best = np.flatnonzero(d == d.min())
        c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out[i] = c | (len(table) // 2 if v < 0 else 0)
    return out


@pytest.mark.parametrize("mode,round_scale", [(3, 0), (3, 2), (2, 2), (5, 2)])
def test_block_floor_and_ocp_scale_rules(mode, round_scale):
    """round_scale 0 takes the exponent of amax / Q_MAX as it stands, so
    amax / scale lies in [Q_MAX, 2 Q_MAX); round_scale 2 is the OCP MX v1.0 rule
    2^(floor(log2 amax) - emax), so amax / scale lies in [2^emax, 2^(emax+1)).
    Every code is then the saturating nearest-value code of x / scale (MX-FP4:
    brute force over the 8 magnitudes, element 2i in the low nibble)."""
    qmax = {2: 448.0, 3: 6.0, 5: 57344.0}[mode]
    emax = {2: 8, 3: 2, 5: 15}[mode]
    x = _block_input(48, 256, 401 + mode + round_scale)
    for r in range(x.shape[0]):
        row = x[r]
        codes, scales = oracle.block_row(mode, wl.u16(row), round_scale=round_scale)
        xv = row.double().numpy().reshape(-1, 32)
        amax = np.abs(xv).max(axis=1)
        scale = np.exp2(scales.astype(np.float64) - 127)
        ok = (amax > 2.0 ** -100)  # away from the E8M0 clamp
        r_ = amax[ok] / scale[ok]
        if round_scale == 0:
            assert np.all(r_ >= qmax * (1 - 2.0 ** -23)) and np.all(r_ < 2 * qmax * (1 + 2.0 ** -23))
        else:
            assert np.all(r_ >= 2.0 ** emax) and np.all(r_ < 2.0 ** (emax + 1))
        assert np.all(scales[amax == 0] == 0)
        if mode == 3:
            table = [oracle.e2m1_value(c) for c in range(16)]
            got = np.stack([codes & 0xF, codes >> 4], axis=1).reshape(-1, 32)
        else:
            table = [oracle.e4m3_value(c) if mode == 2 else oracle.e5m2_value(c) for c in range(256)]
            got = codes.reshape(-1, 32).astype(np.int64)
        for gi in np.flatnonzero(ok):
            y = (xv[gi] / scale[gi]).astype(np.float32).astype(np.float64)
            if mode == 3:
                want = _nearest_saturating(y, table)
            else:
                # FP8: compare values (the oracle's codec is pinned exhaustively elsewhere);
                # the value must be the saturating nearest of x / scale
                vals = np.array([table[c] for c in got[gi]])
                fin = np.array([v for v in table if np.isfinite(v)])
                top = fin.max()
                for v, yy in zip(vals, y):
                    t = min(abs(yy), top)
                    assert abs(abs(v) - t) <= np.abs(fin - t).min() + 1e-300
                continue
            assert np.array_equal(got[gi] & 0x7, want & 0x7) and np.all(
                ((got[gi] >> 3) == (want >> 3)) | ((want & 0x7) == 0)), (r, gi)
