/*
 * kvq_oracle.c -- the CPU oracle for the quantized KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * statement of what the CUDA library computes.  It is compiled and called only
 * by the tests, by the package entry's smoke check and by the benchmark's CPU
 * baseline leg.  The product path never links, loads or calls it, and it shares
 * no source, header, table or helper with the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC -lm
 * (done on demand by oracle/__init__.py).  All single-precision expressions are
 * evaluated in IEEE binary32 (x86-64 SSE, FLT_EVAL_METHOD == 0) with the default
 * round-to-nearest-even mode, one rounding per operation, no contraction.
 *
 * Sources, by page title and section:
 *   [P1] ExecuTorch PR 24473 (quantized KV cache with attention sink), Summary:
 *        int8 entries quantized per token and head, affine asymmetric, float32
 *        scale + int8 zero point; slots from CachePositionsManagerWithSink; an
 *        additive float mask from _create_causal_mask_for_attention_sink; a
 *        full-context cache keeps plain causal attention.
 *   [P3] abaddon 0.2.0-rc.1, src/attention_cache/mod.rs, trait KvCache:
 *        append() takes [batch, num_kv_heads, seq_len, head_dim];
 *        forward_attention(q [batch, num_heads, q_len, head_dim], num_heads,
 *        scale = 1/sqrt(head_dim) typically); GQA via repeat_kv.
 *   [P4] ExecuTorch PR 20351 "[cuda backend] reduce memory consumption on
 *        gemma4_31b ...", commit notes: writes are a static scatter along the
 *        position dim; kv_len bounds the KV loop; per-tile causal upper bound
 *        loop_end = min(kv_len, (kv_len - Lq) + max(seq_pos) + 1).
 *   [P5] IndexerQuantCache operator page, sections 功能说明 (function),
 *        计算公式 (formula), 参数说明 (parameters), 约束说明 (constraints):
 *        per-block dynamic quantization scale_g = max|x_g| / Q_MAX,
 *        q_i = round(x_i / scale_g), scattered by slot_mapping, -1 = skip.
 *   Number formats: OCP 8-bit floating point (E4M3, "fn" variant: no
 *   infinities, S.1111.111 = NaN) and OCP Microscaling formats v1.0 (E2M1
 *   element, E8M0 scale, block of 32).
 *
 * Readings taken where the pages are silent (each one also listed in the
 * design notes): the affine formula itself and its epsilon floor; the E8M0
 * scale is rounded UP to a power of two for MX-FP8 (round_scale=true) and
 * MX-FP4; FP4 element 2i goes to the low nibble; an all-zero group writes
 * zero codes and a zero scale (E8M0 byte 0); the sink/ring slot formula; the
 * mask visibility rule; GQA head h uses kv head h / (Hq / Hkv).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KVQO_MODE_INT8_AFFINE 0
#define KVQO_MODE_FP8_E4M3 1
#define KVQO_MODE_MXFP8 2
#define KVQO_MODE_MXFP4 3
#define KVQO_MODE_FP8_E5M2 4   /* Normal, FLOAT8_E5M2 cache, float32 scale */
#define KVQO_MODE_MXFP8_E5M2 5 /* MX-FP8, FLOAT8_E5M2 cache, E8M0 scale */
#define KVQO_MODE_INT8_SYM 6   /* Normal, UINT8 cache holding int8 codes, float32 scale */
#define KVQO_MODE_INT4_AFFINE 7 /* TQ4 packing: 4-bit affine per token and head, two codes per byte */

/* ------------------------------------------------------------------------- */
/* bfloat16: the top 16 bits of a binary32.  Widening is exact.              */
/* ------------------------------------------------------------------------- */
static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------- */
/* FP8 E4M3 (OCP "fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.   */
/* Normal: (1 + m/8) * 2^(e-7); subnormal (e == 0): (m/8) * 2^-6;            */
/* S.1111.111 is NaN; there is no infinity; largest finite is 448.           */
/* ------------------------------------------------------------------------- */
double kvqo_e4m3_value(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);          /* (m/8) * 2^-6 */
    else
        mag = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -mag : mag;
}

/* Round to nearest, ties to the even code (even mantissa), saturating to the
 * largest finite magnitude; the sign of the input is kept, so a negative
 * value that rounds to zero encodes as 0x80.  Found by exhaustive search over
 * every finite non-negative code.  Non-finite input is outside the contract. */
uint8_t kvqo_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    uint8_t best = 0;
    double bestdiff = a;
    if (a >= 448.0)
        return sign | 0x7E;
    for (int c = 1; c <= 0x7E; ++c) {
        double diff = fabs(kvqo_e4m3_value((uint8_t)c) - a);
        if (diff < bestdiff || (diff == bestdiff && (c & 1) == 0)) {
            best = (uint8_t)c;
            bestdiff = diff;
        }
    }
    return sign | best;
}

/* ------------------------------------------------------------------------- */
/* FP8 E5M2 (OCP): 1 sign, 5 exponent bits (bias 15), 2 mantissa bits.       */
/* Normal: (1 + m/4) * 2^(e-15); subnormal (e == 0): (m/4) * 2^-14;          */
/* e == 31 is infinity (m == 0) or NaN; largest finite is 57344.             */
/* ------------------------------------------------------------------------- */
double kvqo_e5m2_value(uint8_t c)
{
    int s = c >> 7, e = (c >> 2) & 31, m = c & 3;
    double mag;
    if (e == 31)
        return m ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0)
        mag = ldexp((double)m, -16);          /* (m/4) * 2^-14 */
    else
        mag = ldexp((double)(4 + m), e - 17); /* (1 + m/4) * 2^(e-15) */
    return s ? -mag : mag;
}

/* Same rule as the E4M3 encoder: nearest, ties to the even code, saturating
 * to the largest finite magnitude (never infinity), sign kept. */
uint8_t kvqo_e5m2_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    uint8_t best = 0;
    double bestdiff = a;
    if (a >= 57344.0)
        return sign | 0x7B;
    for (int c = 1; c <= 0x7B; ++c) {
        double diff = fabs(kvqo_e5m2_value((uint8_t)c) - a);
        if (diff < bestdiff || (diff == bestdiff && (c & 1) == 0)) {
            best = (uint8_t)c;
            bestdiff = diff;
        }
    }
    return sign | best;
}

/* ------------------------------------------------------------------------- */
/* FP4 E2M1 (OCP MX): 1 sign, 2 exponent bits (bias 1), 1 mantissa bit.      */
/* Magnitudes: 0, 0.5, 1, 1.5, 2, 3, 4, 6.  No NaN, no infinity.             */
/* ------------------------------------------------------------------------- */
double kvqo_e2m1_value(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp((double)(2 + m), e - 2);
    return s ? -mag : mag;
}

uint8_t kvqo_e2m1_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs((double)v);
    uint8_t best = 0;
    double bestdiff = a;
    if (a >= 6.0)
        return sign | 0x7;
    for (int c = 1; c <= 7; ++c) {
        double diff = fabs(kvqo_e2m1_value((uint8_t)c) - a);
        if (diff < bestdiff || (diff == bestdiff && (c & 1) == 0)) {
            best = (uint8_t)c;
            bestdiff = diff;
        }
    }
    return sign | best;
}

/* ------------------------------------------------------------------------- */
/* E8M0 (OCP MX scale): value 2^(e - 127), e = 0..254; 0xFF is NaN.          */
/* ------------------------------------------------------------------------- */
double kvqo_e8m0_value(uint8_t e)
{
    if (e == 0xFF)
        return NAN;
    return ldexp(1.0, (int)e - 127);
}

/* The smallest power of two >= s, as an E8M0 byte clamped to [0, 254]
 * (reading of round_scale=true: rounding up is the only direction under
 * which q = x / scale never exceeds Q_MAX).  s <= 0 gives 0. */
uint8_t kvqo_e8m0_ceil(float s)
{
    int k, l, e;
    double f;
    if (!(s > 0.0f))
        return 0;
    f = frexp((double)s, &k); /* s = f * 2^k, 0.5 <= f < 1 */
    l = (f == 0.5) ? k - 1 : k; /* ceil(log2 s) */
    e = l + 127;
    if (e < 0)
        e = 0;
    if (e > 254)
        e = 254;
    return (uint8_t)e;
}

/* The largest power of two <= s, as an E8M0 byte clamped to [0, 254]
 * (reading of round_scale=false: the scale is not rounded, so its exponent is
 * taken as it stands; codes then saturate at Q_MAX).  s <= 0 gives 0. */
uint8_t kvqo_e8m0_floor(float s)
{
    int k, e;
    if (!(s > 0.0f))
        return 0;
    (void)frexp((double)s, &k); /* s = f * 2^k, 0.5 <= f < 1: floor(log2 s) = k - 1 */
    e = (k - 1) + 127;
    if (e < 0)
        e = 0;
    if (e > 254)
        e = 254;
    return (uint8_t)e;
}

/* The OCP MX rule (OCP Microscaling Formats v1.0, section 6.3: the shared   */
/* exponent is floor(log2 amax) minus the element format's largest exponent, */
/* emax 8 for E4M3, 15 for E5M2, 2 for E2M1), as an E8M0 byte clamped to     */
/* [0, 254]; amax <= 0 gives 0.  Codes may then exceed Q_MAX and saturate.   */
uint8_t kvqo_e8m0_ocp(float amax, int emax_elem)
{
    int k, e;
    if (!(amax > 0.0f))
        return 0;
    (void)frexp((double)amax, &k); /* amax = f * 2^k, 0.5 <= f < 1: floor(log2 amax) = k - 1 */
    e = (k - 1) - emax_elem + 127;
    if (e < 0)
        e = 0;
    if (e > 254)
        e = 254;
    return (uint8_t)e;
}

/* ------------------------------------------------------------------------- */
/* [P1] per-token-and-head affine asymmetric int8, one row of D values.      */
/* fp32, each step rounded to nearest even, in exactly this order:           */
/*   mn = min(0, min x), mx = max(0, max x)                                  */
/*   scale = (mx - mn) / 255, floored at FLT_EPSILON                         */
/*   zp = clamp(-128 - rne(mn / scale), -128, 127)                           */
/*   q_i = clamp(rne(x_i / scale) + zp, -128, 127)                           */
/* Dequantization is (q - zp) * scale.                                       */
/* ------------------------------------------------------------------------- */
static long clampl(long v, long lo, long hi) { return v < lo ? lo : (v > hi ? hi : v); }

void kvqo_affine_int8_row(const uint16_t *x, int D, int8_t *q, float *scale_out, int8_t *zp_out)
{
    float mn = 0.0f, mx = 0.0f, scale;
    long zp;
    for (int i = 0; i < D; ++i) {
        float v = bf16_to_float(x[i]);
        if (v < mn)
            mn = v;
        if (v > mx)
            mx = v;
    }
    scale = (mx - mn) / 255.0f;
    if (scale < FLT_EPSILON)
        scale = FLT_EPSILON;
    zp = clampl(-128L - lrintf(mn / scale), -128, 127);
    for (int i = 0; i < D; ++i) {
        float v = bf16_to_float(x[i]);
        q[i] = (int8_t)clampl(lrintf(v / scale) + zp, -128, 127);
    }
    *scale_out = scale;
    *zp_out = (int8_t)zp;
}

/* ------------------------------------------------------------------------- */
/* [P4] TQ4 cache: nibble-packed along the last dim (D/2 bytes per slot),    */
/* written along the position dim.  The pages give only the packing; the     */
/* code is read here as the 4-bit form of the affine per-token-and-head      */
/* quantizer above, onto [0, 15], same fp32 order and rounding:              */
/*   mn = min(0, min x), mx = max(0, max x)                                  */
/*   scale = (mx - mn) / 15, floored at FLT_EPSILON                          */
/*   zp = clamp(-rne(mn / scale), 0, 15)                                     */
/*   q_i = clamp(rne(x_i / scale) + zp, 0, 15)                               */
/* packed[i] = q_{2i} | q_{2i+1} << 4 (element 2i in the low nibble).        */
/* Dequantization is (q - zp) * scale.                                       */
/* ------------------------------------------------------------------------- */
void kvqo_affine_int4_row(const uint16_t *x, int D, uint8_t *packed, float *scale_out, uint8_t *zp_out)
{
    float mn = 0.0f, mx = 0.0f, scale;
    long zp;
    for (int i = 0; i < D; ++i) {
        float v = bf16_to_float(x[i]);
        if (v < mn)
            mn = v;
        if (v > mx)
            mx = v;
    }
    scale = (mx - mn) / 15.0f;
    if (scale < FLT_EPSILON)
        scale = FLT_EPSILON;
    zp = clampl(-lrintf(mn / scale), 0, 15);
    for (int i = 0; i < D; i += 2) {
        long q0 = clampl(lrintf(bf16_to_float(x[i]) / scale) + zp, 0, 15);
        long q1 = clampl(lrintf(bf16_to_float(x[i + 1]) / scale) + zp, 0, 15);
        packed[i / 2] = (uint8_t)(q0 | (q1 << 4));
    }
    *scale_out = scale;
    *zp_out = (uint8_t)zp;
}

/* ------------------------------------------------------------------------- */
/* [P5] 计算公式: per-block dynamic quantization of one row of d values,      */
/* groups of 32 along d.  scale_g = max|x_g| / Q_MAX, q_i = round(x_i/scale). */
/*   mode 1 (Normal, FP8 E4M3): Q_MAX 448, scale stored as float32.          */
/*   mode 4 (Normal, FP8 E5M2): Q_MAX 57344, scale stored as float32.        */
/*   mode 6 (Normal, INT8 in a UINT8 cache): Q_MAX 127, q = rne(x/scale)     */
/*          clamped to [-127, 127], stored as its two's-complement byte;     */
/*          scale stored as float32.                                         */
/*   mode 2 (MX-FP8, E4M3) / mode 5 (MX-FP8, E5M2): Q_MAX 448 / 57344; the   */
/*          scale becomes a power of two stored as E8M0.                     */
/*   mode 3 (MX-FP4): Q_MAX 6, E2M1 codes, two per byte (2i low nibble),     */
/*          scale a power of two stored as E8M0.                             */
/*   The power of two for modes 2, 3, 5 follows round_scale: 1 (the default) */
/*   rounds amax / Q_MAX up, 0 takes its exponent as it stands (floor), 2    */
/*   takes the OCP MX rule floor(log2 amax) - emax (kvqo_e8m0_ocp).          */
/* An all-zero group writes zero codes and a zero scale (E8M0 byte 0).       */
/* codes: d bytes (modes 1, 2, 4, 5, 6) or d/2 bytes (mode 3);               */
/* scale: d/32 entries.                                                      */
/* ------------------------------------------------------------------------- */
void kvqo_block_row(int mode, int round_scale, const uint16_t *x, int d, uint8_t *codes, float *scale_f32,
                    uint8_t *scale_e8m0)
{
    for (int g = 0; g < d / 32; ++g) {
        const uint16_t *xg = x + 32 * g;
        float amax = 0.0f;
        for (int i = 0; i < 32; ++i) {
            float a = fabsf(bf16_to_float(xg[i]));
            if (a > amax)
                amax = a;
        }
        if (mode == KVQO_MODE_FP8_E4M3 || mode == KVQO_MODE_FP8_E5M2) {
            int e5 = (mode == KVQO_MODE_FP8_E5M2);
            float scale = amax / (e5 ? 57344.0f : 448.0f);
            scale_f32[g] = scale;
            for (int i = 0; i < 32; ++i) {
                float y = bf16_to_float(xg[i]) / scale;
                codes[32 * g + i] = (amax == 0.0f) ? 0 : (e5 ? kvqo_e5m2_encode(y) : kvqo_e4m3_encode(y));
            }
        } else if (mode == KVQO_MODE_INT8_SYM) {
            float scale = amax / 127.0f;
            scale_f32[g] = scale;
            for (int i = 0; i < 32; ++i) {
                long q = (amax == 0.0f) ? 0 : clampl(lrintf(bf16_to_float(xg[i]) / scale), -127, 127);
                codes[32 * g + i] = (uint8_t)(int8_t)q;
            }
        } else if (mode == KVQO_MODE_MXFP8 || mode == KVQO_MODE_MXFP8_E5M2) {
            int e5 = (mode == KVQO_MODE_MXFP8_E5M2);
            float s = amax / (e5 ? 57344.0f : 448.0f);
            uint8_t e = round_scale == 2 ? kvqo_e8m0_ocp(amax, e5 ? 15 : 8)
                        : round_scale   ? kvqo_e8m0_ceil(s)
                                        : kvqo_e8m0_floor(s);
            float scale = (float)ldexp(1.0, (int)e - 127); /* exact, possibly subnormal */
            scale_e8m0[g] = e;
            for (int i = 0; i < 32; ++i) {
                float y = bf16_to_float(xg[i]) / scale;
                codes[32 * g + i] = (amax == 0.0f) ? 0 : (e5 ? kvqo_e5m2_encode(y) : kvqo_e4m3_encode(y));
            }
        } else { /* KVQO_MODE_MXFP4 */
            float s = amax / 6.0f;
            uint8_t e = round_scale == 2 ? kvqo_e8m0_ocp(amax, 2)
                        : round_scale   ? kvqo_e8m0_ceil(s)
                                        : kvqo_e8m0_floor(s);
            float scale = (float)ldexp(1.0, (int)e - 127);
            scale_e8m0[g] = e;
            for (int i = 0; i < 32; i += 2) {
                uint8_t lo = (amax == 0.0f) ? 0 : kvqo_e2m1_encode(bf16_to_float(xg[i]) / scale);
                uint8_t hi = (amax == 0.0f) ? 0 : kvqo_e2m1_encode(bf16_to_float(xg[i + 1]) / scale);
                codes[16 * g + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* The cache write: quantize x[b, h, t, :] and scatter it to cache slot      */
/* slot_mapping[b*T + t] of (b, h).  [P5] 约束说明: -1 means skip; valid      */
/* slots lie in [0, num_slots); duplicates are undefined.  [P1]: a write     */
/* outside the slot range is rejected -- here: skipped and reported in *err  */
/* (bit 0).  x element (b,h,t,i) is at x[b*xs[0] + h*xs[1] + t*xs[2] + i].   */
/* Cache layouts, all row-major:                                             */
/*   mode 0: codes int8 [B,H,S,D], scales f32 [B,H,S], zps int8 [B,H,S]     */
/*   mode 1: codes u8 [B,H,S,D], scales f32 [B,H,S,D/32]                     */
/*   mode 2: codes u8 [B,H,S,D], scales e8m0 [B,H,S,D/32]                    */
/*   mode 3: codes u8 [B,H,S,D/2], scales e8m0 [B,H,S,D/32]                  */
/*   modes 4, 6: as mode 1;  mode 5: as mode 2                               */
/*   mode 7: codes u8 [B,H,S,D/2] (nibbles), scales f32 [B,H,S],             */
/*           zps [B,H,S] holding 0..15                                       */
/* With B = H = 1 this is the page's cache [num_slots, d] layout.            */
/* ------------------------------------------------------------------------- */
void kvqo_write(int mode, int round_scale, const uint16_t *x, int B, int H, int T, int D, const int64_t *xs,
                const int32_t *slot_mapping, int64_t S, void *codes, void *scales, int8_t *zps,
                int32_t *err)
{
    int64_t code_row = (mode == KVQO_MODE_MXFP4 || mode == KVQO_MODE_INT4_AFFINE) ? D / 2 : D;
    int64_t scale_row = (mode == KVQO_MODE_INT8_AFFINE || mode == KVQO_MODE_INT4_AFFINE) ? 1 : D / 32;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < T; ++t) {
            int32_t slot = slot_mapping[(int64_t)b * T + t];
            if (slot == -1)
                continue;
            if (slot < 0 || slot >= S) {
                *err |= 1;
                continue;
            }
            for (int h = 0; h < H; ++h) {
                const uint16_t *row = x + b * xs[0] + h * xs[1] + t * xs[2];
                int64_t r = ((int64_t)b * H + h) * S + slot;
                if (mode == KVQO_MODE_INT8_AFFINE) {
                    kvqo_affine_int8_row(row, D, (int8_t *)codes + r * code_row, (float *)scales + r,
                                         zps + r);
                } else if (mode == KVQO_MODE_INT4_AFFINE) {
                    kvqo_affine_int4_row(row, D, (uint8_t *)codes + r * code_row, (float *)scales + r,
                                         (uint8_t *)zps + r);
                } else {
                    kvqo_block_row(mode, round_scale, row, D, (uint8_t *)codes + r * code_row,
                                   (float *)scales + r * scale_row, (uint8_t *)scales + r * scale_row);
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* [P1] attention-sink / ring layout (CachePositionsManagerWithSink):        */
/*   slot(p) = p                                  for p < sink               */
/*           = sink + (p - sink) mod (S - sink)   otherwise                  */
/* sink = 0 is the plain ring cache.  slot_pos[slot] records the position     */
/* the slot now holds (-1 = never written); the filled slots are always       */
/* [0, min(last + 1, S)), which is returned as the attention bound kv_len.    */
/* All B batch rows use the same positions.                                  */
/* ------------------------------------------------------------------------- */
void kvqo_sink_plan(int32_t input_pos, int B, int T, int sink, int64_t S, int32_t *slot_mapping,
                    int32_t *slot_pos, int32_t *kv_len)
{
    for (int t = 0; t < T; ++t) {
        int64_t p = (int64_t)input_pos + t;
        int64_t slot = (p < sink) ? p : sink + (p - sink) % (S - sink);
        for (int b = 0; b < B; ++b)
            slot_mapping[(int64_t)b * T + t] = (int32_t)slot;
        slot_pos[slot] = (int32_t)p;
    }
    {
        int64_t end = (int64_t)input_pos + T;
        *kv_len = (int32_t)(end < S ? end : S);
    }
}

/* [P1] _create_causal_mask_for_attention_sink, read as: query row r sits at
 * position input_pos + r and sees slot s iff the slot holds a position that
 * is not in its future.  Additive: 0 visible, -inf hidden.  mask is [Lq, S]. */
void kvqo_sink_mask(int32_t input_pos, int Lq, const int32_t *slot_pos, int64_t S, float *mask)
{
    for (int r = 0; r < Lq; ++r) {
        int64_t qpos = (int64_t)input_pos + r;
        for (int64_t s = 0; s < S; ++s)
            mask[(int64_t)r * S + s] = (slot_pos[s] >= 0 && slot_pos[s] <= qpos) ? 0.0f : -INFINITY;
    }
}

/* ------------------------------------------------------------------------- */
/* Scaled dot-product attention over the int8 cache, in fp64, one query row. */
/* [P3] q [B,Hq,Lq,D], caches [B,Hkv,S,D] (+ [B,Hkv,S] scale / zero point);   */
/* q head h reads kv head h / (Hq/Hkv).  [P4] only slots j < kv_len take     */
/* part; with is_causal, row i (of Lq) sees j <= kv_len - Lq + i.  [P1] an   */
/* additive mask [Lq, S] (row stride S) is added to the scaled scores.        */
/* K and V are dequantized as (c - zp) * scale: c an int8 code (kbits 8), or */
/* a 4-bit code 0..15 of the TQ4 packing (kbits 4: D/2 bytes per slot, code  */
/* d in the low nibble of byte d/2 when d is even, else the high nibble).    */
/* A row that sees nothing outputs zeros.                                    */
/* ------------------------------------------------------------------------- */
static double code_at(const int8_t *c, int64_t slot, int D, int d, int kbits)
{
    if (kbits == 4) {
        uint8_t byte = (uint8_t)c[slot * (D / 2) + d / 2];
        return (double)((d & 1) ? (byte >> 4) : (byte & 15));
    }
    return (double)c[slot * D + d];
}

void kvqo_sdpa_row(const uint16_t *q, int B, int Hq, int Lq, int D, int kbits, const int8_t *k, const float *ks,
                   const int8_t *kz, const int8_t *v, const float *vs, const int8_t *vz, int Hkv,
                   int64_t S, int32_t kv_len, const float *mask, int is_causal, float sm_scale, int b,
                   int h, int i, double *out)
{
    int G = Hq / Hkv, hk = h / G;
    const uint16_t *qr = q + (((int64_t)b * Hq + h) * Lq + i) * D;
    int64_t base = ((int64_t)b * Hkv + hk) * S;
    double *s = (double *)malloc(sizeof(double) * (kv_len > 0 ? (size_t)kv_len : 1));
    double m = -INFINITY, l = 0.0;
    (void)B;
    for (int64_t j = 0; j < kv_len; ++j) {
        if (is_causal && j > (int64_t)kv_len - Lq + i) {
            s[j] = -INFINITY;
        } else {
            double dot = 0.0;
            for (int d = 0; d < D; ++d) {
                double kd = (code_at(k, base + j, D, d, kbits) - (double)kz[base + j]) * (double)ks[base + j];
                dot += (double)bf16_to_float(qr[d]) * kd;
            }
            s[j] = dot * (double)sm_scale + (mask ? (double)mask[(int64_t)i * S + j] : 0.0);
        }
        if (s[j] > m)
            m = s[j];
    }
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    if (m == -INFINITY) {
        free(s);
        return;
    }
    for (int64_t j = 0; j < kv_len; ++j) {
        double p = exp(s[j] - m);
        l += p;
        if (p == 0.0)
            continue;
        for (int d = 0; d < D; ++d)
            out[d] += p * (code_at(v, base + j, D, d, kbits) - (double)vz[base + j]) * (double)vs[base + j];
    }
    for (int d = 0; d < D; ++d)
        out[d] /= l;
    free(s);
}

/* Every row: out is [B, Hq, Lq, D]. */
void kvqo_sdpa(const uint16_t *q, int B, int Hq, int Lq, int D, int kbits, const int8_t *k, const float *ks,
               const int8_t *kz, const int8_t *v, const float *vs, const int8_t *vz, int Hkv, int64_t S,
               int32_t kv_len, const float *mask, int is_causal, float sm_scale, double *out)
{
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h)
            for (int i = 0; i < Lq; ++i)
                kvqo_sdpa_row(q, B, Hq, Lq, D, kbits, k, ks, kz, v, vs, vz, Hkv, S, kv_len, mask, is_causal,
                              sm_scale, b, h, i, out + (((int64_t)b * Hq + h) * Lq + i) * D);
}

/* ------------------------------------------------------------------------- */
/* [P5] dequantization of the per-32 block caches (the inverse the page's    */
/* formula implies: x ~ code_value * scale_g), for attention over them:      */
/*   modes 1, 4, 6: code value (E4M3 / E5M2 / int8) * float32 scale          */
/*   modes 2, 5, 3: code value (E4M3 / E5M2 / E2M1 nibble) * 2^(e - 127)     */
/* codes: rows x d (mode 3: rows x d/2, element 2i in the low nibble);       */
/* scales: rows x d/32 (float32 or E8M0 bytes).  out: rows x d, fp64.        */
/* ------------------------------------------------------------------------- */
void kvqo_dequant_block(int mode, const uint8_t *codes, const void *scales, int64_t rows, int d, double *out)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int i = 0; i < d; ++i) {
            int64_t g = r * (d / 32) + i / 32;
            double code, scale;
            if (mode == KVQO_MODE_MXFP4) {
                uint8_t byte = codes[r * (d / 2) + i / 2];
                code = kvqo_e2m1_value((i & 1) ? (byte >> 4) : (byte & 15));
            } else {
                uint8_t c = codes[r * d + i];
                if (mode == KVQO_MODE_FP8_E4M3 || mode == KVQO_MODE_MXFP8)
                    code = kvqo_e4m3_value(c);
                else if (mode == KVQO_MODE_FP8_E5M2 || mode == KVQO_MODE_MXFP8_E5M2)
                    code = kvqo_e5m2_value(c);
                else
                    code = (double)(int8_t)c; /* KVQO_MODE_INT8_SYM */
            }
            if (mode == KVQO_MODE_FP8_E4M3 || mode == KVQO_MODE_FP8_E5M2 || mode == KVQO_MODE_INT8_SYM)
                scale = (double)((const float *)scales)[g];
            else
                scale = kvqo_e8m0_value(((const uint8_t *)scales)[g]);
            out[r * d + i] = code * scale;
        }
    }
}

/* fp64 attention for one row over dense fp64 K, V [B, Hkv, S, D] -- the same */
/* definition as kvqo_sdpa_row ([P3] shapes and GQA, [P4] kv_len and causal  */
/* rule, [P1] additive mask), with K and V given as values.                  */
void kvqo_sdpa_dense_row(const uint16_t *q, int B, int Hq, int Lq, int D, const double *K, const double *V,
                         int Hkv, int64_t S, int32_t kv_len, const float *mask, int is_causal, float sm_scale,
                         int b, int h, int i, double *out)
{
    int G = Hq / Hkv, hk = h / G;
    const uint16_t *qr = q + (((int64_t)b * Hq + h) * Lq + i) * D;
    int64_t base = ((int64_t)b * Hkv + hk) * S;
    double *s = (double *)malloc(sizeof(double) * (kv_len > 0 ? (size_t)kv_len : 1));
    double m = -INFINITY, l = 0.0;
    (void)B;
    for (int64_t j = 0; j < kv_len; ++j) {
        if (is_causal && j > (int64_t)kv_len - Lq + i) {
            s[j] = -INFINITY;
        } else {
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += (double)bf16_to_float(qr[d]) * K[(base + j) * D + d];
            s[j] = dot * (double)sm_scale + (mask ? (double)mask[(int64_t)i * S + j] : 0.0);
        }
        if (s[j] > m)
            m = s[j];
    }
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    if (m == -INFINITY) {
        free(s);
        return;
    }
    for (int64_t j = 0; j < kv_len; ++j) {
        double p = exp(s[j] - m);
        l += p;
        if (p == 0.0)
            continue;
        for (int d = 0; d < D; ++d)
            out[d] += p * V[(base + j) * D + d];
    }
    for (int d = 0; d < D; ++d)
        out[d] /= l;
    free(s);
}
