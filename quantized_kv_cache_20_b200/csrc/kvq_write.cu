// kvq_write.cu -- the quantized KV-cache write (quantize + scatter by slot).
//
// Work is cut into 32-element groups along the last dim; one lane owns one
// group (64 bytes of bf16 x: four 16-byte loads) and writes its codes.
//   - block modes (IndexerQuantCache page, 计算公式: scale_g = max|x_g| / Q_MAX,
//     q_i = round(x_i / scale_g)) need nothing outside the group;
//   - the int8 affine mode (ExecuTorch PR 24473, Summary: per token and head)
//     reduces min/max over the D/32 lanes of a row with xor-shuffles.
// A warp covers 32 consecutive groups, i.e. 2 KB of contiguous input for
// contiguous K/V.  Tokens whose slot is -1 are skipped before their x is read
// (IndexerQuantCache page, 约束说明), so skipped rows cost no input bandwidth.
//
// The arithmetic is binary32, one round-to-nearest-even per operation, in the
// order the definitions state, so codes, scales and zero points are
// reproducible bit for bit.  Division by a per-row/per-group scale takes the
// quotient from Markstein's correction of x * rcp(scale) (rcp correctly
// rounded), which is the correctly rounded quotient wherever it can move a code;
// groups of tiny values (amax < 2^-60) divide exactly (__fdiv_rn).  MX scales are
// powers of two, so their quotients are exact products.
#include <cuda_bf16.h>
#include <float.h>

#include "kvq_common.cuh"

namespace kvq {
namespace {

// Division by a run-time invariant divisor d >= 1 for numerators n < 2^31
// (Granlund & Montgomery, "Division by invariant integers using
// multiplication", 1994): q = (umulhi(n, m) + n) >> s.
struct FastDiv {
  uint32_t d, m, s;
  FastDiv() = default;
  explicit FastDiv(uint32_t div) : d(div) {
    s = 0;
    while ((1ull << s) < div) ++s;
    m = static_cast<uint32_t>(((1ull << 32) * ((1ull << s) - div)) / div + 1);
  }
  KVQ_DEVINL uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> s; }
};

// One tensor written: its input and its cache.
struct WriteTensor {
  const uint16_t *x;
  int64_t xs0, xs1, xs2;  // element strides of b, h, t
  void *codes;
  void *scales;
  int8_t *zps;
};

struct WriteArgs {
  WriteTensor t[2];       // K and V for kvq_write_kv; t[0] alone for kvq_write
  int ntens;
  int B, H, T, D, GPR;    // GPR: 32-element groups per row
  FastDiv div_T, div_H, div_G;
  const int32_t *slot_mapping;
  int64_t S;
  int32_t *err;
  uint32_t groups;  // groups of one tensor
  int round_scale;  // MX modes: KVQ_SCALE_CEIL, KVQ_SCALE_FLOOR or KVQ_SCALE_OCP
};

constexpr int kThreads = 256;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: v + kMagic holds rne(v) in its low mantissa bits

// E4M3 / E2M1 conversion on the hardware cvt (round-to-nearest-even,
// saturating to the largest finite value).  PTX puts the FIRST source in the
// UPPER half, so the element that must land low is passed second.
KVQ_DEVINL uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

KVQ_DEVINL uint32_t e5m2x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
template <bool E5>
KVQ_DEVINL uint32_t fp8x2(float lo, float hi) {
  return E5 ? e5m2x2(lo, hi) : e4m3x2(lo, hi);
}

KVQ_DEVINL uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6, float v7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// ceil(log2 s) + 127 for a finite s >= 0, from the binary32 fields, clamped to
// [0, 254]; s == 0 gives 0.  (Smallest power of two not below s, as E8M0.)
KVQ_DEVINL int e8m0_ceil(float s) {
  const uint32_t u = __float_as_uint(s);
  if (u == 0) return 0;
  const int E = static_cast<int>(u >> 23);
  const uint32_t M = u & 0x7FFFFFu;
  int l;
  if (E > 0)
    l = E - 127 + (M != 0 ? 1 : 0);
  else
    l = -149 + (32 - __clz(static_cast<int>(M - 1)));  // subnormal: ceil(log2 M) - 149
  const int e = l + 127;
  return e < 0 ? 0 : (e > 254 ? 254 : e);
}

// floor(log2 s) + 127 for a finite s >= 0, clamped to [0, 254]; s == 0 gives 0.
// (Largest power of two not above s, as E8M0.)
KVQ_DEVINL int e8m0_floor(float s) {
  const uint32_t u = __float_as_uint(s);
  if (u == 0) return 0;
  const int E = static_cast<int>(u >> 23);
  if (E == 0) return 0;  // subnormal: below 2^-126, clamped
  return E > 254 ? 254 : E;  // floor(log2 s) + 127 is the biased exponent field
}

// The OCP MX v1.0 shared exponent floor(log2 amax) - emax + 127 for a finite
// amax >= 0, clamped to [0, 254]; amax == 0 gives 0.
KVQ_DEVINL int e8m0_ocp(float amax, int emax) {
  const uint32_t u = __float_as_uint(amax);
  if (u == 0) return 0;
  const int E = static_cast<int>(u >> 23);
  const int l = E > 0 ? E - 127 : (31 - __clz(static_cast<int>(u & 0x7FFFFFu))) - 149;  // floor(log2 amax)
  const int e = l - emax + 127;
  return e < 0 ? 0 : (e > 254 ? 254 : e);
}

// 2^(127 - e) as a binary32 (exact for e in [0, 254]; e = 254 is subnormal).
KVQ_DEVINL float e8m0_inverse(int e) {
  const int k = 127 - e;  // in [-127, 127]
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(1u << 22);
}

// Locate group g: row (b, h, t) with t fastest, and the group index in the row.
KVQ_DEVINL void group_coords(const WriteArgs &a, uint32_t g, int &b, int &h, int &t, int &gi) {
  const uint32_t row = a.div_G.div(g);
  gi = static_cast<int>(g - row * a.div_G.d);
  const uint32_t bh = a.div_T.div(row);
  t = static_cast<int>(row - bh * a.div_T.d);
  const uint32_t bq = a.div_H.div(bh);
  h = static_cast<int>(bh - bq * a.div_H.d);
  b = static_cast<int>(bq);
}

// x / s correctly rounded, for two x, by Markstein's correction of x * rcp
// (rcp = RN(1 / s); IBM J. Res. Develop. 34(1), 1990): the residual
// s * q0 - x is exact in one FMA and RN(q0 - r * rcp) is the correctly rounded
// quotient unless x or the quotient is subnormal (there both stay within an ulp
// or two, with the same sign).  Taking the residual as s * q0 - x keeps the sign
// of a zero x: q0 - (+0) * rcp = -0 for x = -0, as -0 / s is.
KVQ_DEVINL float2 div2_markstein(float2 x, float s, float rcp) {
  const float2 q0 = __fmul2_rn(x, make_float2(rcp, rcp));
  const float2 r = __ffma2_rn(q0, make_float2(s, s), make_float2(-x.x, -x.y));
  return __ffma2_rn(r, make_float2(-rcp, -rcp), q0);
}
// Groups with amax at least this use div2_markstein: the scale (amax / Q_MAX,
// Q_MAX <= 57344) is then a normal float with a finite reciprocal, and a
// subnormal x has a quotient below 2^-50, far under half the smallest FP8 or
// integer step, so its code is 0 however it is rounded.
constexpr float kMarksteinMin = 0x1p-60f;

// Low bytes of four floats that hold integers in their low mantissa bits.
KVQ_DEVINL uint32_t pack_low_bytes(float a, float b, float c, float d) {
  const uint32_t ab = __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040u);
  const uint32_t cd = __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040u);
  return __byte_perm(ab, cd, 0x5410u);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads) write_kernel(const __grid_constant__ WriteArgs a) {
  // launched as a programmatic dependent: read nothing before the kernel ahead has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the grid fits one wave, so every CTA is resident by now: let the next kernel's launch
  // (a programmatic dependent, which in turn waits for this grid to complete) start
  asm volatile("griddepcontrol.launch_dependents;");
  const uint32_t stride = gridDim.x * kThreads;
  // Every lane of a warp runs the loop the same number of times (the bound is
  // rounded up to whole warps), so the int8 mode's row shuffles see the whole
  // warp.  With two tensors the V groups follow the K groups; a row never
  // straddles the two (groups is a multiple of the groups per row).
  const uint32_t all = a.groups * static_cast<uint32_t>(a.ntens);
  const uint32_t total = (all + 31u) & ~31u;
  for (uint32_t gg = blockIdx.x * kThreads + threadIdx.x; gg < total; gg += stride) {
    const int ti = gg >= a.groups ? 1 : 0;
    const uint32_t g = gg - (ti ? a.groups : 0u);
    const WriteTensor &wt = a.t[ti];
    int b = 0, h = 0, t = 0, gi = 0, slot = -1;
    // The group's x is loaded together with its slot, not after it: the two loads'
    // latencies overlap, at the price of reading the x of skipped tokens too.
    uint32_t wx[16];  // 32 bf16 values, element 2j in the low half of wx[j]
#pragma unroll
    for (int j = 0; j < 16; ++j) wx[j] = 0u;
    if (gg < all) {
      group_coords(a, g, b, h, t, gi);
      const int s = __ldg(a.slot_mapping + static_cast<int64_t>(b) * a.T + t);
      const uint4 *p =
          reinterpret_cast<const uint4 *>(wt.x + b * wt.xs0 + h * wt.xs1 + static_cast<int64_t>(t) * wt.xs2 + gi * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 c = __ldg(p + k);
        wx[4 * k] = c.x;
        wx[4 * k + 1] = c.y;
        wx[4 * k + 2] = c.z;
        wx[4 * k + 3] = c.w;
      }
      if (s != -1 && (s < 0 || s >= a.S)) {
        if (gi == 0) report(a.err, KVQ_ERR_SLOT_RANGE);
      } else {
        slot = s;
      }
    }
    if (slot < 0) {  // skipped: the int8 mode still shuffles row statistics, over zeros
#pragma unroll
      for (int j = 0; j < 16; ++j) wx[j] = 0u;
    }
    const int64_t r = (static_cast<int64_t>(b) * a.H + h) * a.S + (slot < 0 ? 0 : slot);

    if constexpr (MODE == KVQ_MODE_INT8_AFFINE || MODE == KVQ_MODE_INT4_AFFINE) {
      // int8 (mode 0): codes [-128, 127]; TQ4 (mode 7): codes [0, 15], two per byte
      constexpr bool Q4 = MODE == KVQ_MODE_INT4_AFFINE;
      constexpr float kLevels = Q4 ? 15.0f : 255.0f, kLo = Q4 ? 0.0f : -128.0f, kHi = Q4 ? 15.0f : 127.0f;
      // mn = min(0, min x), mx = max(0, max x) over the row: exact, order-free,
      // taken two bf16 at a time
      __nv_bfloat162 mn2 = __float2bfloat162_rn(0.0f), mx2 = mn2;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const __nv_bfloat162 x2 = *reinterpret_cast<const __nv_bfloat162 *>(&wx[j]);
        mn2 = __hmin2(mn2, x2);
        mx2 = __hmax2(mx2, x2);
      }
      float mn = fminf(__low2float(mn2), __high2float(mn2));
      float mx = fmaxf(__low2float(mx2), __high2float(mx2));
      for (int o = a.GPR >> 1; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (slot < 0) continue;
      float scale = __fdiv_rn(__fsub_rn(mx, mn), kLevels);
      if (scale < FLT_EPSILON) scale = FLT_EPSILON;
      int zp = static_cast<int>(kLo) - __float2int_rn(__fdiv_rn(mn, scale));
      zp = zp < static_cast<int>(kLo) ? static_cast<int>(kLo) : (zp > static_cast<int>(kHi) ? static_cast<int>(kHi) : zp);
      // q = clamp(rne(x / scale) + zp): the quotient x / scale correctly rounded by
      // Markstein's correction (IBM J. Res. Develop. 34(1), 1990) of q0 = x * rcp
      // with rcp = RN(1 / scale): r = x - scale * q0 is exact (one FMA), and
      // RN(q0 + r * rcp) is RN(x / scale) for every x of the row except subnormal
      // ones, whose quotients lie far below 0.5 and give the code zp either way.
      // Adding 1.5 * 2^23 then rounds it to an integer (rne), the zero point is an
      // exact integer add, and the clamp is exact; the code is the low mantissa byte.
      const float rcp = __frcp_rn(scale);
      const float2 mg2 = make_float2(kMagic, kMagic), zp2 = make_float2(static_cast<float>(zp), static_cast<float>(zp));
      const float t_lo = kMagic + kLo, t_hi = kMagic + kHi;
      float t2[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 q = div2_markstein(make_float2(bf16lo(wx[j]), bf16hi(wx[j])), scale, rcp);
        const float2 t = __fadd2_rn(__fadd2_rn(q, mg2), zp2);
        t2[2 * j] = fminf(fmaxf(t.x, t_lo), t_hi);
        t2[2 * j + 1] = fminf(fmaxf(t.y, t_lo), t_hi);
      }
      if constexpr (Q4) {
        // the code sits in the low mantissa bits of t2; element 2i goes to the low nibble of byte i
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t acc = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) acc |= (__float_as_uint(t2[8 * k + j]) & 0xFu) << (4 * j);
          w[k] = acc;
        }
        *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(wt.codes) + r * (a.D >> 1) + gi * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      } else {
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = pack_low_bytes(t2[4 * k], t2[4 * k + 1], t2[4 * k + 2], t2[4 * k + 3]);
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<int8_t *>(wt.codes) + r * a.D + gi * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      if (gi == 0) {
        static_cast<float *>(wt.scales)[r] = scale;
        wt.zps[r] = static_cast<int8_t>(zp);
      }
    } else {
      if (slot < 0) continue;
      __nv_bfloat162 am2 = __float2bfloat162_rn(0.0f);
#pragma unroll
      for (int j = 0; j < 16; ++j) am2 = __hmax2(am2, __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&wx[j])));
      const float amax = fmaxf(__low2float(am2), __high2float(am2));
      float v[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[2 * j] = bf16lo(wx[j]);
        v[2 * j + 1] = bf16hi(wx[j]);
      }
      const int64_t sidx = r * a.GPR + gi;  // scale index
      if constexpr (MODE == KVQ_MODE_FP8_E4M3 || MODE == KVQ_MODE_FP8_E5M2) {
        constexpr bool E5 = MODE == KVQ_MODE_FP8_E5M2;
        const float scale = __fdiv_rn(amax, E5 ? 57344.0f : 448.0f);
        uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (amax >= kMarksteinMin) {  // the correctly rounded quotient, then one cvt per pair
          const float rcp = __frcp_rn(scale);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float2 y0 = div2_markstein(make_float2(v[4 * k], v[4 * k + 1]), scale, rcp);
            const float2 y1 = div2_markstein(make_float2(v[4 * k + 2], v[4 * k + 3]), scale, rcp);
            w[k] = fp8x2<E5>(y0.x, y0.y) | (fp8x2<E5>(y1.x, y1.y) << 16);
          }
        } else if (amax != 0.0f) {  // a group of tiny values: exact division
#pragma unroll
          for (int k = 0; k < 8; ++k)
            w[k] = fp8x2<E5>(__fdiv_rn(v[4 * k], scale), __fdiv_rn(v[4 * k + 1], scale)) |
                   (fp8x2<E5>(__fdiv_rn(v[4 * k + 2], scale), __fdiv_rn(v[4 * k + 3], scale)) << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(wt.codes) + r * a.D + gi * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        static_cast<float *>(wt.scales)[sidx] = scale;
      } else if constexpr (MODE == KVQ_MODE_INT8_SYM) {
        // q = clamp(rne(x / scale), -127, 127), scale = amax / 127: the correctly
        // rounded quotient, rounded to an integer by the 1.5 * 2^23 add, clamped
        const float scale = __fdiv_rn(amax, 127.0f);
        float t2[32];
        if (amax >= kMarksteinMin) {
          const float rcp = __frcp_rn(scale);
          const float2 mg2 = make_float2(kMagic, kMagic);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 t = __fadd2_rn(div2_markstein(make_float2(v[2 * j], v[2 * j + 1]), scale, rcp), mg2);
            t2[2 * j] = fminf(fmaxf(t.x, kMagic - 127.0f), kMagic + 127.0f);
            t2[2 * j + 1] = fminf(fmaxf(t.y, kMagic - 127.0f), kMagic + 127.0f);
          }
        } else {  // zero or a group of tiny values: exact division
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            int q = amax != 0.0f ? __float2int_rn(__fdiv_rn(v[i], scale)) : 0;
            q = q < -127 ? -127 : (q > 127 ? 127 : q);
            t2[i] = __uint_as_float(0x4B400000u + static_cast<uint32_t>(q));
          }
        }
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = pack_low_bytes(t2[4 * k], t2[4 * k + 1], t2[4 * k + 2], t2[4 * k + 3]);
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(wt.codes) + r * a.D + gi * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        static_cast<float *>(wt.scales)[sidx] = scale;
      } else {
        constexpr bool MX8 = MODE == KVQ_MODE_MXFP8 || MODE == KVQ_MODE_MXFP8_E5M2;
        constexpr bool E5 = MODE == KVQ_MODE_MXFP8_E5M2;
        constexpr float kQmax = MX8 ? (E5 ? 57344.0f : 448.0f) : 6.0f;
        constexpr int kEmax = MX8 ? (E5 ? 15 : 8) : 2;  // the element format's largest exponent
        const float s_ = __fdiv_rn(amax, kQmax);
        const int e = a.round_scale == KVQ_SCALE_OCP    ? e8m0_ocp(amax, kEmax)
                      : a.round_scale == KVQ_SCALE_CEIL ? e8m0_ceil(s_)
                                                        : e8m0_floor(s_);
        const float inv = e8m0_inverse(e);  // x / 2^(e-127) == x * 2^(127-e), exactly rounded
        float y[32];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 yy = __fmul2_rn(make_float2(v[i], v[i + 1]), make_float2(inv, inv));
          y[i] = yy.x;
          y[i + 1] = yy.y;
        }
        if constexpr (MX8) {
          uint32_t w[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            w[k] = amax != 0.0f ? (fp8x2<E5>(y[4 * k], y[4 * k + 1]) | (fp8x2<E5>(y[4 * k + 2], y[4 * k + 3]) << 16))
                                : 0u;
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(wt.codes) + r * a.D + gi * 32);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            w[k] = amax != 0.0f ? e2m1x8(y[8 * k], y[8 * k + 1], y[8 * k + 2], y[8 * k + 3], y[8 * k + 4],
                                         y[8 * k + 5], y[8 * k + 6], y[8 * k + 7])
                                : 0u;
          *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(wt.codes) + r * (a.D >> 1) + gi * 16) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        static_cast<uint8_t *>(wt.scales)[sidx] = static_cast<uint8_t>(e);
      }
    }
  }
}

template <int MODE>
int launch_write(const WriteArgs &a, cudaStream_t stream) {
  const int64_t blocks_needed = (static_cast<int64_t>(a.groups) * a.ntens + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;  // 8 x 256 threads = a full SM
  const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, write_kernel<MODE>, a) != cudaSuccess) return KVQ_ECUDA;
  return launch_status();
}

}  // namespace
}  // namespace kvq

namespace kvq {
namespace {
// Checks shared by kvq_write and kvq_write_kv; returns KVQ_OK or the error.
int check_common(int mode, int B, int H, int T, int D, int64_t num_slots) {
  if (mode < KVQ_MODE_INT8_AFFINE || mode > KVQ_MODE_INT4_AFFINE) return KVQ_EINVAL;
  if (B < 0 || H < 0 || T < 0 || D <= 0 || num_slots <= 0 || num_slots > INT32_MAX) return KVQ_EINVAL;
  if (mode == KVQ_MODE_INT8_AFFINE || mode == KVQ_MODE_INT4_AFFINE) {
    if (D != 64 && D != 128 && D != 256) return KVQ_EUNSUPPORTED;
  } else {
    if (D % 32 != 0 || D > 8192) return KVQ_EUNSUPPORTED;
  }
  return KVQ_OK;
}

// Checks of one tensor's input and cache; fills `t`.
int check_tensor(int mode, const void *x, const int64_t *x_strides, void *codes, void *scales, int8_t *zero_points,
                 WriteTensor &t) {
  if (!x || !x_strides || !codes || !scales) return KVQ_EINVAL;
  if ((mode == KVQ_MODE_INT8_AFFINE || mode == KVQ_MODE_INT4_AFFINE) && !zero_points) return KVQ_EINVAL;
  // every row start 16-byte aligned: base aligned and strides multiples of 8 elements
  if (!aligned16(x) || !aligned16(codes)) return KVQ_EINVAL;
  for (int i = 0; i < 3; ++i)
    if (x_strides[i] < 0 || (x_strides[i] & 7) != 0) return KVQ_EINVAL;
  // float scales (modes 0, 1, 4, 6, 7) must be 4-byte aligned; E8M0 scales are bytes
  const bool f32_scales = mode == KVQ_MODE_INT8_AFFINE || mode == KVQ_MODE_FP8_E4M3 || mode == KVQ_MODE_FP8_E5M2 ||
                          mode == KVQ_MODE_INT8_SYM || mode == KVQ_MODE_INT4_AFFINE;
  if (f32_scales && (reinterpret_cast<uintptr_t>(scales) & 3u)) return KVQ_EINVAL;
  t.x = static_cast<const uint16_t *>(x);
  t.xs0 = x_strides[0];
  t.xs1 = x_strides[1];
  t.xs2 = x_strides[2];
  t.codes = codes;
  t.scales = scales;
  t.zps = zero_points;
  return KVQ_OK;
}

int write_impl(int mode, int round_scale, int B, int H, int T, int D, const int32_t *slot_mapping, int64_t num_slots,
               const WriteTensor *tens, int ntens, int32_t *err_word, void *stream) {
  // group indices use 32-bit arithmetic
  const int64_t groups = static_cast<int64_t>(B) * H * T * (D / 32);
  if (groups * ntens >= (int64_t(1) << 31)) return KVQ_EUNSUPPORTED;
  WriteArgs a;
  a.t[0] = tens[0];
  a.t[1] = ntens > 1 ? tens[1] : tens[0];
  a.ntens = ntens;
  a.B = B;
  a.H = H;
  a.T = T;
  a.D = D;
  a.GPR = D / 32;
  a.div_T = FastDiv(static_cast<uint32_t>(T));
  a.div_H = FastDiv(static_cast<uint32_t>(H));
  a.div_G = FastDiv(static_cast<uint32_t>(D / 32));
  a.slot_mapping = slot_mapping;
  a.S = num_slots;
  a.err = err_word;
  a.groups = static_cast<uint32_t>(groups);
  if (round_scale < KVQ_SCALE_FLOOR || round_scale > KVQ_SCALE_OCP) return KVQ_EINVAL;
  a.round_scale = round_scale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (mode) {
    case KVQ_MODE_INT8_AFFINE: return launch_write<KVQ_MODE_INT8_AFFINE>(a, s);
    case KVQ_MODE_FP8_E4M3: return launch_write<KVQ_MODE_FP8_E4M3>(a, s);
    case KVQ_MODE_MXFP8: return launch_write<KVQ_MODE_MXFP8>(a, s);
    case KVQ_MODE_MXFP4: return launch_write<KVQ_MODE_MXFP4>(a, s);
    case KVQ_MODE_FP8_E5M2: return launch_write<KVQ_MODE_FP8_E5M2>(a, s);
    case KVQ_MODE_MXFP8_E5M2: return launch_write<KVQ_MODE_MXFP8_E5M2>(a, s);
    case KVQ_MODE_INT8_SYM: return launch_write<KVQ_MODE_INT8_SYM>(a, s);
    default: return launch_write<KVQ_MODE_INT4_AFFINE>(a, s);
  }
}
}  // namespace
}  // namespace kvq

extern "C" int kvq_write(int mode, int round_scale, const void *x, int B, int H, int T, int D,
                         const int64_t *x_strides, const int32_t *slot_mapping, int64_t num_slots, void *codes,
                         void *scales, int8_t *zero_points, int32_t *err_word, void *stream) {
  using namespace kvq;
  if (const int st = check_common(mode, B, H, T, D, num_slots)) return st;
  if (static_cast<int64_t>(B) * H * T == 0) return KVQ_OK;
  if (!slot_mapping) return KVQ_EINVAL;
  WriteTensor t;
  if (const int st = check_tensor(mode, x, x_strides, codes, scales, zero_points, t)) return st;
  return write_impl(mode, round_scale, B, H, T, D, slot_mapping, num_slots, &t, 1, err_word, stream);
}

extern "C" int kvq_write_kv(int mode, int round_scale, const void *k, const void *v, int B, int H, int T, int D,
                            const int64_t *k_strides, const int64_t *v_strides, const int32_t *slot_mapping,
                            int64_t num_slots, void *k_codes, void *k_scales, int8_t *k_zero_points, void *v_codes,
                            void *v_scales, int8_t *v_zero_points, int32_t *err_word, void *stream) {
  using namespace kvq;
  if (const int st = check_common(mode, B, H, T, D, num_slots)) return st;
  if (static_cast<int64_t>(B) * H * T == 0) return KVQ_OK;
  if (!slot_mapping) return KVQ_EINVAL;
  WriteTensor t[2];
  if (const int st = check_tensor(mode, k, k_strides, k_codes, k_scales, k_zero_points, t[0])) return st;
  if (const int st = check_tensor(mode, v, v_strides, v_codes, v_scales, v_zero_points, t[1])) return st;
  return write_impl(mode, round_scale, B, H, T, D, slot_mapping, num_slots, t, 2, err_word, stream);
}
