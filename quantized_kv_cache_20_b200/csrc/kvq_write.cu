// kvq_write.cu -- the quantized KV-cache write (quantize + scatter by slot).
//
// One streaming kernel per mode.  Work is split into units: a (token, head)
// row for the int8 affine mode (ExecuTorch PR 24473, Summary: per token and
// head), a 32-element group for the block modes (IndexerQuantCache page,
// 计算公式: scale_g = max|x_g| / Q_MAX, q_i = round(x_i / scale_g)).  Each unit
// is covered by LANES consecutive lanes, each owning one 16-byte chunk of 8
// bf16 values, so a warp reads 512 contiguous bytes per load instruction and
// reduces with xor-shuffles inside the unit.  UNROLL units per lane are loaded
// before any arithmetic, to keep enough bytes in flight to cover HBM latency.
// Tokens whose slot is -1 are skipped before their x is read (IndexerQuantCache
// page, 约束说明), so skipped rows cost no input bandwidth.
//
// The arithmetic is binary32 with explicit round-to-nearest-even intrinsics
// (__fdiv_rn, __fsub_rn, __float2int_rn) in the order the definitions state,
// so results are bit-reproducible and independent of contraction.
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

struct WriteArgs {
  const uint16_t *x;
  int64_t xs0, xs1, xs2;  // element strides of b, h, t
  int B, H, T, D;
  FastDiv div_T, div_H, div_G;  // by T, by H, by groups per row
  const int32_t *slot_mapping;
  int64_t S;
  void *codes;
  void *scales;
  int8_t *zps;
  int32_t *err;
  int64_t units;  // total units
};

constexpr int kThreads = 256;

// --- E4M3 / E2M1 conversion on the hardware cvt (round-to-nearest-even,
// saturating to the largest finite value).  PTX puts the FIRST source in the
// UPPER half, so the element that must land low is passed second.
KVQ_DEVINL uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// 8 floats -> 4 bytes of E2M1 pairs (element 2i in the low nibble of byte i).
KVQ_DEVINL uint32_t e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
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

// 2^(127 - e) as a binary32 (exact for e in [0, 254]; e = 254 is subnormal).
KVQ_DEVINL float e8m0_inverse(int e) {
  const int k = 127 - e;  // in [-127, 127]
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(1u << 22);
}

// rne(x / scale) as an int, bit-identical to __float2int_rn(__fdiv_rn(x, scale)):
// y = x * rcp (rcp = correctly rounded 1/scale) is within 3 ulp of the
// correctly rounded quotient q, so whenever y is more than 2^-12 away from a
// half-integer (|y| <= 512 here), y and q round to the same integer.  Otherwise
// (about 1 element in 4000) the exact division decides.
KVQ_DEVINL int div_rint(float x, float scale, float rcp) {
  const float y = __fmul_rn(x, rcp);
  const float r = rintf(y);
  if (fabsf(__fsub_rn(y, r)) < 0.5f - 0x1p-12f && fabsf(y) <= 512.0f) return static_cast<int>(r);
  return __float2int_rn(__fdiv_rn(x, scale));
}

// E4M3 codes of (lo / scale, hi / scale), bit-identical to converting the
// correctly rounded quotients: y = x * rcp is within 3 ulp of the quotient, so
// if the codes of y - d and y + d (d = 2^-20 |y|) agree, no E4M3 rounding
// boundary lies between y and the quotient.  Otherwise divide exactly.
KVQ_DEVINL uint32_t e4m3x2(float lo, float hi);
KVQ_DEVINL uint32_t e4m3x2_div(float x0, float x1, float scale, float rcp) {
  const float y0 = __fmul_rn(x0, rcp), y1 = __fmul_rn(x1, rcp);
  const float d0 = fabsf(y0) * 0x1p-20f, d1 = fabsf(y1) * 0x1p-20f;
  const uint32_t c = e4m3x2(y0, y1);
  if (e4m3x2(y0 - d0, y1 - d1) == c && e4m3x2(y0 + d0, y1 + d1) == c) return c;
  return e4m3x2(__fdiv_rn(x0, scale), __fdiv_rn(x1, scale));
}

KVQ_DEVINL void unpack8(const uint4 &c, float (&v)[8]) {
  v[0] = bf16lo(c.x); v[1] = bf16hi(c.x);
  v[2] = bf16lo(c.y); v[3] = bf16hi(c.y);
  v[4] = bf16lo(c.z); v[5] = bf16hi(c.z);
  v[6] = bf16lo(c.w); v[7] = bf16hi(c.w);
}

// Locate unit u: for the affine mode a unit is a row (b, h, t) with t fastest;
// for block modes it is group `gi` of that row.
template <int MODE>
KVQ_DEVINL void unit_coords(const WriteArgs &a, uint32_t u, int &b, int &h, int &t, int &gi) {
  uint32_t row = u;
  gi = 0;
  if (MODE != KVQ_MODE_INT8_AFFINE) {
    row = a.div_G.div(u);
    gi = static_cast<int>(u - row * a.div_G.d);
  }
  const uint32_t bh = a.div_T.div(row);
  t = static_cast<int>(row - bh * a.div_T.d);
  const uint32_t bq = a.div_H.div(bh);
  h = static_cast<int>(bh - bq * a.div_H.d);
  b = static_cast<int>(bq);
}

// LANES lanes per unit; UNROLL units per lane per pass.
template <int MODE, int LANES, int UNROLL>
__global__ void __launch_bounds__(kThreads) write_kernel(const WriteArgs a) {
  constexpr int UPW = 32 / LANES;  // units per warp per unroll step
  const int lane = threadIdx.x & 31;
  const int sub = lane % LANES;
  const int uw = lane / LANES;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;

  for (int64_t base = warp * (UPW * UNROLL); base < a.units; base += nwarps * (UPW * UNROLL)) {
    int64_t unit[UNROLL];
    int slot[UNROLL];
    int bb[UNROLL], hh[UNROLL], gg[UNROLL];
    uint4 raw[UNROLL];
    // Phase 1: slots (one per unit; the same address across the unit's lanes).
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
      unit[k] = base + k * UPW + uw;
      slot[k] = -1;
      bb[k] = hh[k] = gg[k] = 0;
      if (unit[k] < a.units) {
        int t;
        unit_coords<MODE>(a, static_cast<uint32_t>(unit[k]), bb[k], hh[k], t, gg[k]);
        const int s = __ldg(a.slot_mapping + static_cast<int64_t>(bb[k]) * a.T + t);
        if (s != -1 && (s < 0 || s >= a.S)) {
          if (sub == 0) report(a.err, KVQ_ERR_SLOT_RANGE);
          slot[k] = -1;
        } else {
          slot[k] = s;
        }
        if (slot[k] >= 0) {
          const uint16_t *row = a.x + bb[k] * a.xs0 + hh[k] * a.xs1 + static_cast<int64_t>(t) * a.xs2;
          raw[k] = ld_stream_v4(row + gg[k] * 32 + sub * 8);
        }
      }
    }
    // Phase 2: quantize and store.
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
      float v[8];
      if (slot[k] >= 0)
        unpack8(raw[k], v);
      else
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
      const int64_t r = (static_cast<int64_t>(bb[k]) * a.H + hh[k]) * a.S + (slot[k] < 0 ? 0 : slot[k]);

      if constexpr (MODE == KVQ_MODE_INT8_AFFINE) {
        // mn = min(0, min x), mx = max(0, max x): exact, order-free.
        float mn = 0.0f, mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          mn = v[i] < mn ? v[i] : mn;
          mx = v[i] > mx ? v[i] : mx;
        }
#pragma unroll
        for (int o = LANES / 2; o > 0; o >>= 1) {
          const float omn = __shfl_xor_sync(0xffffffffu, mn, o);
          const float omx = __shfl_xor_sync(0xffffffffu, mx, o);
          mn = omn < mn ? omn : mn;
          mx = omx > mx ? omx : mx;
        }
        float scale = __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
        if (scale < FLT_EPSILON) scale = FLT_EPSILON;
        int zp = -128 - __float2int_rn(__fdiv_rn(mn, scale));
        zp = zp < -128 ? -128 : (zp > 127 ? 127 : zp);
        const float rcp = __frcp_rn(scale);
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          int q = div_rint(v[i], scale, rcp) + zp;
          q = q < -128 ? -128 : (q > 127 ? 127 : q);
          w[i >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (i & 3));
        }
        if (slot[k] >= 0) {
          int8_t *crow = static_cast<int8_t *>(a.codes) + r * a.D;
          st_v2(crow + sub * 8, w[0], w[1]);
          if (sub == 0) {
            static_cast<float *>(a.scales)[r] = scale;
            a.zps[r] = static_cast<int8_t>(zp);
          }
        }
      } else {
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int ngroups = a.D >> 5;
        const int64_t gidx = r * ngroups + gg[k];  // scale index
        if constexpr (MODE == KVQ_MODE_FP8_E4M3) {
          const float scale = __fdiv_rn(amax, 448.0f);
          uint32_t w0 = 0u, w1 = 0u;
          if (amax != 0.0f) {
            const float rcp = __frcp_rn(scale);
            w0 = e4m3x2_div(v[0], v[1], scale, rcp) | (e4m3x2_div(v[2], v[3], scale, rcp) << 16);
            w1 = e4m3x2_div(v[4], v[5], scale, rcp) | (e4m3x2_div(v[6], v[7], scale, rcp) << 16);
          }
          if (slot[k] >= 0) {
            uint8_t *crow = static_cast<uint8_t *>(a.codes) + r * a.D;
            st_v2(crow + gg[k] * 32 + sub * 8, w0, w1);
            if (sub == 0) static_cast<float *>(a.scales)[gidx] = scale;
          }
        } else {
          constexpr float kQmax = (MODE == KVQ_MODE_MXFP8) ? 448.0f : 6.0f;
          const int e = e8m0_ceil(__fdiv_rn(amax, kQmax));
          const float inv = e8m0_inverse(e);  // x / 2^(e-127) == x * 2^(127-e), exactly rounded
          float q[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[i], inv);
          if constexpr (MODE == KVQ_MODE_MXFP8) {
            uint32_t w0 = 0u, w1 = 0u;
            if (amax != 0.0f) {
              w0 = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
              w1 = e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16);
            }
            if (slot[k] >= 0) {
              uint8_t *crow = static_cast<uint8_t *>(a.codes) + r * a.D;
              st_v2(crow + gg[k] * 32 + sub * 8, w0, w1);
            }
          } else {
            const uint32_t w = (amax != 0.0f) ? e2m1x8(q) : 0u;
            if (slot[k] >= 0) {
              uint8_t *crow = static_cast<uint8_t *>(a.codes) + r * (a.D >> 1);
              st_u32(crow + gg[k] * 16 + sub * 4, w);
            }
          }
          if (slot[k] >= 0 && sub == 0) static_cast<uint8_t *>(a.scales)[gidx] = static_cast<uint8_t>(e);
        }
      }
    }
  }
}

template <int MODE, int LANES, int UNROLL>
int launch_write(const WriteArgs &a, cudaStream_t stream) {
  constexpr int UPW = 32 / LANES;
  const int64_t warps_needed = (a.units + UPW * UNROLL - 1) / (UPW * UNROLL);
  const int64_t blocks_needed = (warps_needed + (kThreads / 32) - 1) / (kThreads / 32);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;  // 8 x 256 threads = full SM
  const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  write_kernel<MODE, LANES, UNROLL><<<grid, kThreads, 0, stream>>>(a);
  return launch_status();
}

}  // namespace
}  // namespace kvq

extern "C" int kvq_write(int mode, int round_scale, const void *x, int B, int H, int T, int D,
                         const int64_t *x_strides, const int32_t *slot_mapping, int64_t num_slots, void *codes,
                         void *scales, int8_t *zero_points, int32_t *err_word, void *stream) {
  using namespace kvq;
  if (mode < KVQ_MODE_INT8_AFFINE || mode > KVQ_MODE_MXFP4) return KVQ_EINVAL;
  if (B < 0 || H < 0 || T < 0 || D <= 0 || num_slots <= 0 || num_slots > INT32_MAX) return KVQ_EINVAL;
  if (mode == KVQ_MODE_INT8_AFFINE) {
    if (D != 64 && D != 128 && D != 256) return KVQ_EUNSUPPORTED;
  } else {
    if (D % 32 != 0 || D > 8192) return KVQ_EUNSUPPORTED;
    if (mode == KVQ_MODE_MXFP8 && !round_scale) return KVQ_EUNSUPPORTED;
  }
  if (static_cast<int64_t>(B) * H * T == 0) return KVQ_OK;
  if (!x || !x_strides || !slot_mapping || !codes || !scales) return KVQ_EINVAL;
  if (mode == KVQ_MODE_INT8_AFFINE && !zero_points) return KVQ_EINVAL;
  // every row start 16-byte aligned: base aligned and strides multiples of 8 elements
  if (!aligned16(x) || !aligned16(codes)) return KVQ_EINVAL;
  for (int i = 0; i < 3; ++i)
    if (x_strides[i] < 0 || (x_strides[i] & 7) != 0) return KVQ_EINVAL;
  // float scales (modes 0 and 1) must be 4-byte aligned; E8M0 scales are bytes
  if ((mode == KVQ_MODE_INT8_AFFINE || mode == KVQ_MODE_FP8_E4M3) && (reinterpret_cast<uintptr_t>(scales) & 3u))
    return KVQ_EINVAL;
  // unit indices use 32-bit arithmetic
  if (static_cast<int64_t>(B) * H * T * (mode == KVQ_MODE_INT8_AFFINE ? 1 : D / 32) >= (int64_t(1) << 31))
    return KVQ_EUNSUPPORTED;

  WriteArgs a;
  a.x = static_cast<const uint16_t *>(x);
  a.xs0 = x_strides[0];
  a.xs1 = x_strides[1];
  a.xs2 = x_strides[2];
  a.B = B;
  a.H = H;
  a.T = T;
  a.D = D;
  a.div_T = FastDiv(static_cast<uint32_t>(T));
  a.div_H = FastDiv(static_cast<uint32_t>(H));
  a.div_G = FastDiv(static_cast<uint32_t>(mode == KVQ_MODE_INT8_AFFINE ? 1 : D / 32));
  a.slot_mapping = slot_mapping;
  a.S = num_slots;
  a.codes = codes;
  a.scales = scales;
  a.zps = zero_points;
  a.err = err_word;
  const int64_t rows = static_cast<int64_t>(B) * H * T;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (mode) {
    case KVQ_MODE_INT8_AFFINE:
      a.units = rows;
      if (D == 64) return launch_write<KVQ_MODE_INT8_AFFINE, 8, 4>(a, s);
      if (D == 128) return launch_write<KVQ_MODE_INT8_AFFINE, 16, 4>(a, s);
      return launch_write<KVQ_MODE_INT8_AFFINE, 32, 4>(a, s);
    case KVQ_MODE_FP8_E4M3:
      a.units = rows * (D / 32);
      return launch_write<KVQ_MODE_FP8_E4M3, 4, 4>(a, s);
    case KVQ_MODE_MXFP8:
      a.units = rows * (D / 32);
      return launch_write<KVQ_MODE_MXFP8, 4, 4>(a, s);
    default:
      a.units = rows * (D / 32);
      return launch_write<KVQ_MODE_MXFP4, 4, 4>(a, s);
  }
}
