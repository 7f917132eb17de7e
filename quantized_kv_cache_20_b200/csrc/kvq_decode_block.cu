// kvq_decode_block.cu -- one-query (decode) attention over the per-32 block
// caches that kvq_write modes 1-6 produce.
//
// What it computes: the attention of kvq_decode_attn (abaddon
// src/attention_cache/mod.rs, trait KvCache, forward_attention; ExecuTorch PR
// 20351 commit notes on the device-side kv_len; ExecuTorch PR 24473, Summary,
// on the additive mask) with K and V dequantized from the IndexerQuantCache
// block format (计算公式: x ~ code * scale_g, one scale per 32 elements):
//   modes 1 / 4 / 6: E4M3 / E5M2 / int8 codes, float32 scales;
//   modes 2 / 5 / 3: E4M3 / E5M2 / E2M1 (two per byte) codes, E8M0 scales.
//
// Design (CUDA cores; the scales vary along the head dim, the contraction of
// q.k, so they are applied per 32-element group in fp32):
//  - Split-K: grid (splits, Hkv, B); a CTA takes a contiguous slot range of
//    one (b, kv head) for all G q heads (G <= 8), 8 warps x 32 slots at a time.
//  - Each warp stages its 32-slot tile (K and V codes and scales) into shared
//    memory with 16-byte asynchronous copies (cp.async), the next tile while it
//    works on the current one (two buffers for D <= 128, one for D = 256).
//  - q.k: lanes over the head dim.  Lane (g, sub) takes dims [16 sub, 16 sub +
//    16) -- inside one 32-element scale group -- of L = D/16 slots, with q in
//    registers (four heads per pass, fp32).  Codes are decoded two at a time
//    by the sm_100 cvt.rn.f16x2.{e4m3x2, e5m2x2, e2m1x2} conversions (exact),
//    the lane's partial is scaled by its group's scale, and a butterfly
//    reduce-scatter across the L lanes leaves each lane one slot's scores.
//  - p.v: lanes over the head dim (a V row per slot from the staged tile), p
//    broadcast through shared memory; online softmax per warp in the log2
//    domain (the running max is raised only when a score exceeds it by more
//    than 8).
//  - Warps combine through shared memory; each CTA writes its (m, l, O)
//    partial, and a merge kernel combines the splits in order.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_common.cuh"
#include "kvq_decode_blk.h"

namespace kvq {
namespace blk {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxG = 8;
constexpr float kLog2e = 1.4426950408889634f;

struct Args {
  const uint16_t *q;
  const uint8_t *kc, *vc;   // codes [B, Hkv, S, CB]
  const void *ks, *vs;      // scales [B, Hkv, S, D/32] (float or E8M0 bytes)
  const float *mask;        // nullable [S]
  const int32_t *kv_len;
  uint16_t *out;
  float *ws;                // partials [B, Hkv, splits, G, D + 2]
  int32_t *err;
  int64_t S;
  int B, Hq, Hkv, G, splits, span;  // span: slots per split (multiple of 32)
  float qscale;                     // sm_scale * log2(e)
};

template <int MODE>
struct Fmt {
  static constexpr bool FP4 = MODE == KVQ_MODE_MXFP4;
  static constexpr bool E5 = MODE == KVQ_MODE_FP8_E5M2 || MODE == KVQ_MODE_MXFP8_E5M2;
  static constexpr bool I8 = MODE == KVQ_MODE_INT8_SYM;
  static constexpr bool F32_SCALE = MODE == KVQ_MODE_FP8_E4M3 || MODE == KVQ_MODE_FP8_E5M2 || I8;
};

// Two codes (low byte first) -> float2, exact.
template <int MODE>
KVQ_DEVINL float2 decode2(uint32_t two) {
  if constexpr (Fmt<MODE>::I8) {
    return make_float2(static_cast<float>(static_cast<int8_t>(two & 0xFF)),
                       static_cast<float>(static_cast<int8_t>((two >> 8) & 0xFF)));
  } else if constexpr (Fmt<MODE>::FP4) {  // one byte, element 2i in the low nibble
    uint32_t h;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h) : "r"(two & 0xFF));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
  } else {
    uint32_t h;
    const uint16_t b = static_cast<uint16_t>(two & 0xFFFF);
    if constexpr (Fmt<MODE>::E5)
      asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"(b));
    else
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
  }
}


// 16-byte global -> shared copy that completes asynchronously (cp.async.cg).
KVQ_DEVINL void cp_async16(void *dst_smem, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}
KVQ_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
KVQ_DEVINL void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
KVQ_DEVINL void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

KVQ_DEVINL float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One warp's staged tile of 32 slots: K codes, K scales, V codes, V scales
// (each part 16-byte aligned); NBUF tiles per warp (two for D <= 128, so the
// next tile's copies overlap this tile's work).
template <int MODE, int D>
struct VTile {
  static constexpr int CB = Fmt<MODE>::FP4 ? D / 2 : D;
  static constexpr int SB = Fmt<MODE>::F32_SCALE ? 32 * (D / 32) * 4 : 32 * (D / 32);
  static constexpr int SBP = (SB + 15) / 16 * 16;
  static constexpr int KS = 32 * CB, VC = KS + SBP, VS = VC + 32 * CB;  // part offsets
  static constexpr int TB = VS + SBP;                                     // one tile
  static constexpr int NBUF = D == 256 ? 1 : 2;
  static constexpr int BYTES = NBUF * TB;                                 // one warp
};

// The scale of entry idx of a staged scale array (float, or E8M0 2^(e - 127)).
template <int MODE>
KVQ_DEVINL float staged_scale(const uint8_t *p, int idx) {
  if constexpr (Fmt<MODE>::F32_SCALE) {
    return reinterpret_cast<const float *>(p)[idx];
  } else {
    const int e = p[idx];
    return e >= 1 ? __uint_as_float(static_cast<uint32_t>(e) << 23) : __uint_as_float(1u << 22);
  }
}
template <int MODE, int D>
struct BlockTag {};  // names one decode_block_kernel instantiation for ensure_smem

template <int MODE, int D>
__global__ void __launch_bounds__(kThreads) decode_block_kernel(const Args a) {
  constexpr int CB = Fmt<MODE>::FP4 ? D / 2 : D;  // code bytes per slot
  constexpr int NGRP = D / 32;
  constexpr int DPL = D / 32;                     // head dims per lane in p.v
  constexpr bool F32S = Fmt<MODE>::F32_SCALE;
  __shared__ __align__(16) float q_s[kMaxG * D];
  __shared__ __align__(16) float p_s[kWarps][32][kMaxG];
  __shared__ float mc_s[kMaxG], lc_s[kMaxG];  // the CTA's combined state, warp by warp
  __shared__ __align__(16) float oc_s[kMaxG][D];
  // each warp's V tile (dynamic shared memory): codes of its 32 slots, then their scales
  extern __shared__ __align__(16) uint8_t vt_s[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = a.G;
  int kv = *a.kv_len;
  if (kv < 0 || kv > a.S) {
    if (tid == 0 && split == 0 && hk == 0 && b == 0) report(a.err, KVQ_ERR_KV_LEN_RANGE);
    kv = kv < 0 ? 0 : static_cast<int>(a.S);
  }
  const int s_begin = split * a.span, s_end = min(kv, s_begin + a.span);
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;

  // q for the G heads of this kv head, scaled into the log2 domain
  for (int e = tid; e < G * D; e += kThreads) {
    const int h = e / D, d = e - h * D;
    const uint16_t qb = a.q[(static_cast<int64_t>(b) * a.Hq + hk * G + h) * D + d];
    q_s[h * D + d] = __uint_as_float(static_cast<uint32_t>(qb) << 16) * a.qscale;
  }
  __syncthreads();

  float m[kMaxG], lsum[kMaxG], acc[kMaxG][DPL];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) {
    m[h] = -INFINITY;
    lsum[h] = 0.0f;
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[h][k] = 0.0f;
  }

  using TL = VTile<MODE, D>;
  uint8_t *wt = vt_s + warp * TL::BYTES;
  // issue the copies of the tile at slot bs into dst (rows up to the slab end
  // only: S % 16 == 0, so 16 or 32 rows)
  auto stage = [&](int bs, uint8_t *dst) {
    const int nrow = a.S - bs < 32 ? static_cast<int>(a.S - bs) : 32;
    const int64_t row0 = bh * a.S + bs;
    const int cbytes = nrow * CB, sbytes = nrow * NGRP * (F32S ? 4 : 1);
    const int64_t soff = row0 * NGRP * (F32S ? 4 : 1);
    for (int o = lane * 16; o < cbytes; o += 32 * 16) {
      cp_async16(dst + o, a.kc + row0 * CB + o);
      cp_async16(dst + TL::VC + o, a.vc + row0 * CB + o);
    }
    for (int o = lane * 16; o < sbytes; o += 32 * 16) {
      cp_async16(dst + TL::KS + o, static_cast<const uint8_t *>(a.ks) + soff + o);
      cp_async16(dst + TL::VS + o, static_cast<const uint8_t *>(a.vs) + soff + o);
    }
    cp_async_commit();
  };
  int it = 0;
  if (s_begin + warp * 32 < s_end) stage(s_begin + warp * 32, wt);
  for (int base = s_begin + warp * 32; base < s_end; base += kWarps * 32, ++it) {
    const uint8_t *cur = wt + (TL::NBUF == 2 ? (it & 1) * TL::TB : 0);
    const int nb = base + kWarps * 32;
    if (TL::NBUF == 2 && nb < s_end) {
      stage(nb, wt + ((it + 1) & 1) * TL::TB);  // the next tile, while this one is worked on
      cp_async_wait_one();
    } else {
      cp_async_wait_all();
    }
    __syncwarp();
    // ---- q.k, lanes over the head dim: lane (g, sub) takes dims [16 sub, 16 sub + 16)
    // -- inside one 32-element scale group -- of slots g + NG jj, with q in
    // registers (four heads per pass); a butterfly reduce-scatter across the L
    // lanes of a slot group leaves lane (g, sub) with the scores of slot g + NG sub.
    constexpr int L = D / 16, NG = 32 / L;
    const int g = lane / L, sub = lane % L;
    const int own = g + NG * sub;
    float sc[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) sc[h] = 0.0f;
#pragma unroll
    for (int h0 = 0; h0 < kMaxG; h0 += 4) {
      if (h0 >= G) break;
      float qr[4][16];
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const float4 q4 = h0 + hh < G ? *reinterpret_cast<const float4 *>(&q_s[(h0 + hh) * D + sub * 16 + 4 * k4])
                                        : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          qr[hh][4 * k4] = q4.x;
          qr[hh][4 * k4 + 1] = q4.y;
          qr[hh][4 * k4 + 2] = q4.z;
          qr[hh][4 * k4 + 3] = q4.w;
        }
      }
      float part[L][4];
#pragma unroll
      for (int jj = 0; jj < L; ++jj) {
        const int slot = base + g + NG * jj;
        float pj[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (slot < s_end) {
          const int sl = g + NG * jj;  // slot within the tile
          float v[16];
          if constexpr (Fmt<MODE>::FP4) {  // 8 bytes, element 2i in the low nibble of byte i
            const uint2 w = *reinterpret_cast<const uint2 *>(cur + sl * CB + sub * 8);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 t = decode2<MODE>((i < 4 ? w.x : w.y) >> (8 * (i & 3)));
              v[2 * i] = t.x;
              v[2 * i + 1] = t.y;
            }
          } else {
            const uint4 w = *reinterpret_cast<const uint4 *>(cur + sl * CB + sub * 16);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 t = decode2<MODE>(ww[i >> 1] >> (16 * (i & 1)));
              v[2 * i] = t.x;
              v[2 * i + 1] = t.y;
            }
          }
#pragma unroll
          for (int d = 0; d < 16; ++d)
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) pj[hh] = fmaf(qr[hh][d], v[d], pj[hh]);
          const float gs = staged_scale<MODE>(cur + TL::KS, sl * NGRP + sub / 2);
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) pj[hh] *= gs;
        }
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) part[jj][hh] = pj[hh];
      }
#pragma unroll
      for (int o = L / 2; o >= 1; o >>= 1) {
        const bool upper = (sub & o) != 0;
#pragma unroll
        for (int j = 0; j < o; ++j)
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            const float keep = upper ? part[j + o][hh] : part[j][hh];
            const float send = upper ? part[j][hh] : part[j + o][hh];
            part[j][hh] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
      }
#pragma unroll
      for (int hh = 0; hh < 4; ++hh)
        if (h0 + hh < kMaxG) sc[h0 + hh] = part[0][hh];
    }
    const int slot = base + own;
    const bool valid = slot < s_end;
    if (valid && a.mask) {
      const float madd = __ldg(a.mask + slot) * kLog2e;
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) sc[h] += madd;
    }
    // ---- online softmax over the warp's 32 slots
    bool need = false;
    float mt[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      sc[h] = valid ? sc[h] : -INFINITY;
      mt[h] = sc[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], o));
      need |= mt[h] > m[h] + 8.0f;
    }
    if (need) {  // warp-uniform
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        const float mnew = fmaxf(m[h], mt[h]);
        if (mnew > m[h]) {
          const float al = m[h] == -INFINITY ? 0.0f : ex2(m[h] - mnew);
          lsum[h] *= al;
#pragma unroll
          for (int k = 0; k < DPL; ++k) acc[h][k] *= al;
          m[h] = mnew;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      const float p = sc[h] == -INFINITY ? 0.0f : ex2(sc[h] - m[h]);
      lsum[h] += p;
      p_s[warp][own][h] = p;
    }
    __syncwarp();
    // ---- p.v, lanes over the head dim, V from the staged tile
    const int nval = min(32, s_end - base);
    for (int j = 0; j < nval; ++j) {
      const int d0 = lane * DPL;
      const float vscale = staged_scale<MODE>(cur + TL::VS, j * NGRP + d0 / 32);
      float val[DPL];
      if constexpr (Fmt<MODE>::FP4) {  // DPL/2 bytes
        const uint8_t *vp = cur + TL::VC + j * CB + d0 / 2;
        uint32_t bytes;
        if constexpr (DPL == 2) bytes = vp[0];
        else if constexpr (DPL == 4) bytes = *reinterpret_cast<const uint16_t *>(vp);
        else bytes = *reinterpret_cast<const uint32_t *>(vp);
#pragma unroll
        for (int k = 0; k < DPL; k += 2) {
          const float2 v = decode2<MODE>(bytes >> (4 * k));
          val[k] = v.x * vscale;
          val[k + 1] = v.y * vscale;
        }
      } else {
        const uint8_t *vp = cur + TL::VC + j * CB + d0;
        uint32_t w0 = 0, w1 = 0;
        if constexpr (DPL == 2) w0 = *reinterpret_cast<const uint16_t *>(vp);
        else if constexpr (DPL == 4) w0 = *reinterpret_cast<const uint32_t *>(vp);
        else {
          const uint2 t = *reinterpret_cast<const uint2 *>(vp);
          w0 = t.x;
          w1 = t.y;
        }
#pragma unroll
        for (int k = 0; k < DPL; k += 2) {
          const uint32_t src = k < 4 ? w0 : w1;
          const float2 v = decode2<MODE>(src >> (8 * (k & 3)));
          val[k] = v.x * vscale;
          val[k + 1] = v.y * vscale;
        }
      }
      const float4 *pj = reinterpret_cast<const float4 *>(&p_s[warp][j][0]);
      const float4 p0 = pj[0], p1 = pj[1];
      const float pv[kMaxG] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int h = 0; h < kMaxG; ++h)
        if (h < G)
#pragma unroll
          for (int k = 0; k < DPL; ++k) acc[h][k] = fmaf(pv[h], val[k], acc[h][k]);
    }
    __syncwarp();  // this tile's buffer is free
    if (TL::NBUF == 1 && base + kWarps * 32 < s_end) stage(base + kWarps * 32, wt);
  }

  // ---- combine the warps in order (shared running state), write this split's partial
#pragma unroll
  for (int h = 0; h < kMaxG; ++h)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
  for (int w = 0; w < kWarps; ++w) {
    if (warp == w) {
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        if (h >= G) continue;
        const float mo = w == 0 ? -INFINITY : mc_s[h];
        const float lo = w == 0 ? 0.0f : lc_s[h];
        const float M = fmaxf(mo, m[h]);
        const float fo = mo == -INFINITY ? 0.0f : ex2(mo - M);
        const float fs = m[h] == -INFINITY ? 0.0f : ex2(m[h] - M);
#pragma unroll
        for (int k = 0; k < DPL; ++k) {
          const int d = lane * DPL + k;
          const float prev = w == 0 ? 0.0f : oc_s[h][d];
          oc_s[h][d] = fmaf(prev, fo, acc[h][k] * fs);
        }
        __syncwarp();
        if (lane == 0) {
          mc_s[h] = M;
          lc_s[h] = fmaf(lo, fo, lsum[h] * fs);
        }
      }
    }
    __syncthreads();
  }
  float *rec = a.ws + (bh * a.splits + split) * static_cast<int64_t>(G) * (D + 2);
  for (int e = tid; e < G * D; e += kThreads) {
    const int h = e / D, d = e - h * D;
    rec[h * (D + 2) + d] = oc_s[h][d];
    if (d == 0) {
      rec[h * (D + 2) + D] = mc_s[h];
      rec[h * (D + 2) + D + 1] = lc_s[h];
    }
  }
}

// Combine the splits of one (b, q head), in split order.
template <int D>
__global__ void __launch_bounds__(D) merge_block_kernel(const Args a) {
  const int bq = blockIdx.x, d = threadIdx.x;
  const int b = bq / a.Hq, hq = bq - b * a.Hq;
  const int hk = hq / a.G, h = hq - hk * a.G;
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;
  float M = -INFINITY;
  for (int s = 0; s < a.splits; ++s)
    M = fmaxf(M, a.ws[((bh * a.splits + s) * a.G + h) * (D + 2) + D]);
  float L = 0.0f, O = 0.0f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.splits; ++s) {
      const float *rec = a.ws + ((bh * a.splits + s) * a.G + h) * (D + 2);
      const float ms = rec[D];
      const float f = ms == -INFINITY ? 0.0f : ex2(ms - M);
      L = fmaf(f, rec[D + 1], L);
      O = fmaf(f, rec[d], O);
    }
  }
  const float r = L > 0.0f ? O / L : 0.0f;
  a.out[(static_cast<int64_t>(b) * a.Hq + hq) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
}

struct Split {
  int splits, span;
};
// Enough CTAs to cover the SMs about twice, each split at least 256 slots.
inline Split split_for(int B, int Hkv, int64_t S, int ctas) {
  const int64_t units = static_cast<int64_t>(B) * Hkv;
  int64_t splits = (2 * ctas + units - 1) / units;
  const int64_t most = (S + 255) / 256;
  if (splits > most) splits = most;
  if (splits < 1) splits = 1;
  int64_t span = (S + splits - 1) / splits;
  span = (span + 31) / 32 * 32;
  splits = (S + span - 1) / span;
  return {static_cast<int>(splits), static_cast<int>(span)};
}

template <int MODE, int D>
int launch(const Args &a, cudaStream_t s) {
  constexpr int dyn = kWarps * VTile<MODE, D>::BYTES;
  if (const int st = ensure_smem<BlockTag<MODE, D>>(decode_block_kernel<MODE, D>, dyn)) return st;
  decode_block_kernel<MODE, D><<<dim3(a.splits, a.Hkv, a.B), kThreads, dyn, s>>>(a);
  if (cudaGetLastError() != cudaSuccess) return KVQ_ECUDA;
  merge_block_kernel<D><<<a.B * a.Hq, D, 0, s>>>(a);
  return launch_status();
}

template <int D>
int dispatch_mode(int mode, const Args &a, cudaStream_t s) {
  switch (mode) {
    case KVQ_MODE_FP8_E4M3: return launch<KVQ_MODE_FP8_E4M3, D>(a, s);
    case KVQ_MODE_MXFP8: return launch<KVQ_MODE_MXFP8, D>(a, s);
    case KVQ_MODE_MXFP4: return launch<KVQ_MODE_MXFP4, D>(a, s);
    case KVQ_MODE_FP8_E5M2: return launch<KVQ_MODE_FP8_E5M2, D>(a, s);
    case KVQ_MODE_MXFP8_E5M2: return launch<KVQ_MODE_MXFP8_E5M2, D>(a, s);
    default: return launch<KVQ_MODE_INT8_SYM, D>(a, s);
  }
}

}  // namespace blk
}  // namespace kvq

// The larger of the two paths' needs: the tensor-core path (modes 1, 2, 4, 5, 6:
// merge counters + two partial records per CTA) and the CUDA-core path (mode 3:
// per-split partials).
extern "C" size_t kvq_decode_block_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t S) {
  using namespace kvq;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S % 16 != 0) return 0;
  if (D != 64 && D != 128 && D != 256) return 0;
  const blk::Split sp = blk::split_for(B, Hkv, S, sm_count());
  const size_t simt = static_cast<size_t>(B) * Hkv * sp.splits * (Hq / Hkv) * (D + 2) * sizeof(float);
  const size_t mma = decode_blk_ws_bytes(Hq / Hkv, D);
  return simt > mma ? simt : mma;
}

extern "C" int kvq_decode_attn_block(int mode, const void *q, int B, int Hq, int Hkv, int D, const uint8_t *k_codes,
                                     const void *k_scales, const uint8_t *v_codes, const void *v_scales, int64_t S,
                                     const int32_t *kv_len, const float *mask, float sm_scale, void *out,
                                     void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream) {
  using namespace kvq;
  if (mode < KVQ_MODE_FP8_E4M3 || mode > KVQ_MODE_INT8_SYM) return KVQ_EINVAL;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S > INT32_MAX) return KVQ_EINVAL;
  if (D != 64 && D != 128 && D != 256) return KVQ_EUNSUPPORTED;
  if (S % 16 != 0 || Hq / Hkv > blk::kMaxG) return KVQ_EUNSUPPORTED;
  if (B == 0) return KVQ_OK;
  if (!q || !k_codes || !k_scales || !v_codes || !v_scales || !kv_len || !out) return KVQ_EINVAL;
  const void *ptrs[] = {q, k_codes, k_scales, v_codes, v_scales, out};  // tiles are staged by 16-byte copies
  for (const void *p : ptrs)
    if (!aligned16(p)) return KVQ_EINVAL;
  const bool f32 = mode == KVQ_MODE_FP8_E4M3 || mode == KVQ_MODE_FP8_E5M2 || mode == KVQ_MODE_INT8_SYM;
  if (f32 && ((reinterpret_cast<uintptr_t>(k_scales) | reinterpret_cast<uintptr_t>(v_scales)) & 3u))
    return KVQ_EINVAL;
  if (mask && (reinterpret_cast<uintptr_t>(mask) & 3u)) return KVQ_EINVAL;
  if (!(sm_scale == sm_scale)) return KVQ_EINVAL;
  const size_t need = kvq_decode_block_workspace_bytes(B, Hq, Hkv, D, S);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15u)) return KVQ_EINVAL;
  if (static_cast<int64_t>(B) * Hkv > 65535 || B > 65535 || static_cast<int64_t>(B) * Hq > INT32_MAX)
    return KVQ_EUNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (mode != KVQ_MODE_MXFP4 || D >= 128) {  // the tensor-core decode (E2M1 codes from D = 128)
    if (mask && !aligned16(mask)) return KVQ_EINVAL;  // the mask arrives by bulk copies
    BlkCall c{q, B, Hq, Hkv, D, k_codes, v_codes, k_scales, v_scales, S, kv_len, mask, sm_scale, out,
              workspace, workspace_bytes, err_word, s};
    switch (mode) {
      case KVQ_MODE_FP8_E4M3: return decode_blk_run<KVQ_MODE_FP8_E4M3>(c);
      case KVQ_MODE_MXFP8: return decode_blk_run<KVQ_MODE_MXFP8>(c);
      case KVQ_MODE_MXFP4: return decode_blk_run<KVQ_MODE_MXFP4>(c);
      case KVQ_MODE_FP8_E5M2: return decode_blk_run<KVQ_MODE_FP8_E5M2>(c);
      case KVQ_MODE_MXFP8_E5M2: return decode_blk_run<KVQ_MODE_MXFP8_E5M2>(c);
      default: return decode_blk_run<KVQ_MODE_INT8_SYM>(c);
    }
  }
  const blk::Split sp = blk::split_for(B, Hkv, S, sm_count());
  blk::Args a;
  a.q = static_cast<const uint16_t *>(q);
  a.kc = k_codes;
  a.vc = v_codes;
  a.ks = k_scales;
  a.vs = v_scales;
  a.mask = mask;
  a.kv_len = kv_len;
  a.out = static_cast<uint16_t *>(out);
  a.ws = static_cast<float *>(workspace);
  a.err = err_word;
  a.S = S;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.splits = sp.splits;
  a.span = sp.span;
  a.qscale = sm_scale * blk::kLog2e;
  switch (D) {
    case 64: return blk::dispatch_mode<64>(mode, a, s);
    case 128: return blk::dispatch_mode<128>(mode, a, s);
    default: return blk::dispatch_mode<256>(mode, a, s);
  }
}
