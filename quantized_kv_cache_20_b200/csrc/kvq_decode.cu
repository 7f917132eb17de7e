// kvq_decode.cu -- one-query (decode) attention over the int8 KV cache.
//
// What it computes (abaddon src/attention_cache/mod.rs, trait KvCache,
// forward_attention; ExecuTorch PR 20351 commit notes on the kv_len bound;
// ExecuTorch PR 24473, Summary, on the additive mask):
//   out[b,h] = softmax_j(sm_scale * q[b,h] . K[b,hk,j] + mask[j]) . V[b,hk,j],
//   j in [0, kv_len), hk = h / G, K = (k - k_zp) * k_scale, V likewise.
//
// Design (B200, sm_100a).  Decode is HBM-bound in bytes but, with GQA, heavy in
// CUDA-core instructions per byte, so the kernel is built to keep the issue
// slots busy:
//  - Persistent grid: one CTA per SM.  The work -- units (b, kv head, head
//    chunk) x tiles of TS slots, with the tile count derived on the device from
//    *kv_len -- is flattened and cut into equal contiguous ranges, one per CTA,
//    so every SM streams the same number of bytes whatever B, Hkv and kv_len
//    are.  A CTA closes a segment whenever its range moves to the next unit.
//  - One producer warp issues 1-D bulk async copies (TMA) of the K/V code
//    tiles, scales, zero points, mask and (on a unit's first tile) the q rows
//    into an NST-stage shared-memory ring (mbarrier tx counts; one arrival per
//    consumer warp frees a stage).  Every wait is bounded.
//  - NW consumer warps each take 32 slots of a tile.  A lane owns 16 dims of
//    L = D/16 slots in turn.
//      q.k: q is rounded once per segment onto a 16-bit fixed-point grid
//      (n = rne(q * sm_scale * log2e / 2^E), |n| <= 32767, a power-of-two
//      step per head), so the dot product with the int8 codes is exact integer
//      arithmetic on dp4a (high and low bytes of n); the zero point enters as
//      - zp * sum(n).  The only rounding is q's: |error| <= 2^(E-1) per element,
//      i.e. below 2^-15 of max|q| -- far below bf16's own resolution of q.
//      A butterfly reduce-scatter across the L lanes leaves each lane with the
//      full dot products of one slot.
//      softmax: online, per lane group, in the log2 domain, with the running
//      maximum only raised when a new score exceeds it by more than 8 (the
//      accumulators then hold values up to 2^8 times larger, harmless in fp32).
//      p.v: the V codes become exact floats (c - zp) through a byte permute into
//      the mantissa of 2^23 and one packed subtract; p*v_scale is broadcast per
//      slot through shared memory and accumulated with packed fp32 FMA.
//  - Segment close: groups merge by shuffles, warps through shared memory, in
//    a fixed order.  A unit that a CTA covers alone is written directly; a
//    unit split across CTAs leaves one partial per CTA in the workspace, and a
//    small merge kernel, launched behind the decode kernel with programmatic
//    dependent launch, combines them in CTA order.  No atomics, no counters:
//    results are deterministic and the workspace needs no initialisation.
#include <cuda_bf16.h>

#include <mutex>

#include "kvq_common.cuh"

namespace kvq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest p kept without rescaling

struct DecodeArgs {
  const uint16_t *q;
  const int8_t *k;
  const float *ks;
  const int8_t *kz;
  const int8_t *v;
  const float *vs;
  const int8_t *vz;
  const float *mask;
  const int32_t *kv_len;  // one device scalar, or [B] with kv_per_batch
  int kv_per_batch;
  uint16_t *out;
  float *ws_ml;       // [C * smax][HC][2]
  float *ws_o;        // [C * smax][HC][D]
  int merge_ctas;     // grid of the merge kernel
  int32_t *err;
  int64_t S;
  int B, Hq, Hkv, G, nhc, smax;
  float qscale;  // sm_scale * log2(e)
};

template <int D_, int HC_, int NW_, int NST_, bool Q4_ = false>
struct Cfg {
  static constexpr int D = D_, HC = HC_, NW = NW_, NST = NST_;
  static constexpr bool Q4 = Q4_;          // TQ4 cache: 4-bit codes, two per byte
  static constexpr int CB = Q4 ? D / 2 : D;  // code bytes per slot
  static constexpr int L = D / 16;     // lanes per slot group (16 dims per lane)
  static constexpr int NG = 32 / L;    // slot groups per warp
  static constexpr int TS = 32 * NW;   // slots per tile
  // one ring stage
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TS * CB;
  static constexpr int KS_OFF = 2 * TS * CB;
  static constexpr int VS_OFF = KS_OFF + 4 * TS;
  static constexpr int M_OFF = VS_OFF + 4 * TS;
  static constexpr int KZ_OFF = M_OFF + 4 * TS;
  static constexpr int VZ_OFF = KZ_OFF + TS;
  static constexpr int Q_OFF = VZ_OFF + TS;
  static constexpr int STAGE = Q_OFF + 2 * HC * D;
  static_assert(STAGE % 16 == 0, "stage alignment");
  // after the ring
  static constexpr int WBUF_OFF = NST * STAGE;                 // [NW][32][4] float
  static constexpr int OSCR_OFF = WBUF_OFF + NW * 32 * 16;     // [NW][HC][D] float
  static constexpr int MLSCR_OFF = OSCR_OFF + NW * HC * D * 4; // [NW][HC][2] float
  static constexpr int BAR_OFF = MLSCR_OFF + NW * HC * 8;
  static constexpr int SH_OFF = BAR_OFF + 2 * NST * 8;
  static constexpr int SMEM = SH_OFF + 16;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr int THREADS = (NW + 1) * 32;
};

KVQ_DEVINL int dp4a_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
KVQ_DEVINL int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
KVQ_DEVINL int dp4a_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
KVQ_DEVINL int dp4a_uu(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// 8 packed 4-bit codes (element 2i in the low nibble of byte i) -> the even
// elements (0, 2, 4, 6) and the odd elements (1, 3, 5, 7) as bytes 0..15.
KVQ_DEVINL void unpack_nibbles(uint32_t w, uint32_t &even, uint32_t &odd) {
  even = w & 0x0F0F0F0Fu;
  odd = (w >> 4) & 0x0F0F0F0Fu;
}
KVQ_DEVINL float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
KVQ_DEVINL void consumer_sync(int nthreads) { asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory"); }

// Work split: CTA c owns flattened tiles [c*W/C, (c+1)*W/C).
KVQ_DEVINL int64_t range_start(int64_t c, int64_t W, int64_t C) { return c * W / C; }
KVQ_DEVINL int64_t cta_of(int64_t idx, int64_t W, int64_t C) { return ((idx + 1) * C - 1) / W; }
// The CTA after c that owns a tile of [.., last], or -1: CTAs with empty ranges
// (more CTAs than tiles) are skipped.
KVQ_DEVINL int64_t next_owner(int64_t c, int64_t last, int64_t W, int64_t C) {
  const int64_t e = range_start(c + 1, W, C);
  return e > last ? -1 : cta_of(e, W, C);
}

KVQ_DEVINL bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int32_t *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// kv_len of batch row b, clamped to [0, S] (the out-of-range report is made once,
// by max_kv_len).
KVQ_DEVINL int row_kv(const DecodeArgs &a, int b) {
  const int k = a.kv_per_batch ? a.kv_len[b] : *a.kv_len;
  return k < 0 ? 0 : (k > a.S ? static_cast<int>(a.S) : k);
}

// The largest clamped kv_len over the batch, by the whole CTA; `report_bad`
// makes this CTA flag an out-of-range value.  `red` is a shared int.
KVQ_DEVINL int max_kv_len(const DecodeArgs &a, volatile int32_t *red, bool report_bad) {
  if (!a.kv_per_batch) {
    if (threadIdx.x == 0) {
      const int k = *a.kv_len;
      if (report_bad && (k < 0 || k > a.S)) report(a.err, KVQ_ERR_KV_LEN_RANGE);
    }
    return row_kv(a, 0);
  }
  if (threadIdx.x == 0) *red = 0;
  __syncthreads();
  int mx = 0;
  bool bad = false;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    const int k = a.kv_len[b];
    bad |= k < 0 || k > a.S;
    mx = max(mx, k < 0 ? 0 : (k > a.S ? static_cast<int>(a.S) : k));
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if ((threadIdx.x & 31) == 0) atomicMax(const_cast<int32_t *>(red), mx);
  if (report_bad && __any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) report(a.err, KVQ_ERR_KV_LEN_RANGE);
  __syncthreads();
  const int r = *red;
  __syncthreads();
  return r;
}

// VARLEN: kv_len is one value per batch row (a.kv_per_batch); the scalar form
// is a separate instantiation so it carries no per-unit state.
template <class C, bool VARLEN>
__global__ void __launch_bounds__(C::THREADS, 1) decode_kernel(const DecodeArgs a) {
  constexpr int D = C::D, HC = C::HC, NW = C::NW, NST = C::NST, L = C::L, NG = C::NG, TS = C::TS;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + NST;
  volatile int32_t *sh = reinterpret_cast<volatile int32_t *>(smem + C::SH_OFF);  // kv, abort, last

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    fence_mbar_init();
    sh[1] = 0;
    sh[2] = 0;
  }
  __syncthreads();
  // Every unit is cut into ceil(max kv_len / TS) tiles; with per-row lengths a
  // row's tiles past its own kv_len carry no bytes and no work.
  const int kv = max_kv_len(a, sh, blockIdx.x == 0);
  asm volatile("griddepcontrol.launch_dependents;");
  const int ntiles = (kv + TS - 1) / TS;
  const int64_t U = static_cast<int64_t>(a.B) * a.Hkv * a.nhc;
  const int64_t CT = gridDim.x, cta = blockIdx.x;

  if (ntiles == 0) {  // nothing to attend to: every row is zero
    for (int64_t u = cta; u < U; u += CT) {
      const int hc = static_cast<int>(u % a.nhc);
      const int64_t bhk = u / a.nhc;
      const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
      for (int e = tid; e < HC * D; e += C::THREADS) {
        const int hq = hk * a.G + hc * HC + e / D;
        a.out[(static_cast<int64_t>(b) * a.Hq + hq) * D + e % D] = 0;
      }
    }
    return;
  }
  const int64_t W = U * ntiles;
  const int64_t t_begin = range_start(cta, W, CT), t_end = range_start(cta + 1, W, CT);

  // ------------------------------------------------------------------ producer
  if (warp == NW) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int64_t issued = 0;
      int64_t u = t_begin / ntiles;
      int t = static_cast<int>(t_begin - u * ntiles);
      int st = 0;
      uint32_t ephase = 0;  // parity of the empty-barrier phase to wait for at stage st
      int64_t kv_u_of = -1;
      int kv_u = kv;
      for (int64_t idx = t_begin; idx < t_end; ++idx) {
        const int64_t i = idx - t_begin;
        if (i >= NST && !wait_or_abort(&empty[st], ephase, sh + 1)) {
          report(a.err, KVQ_ERR_TIMEOUT);
          sh[1] = 1;
          break;
        }
        const int hc = static_cast<int>(u % a.nhc);
        const int64_t bhk = u / a.nhc;  // = b * Hkv + hk
        if (u != kv_u_of) {
          kv_u_of = u;
          kv_u = VARLEN ? row_kv(a, static_cast<int>(bhk / a.Hkv)) : kv;
        }
        const int s0 = t * TS;
        const int n = max(0, min(TS, kv_u - s0));
        const int n16 = (n + 15) & ~15;  // S % 16 == 0 keeps this inside the slab
        const bool first = (t == 0) || (idx == t_begin);
        uint8_t *stage = smem + st * C::STAGE;
        const uint32_t bytes = static_cast<uint32_t>(n16) * (2 * C::CB + 10) + (a.mask ? 4u * n16 : 0u) +
                               (first ? 2u * HC * D : 0u);
        mbar_arrive_expect_tx(&full[st], bytes);  // 0 bytes: a plain arrival
        const int64_t row = bhk * a.S + s0;
        if (n16 > 0) {
          bulk_g2s_hint(stage + C::K_OFF, a.k + row * C::CB, n16 * C::CB, &full[st], pol);
          bulk_g2s_hint(stage + C::V_OFF, a.v + row * C::CB, n16 * C::CB, &full[st], pol);
          bulk_g2s(stage + C::KS_OFF, a.ks + row, n16 * 4, &full[st]);
          bulk_g2s(stage + C::VS_OFF, a.vs + row, n16 * 4, &full[st]);
          bulk_g2s(stage + C::KZ_OFF, a.kz + row, n16, &full[st]);
          bulk_g2s(stage + C::VZ_OFF, a.vz + row, n16, &full[st]);
          if (a.mask) bulk_g2s(stage + C::M_OFF, a.mask + s0, n16 * 4, &full[st]);
        }
        if (first) {
          const int64_t hk = bhk % a.Hkv, b = bhk / a.Hkv;
          const int64_t q0 = (b * a.Hq + hk * a.G + static_cast<int64_t>(hc) * HC) * D;
          bulk_g2s(stage + C::Q_OFF, a.q + q0, 2 * HC * D, &full[st]);
        }
        issued = i + 1;
        if (++t == ntiles) {
          t = 0;
          ++u;
        }
        if (++st == NST) {  // entering round r = (i+1)/NST waits for empty phase (r-1) & 1
          st = 0;
          if (i + 1 >= 2 * NST) ephase ^= 1u;
        }
      }
      // the last copy issued into each stage must land before the CTA exits
      for (int64_t i = issued > NST ? issued - NST : 0; i < issued; ++i)
        if (!mbar_wait_bounded(&full[i % NST], static_cast<uint32_t>(i / NST) & 1u)) report(a.err, KVQ_ERR_TIMEOUT);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane / L, sub = lane % L;
  const int own = g + NG * sub;  // this lane's slot within the warp's 32 after the reduce-scatter
  float *wbuf = reinterpret_cast<float *>(smem + C::WBUF_OFF) + warp * 32 * 4;

  uint32_t qhi[HC][4], qlo[HC][4];
  int nsum[HC];
  float escale[HC];
  float m[HC], lsum[HC];
  float2 o2[HC][8];
  int64_t cur_u = -1;
  int seg = -1;
  int kv_u = kv;  // kv_len of the current unit's batch row (VARLEN), else kv

  auto close_segment = [&](int64_t u, int sg) {
    // (1) denominators over the lane group, then merge the NG groups of the warp
#pragma unroll
    for (int h = 0; h < HC; ++h) {
#pragma unroll
      for (int o = L / 2; o >= 1; o >>= 1) lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
#pragma unroll
      for (int o = L; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[h], o);
        const float lo = __shfl_xor_sync(0xffffffffu, lsum[h], o);
        const float M = fmaxf(m[h], mo);
        const float fs = m[h] == -INFINITY ? 0.0f : ex2(m[h] - M);
        const float fo = mo == -INFINITY ? 0.0f : ex2(mo - M);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 oo = make_float2(__shfl_xor_sync(0xffffffffu, o2[h][k].x, o),
                                        __shfl_xor_sync(0xffffffffu, o2[h][k].y, o));
          o2[h][k] = __ffma2_rn(o2[h][k], make_float2(fs, fs), __fmul2_rn(oo, make_float2(fo, fo)));
        }
        lsum[h] = lsum[h] * fs + lo * fo;
        m[h] = M;
      }
    }
    // (2) group 0 of each warp publishes the warp's state
    float *oscr = reinterpret_cast<float *>(smem + C::OSCR_OFF);
    float *mlscr = reinterpret_cast<float *>(smem + C::MLSCR_OFF);
    if (g == 0) {
#pragma unroll
      for (int h = 0; h < HC; ++h) {
        float4 *dst = reinterpret_cast<float4 *>(oscr + (warp * HC + h) * D + sub * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dst[k] = make_float4(o2[h][2 * k].x, o2[h][2 * k].y, o2[h][2 * k + 1].x, o2[h][2 * k + 1].y);
        if (sub == 0) {
          mlscr[(warp * HC + h) * 2] = m[h];
          mlscr[(warp * HC + h) * 2 + 1] = lsum[h];
        }
      }
    }
    consumer_sync(NW * 32);
    // (3) merge the warps in order; write the output or this CTA's partial
    const int64_t ntl = ntiles;
    const int64_t c_first = cta_of(u * ntl, W, CT), c_last = cta_of(u * ntl + ntl - 1, W, CT);
    const bool alone = c_first == c_last;
    const int hc = static_cast<int>(u % a.nhc);
    const int64_t bhk = u / a.nhc;
    const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
    const int64_t rec = cta * a.smax + sg;
    for (int e = tid; e < HC * D; e += NW * 32) {
      const int h = e / D, d = e - h * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, mlscr[(w * HC + h) * 2]);
      float Lt = 0.0f, O = 0.0f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float mw = mlscr[(w * HC + h) * 2];
          const float f = mw == -INFINITY ? 0.0f : ex2(mw - M);
          Lt = fmaf(f, mlscr[(w * HC + h) * 2 + 1], Lt);
          O = fmaf(f, oscr[(w * HC + h) * D + d], O);
        }
      }
      if (alone) {
        const int hq = hk * a.G + hc * HC + h;
        const float r = Lt > 0.0f ? O / Lt : 0.0f;
        a.out[(static_cast<int64_t>(b) * a.Hq + hq) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
      } else {
        a.ws_o[(rec * HC + h) * D + d] = O;
        if (d == 0) {
          a.ws_ml[(rec * HC + h) * 2] = M;
          a.ws_ml[(rec * HC + h) * 2 + 1] = Lt;
        }
      }
    }
    consumer_sync(NW * 32);  // scratch free for the next segment
  };

  int64_t u = t_begin / ntiles;
  int t = static_cast<int>(t_begin - u * ntiles);
  int st = 0;
  uint32_t fphase = 0;
  for (int64_t idx = t_begin; idx < t_end; ++idx) {
    const bool ok = wait_or_abort(&full[st], fphase, sh + 1);
    if (!ok && lane == 0) {
      report(a.err, KVQ_ERR_TIMEOUT);
      sh[1] = 1;
    }
    const uint8_t *stage = smem + st * C::STAGE;
    if (u != cur_u) {
      if (cur_u >= 0) close_segment(cur_u, seg);
      cur_u = u;
      ++seg;
      if constexpr (VARLEN) kv_u = row_kv(a, static_cast<int>(u / a.nhc / a.Hkv));
      // new unit: q (from this stage) onto the fixed-point grid, fresh softmax state
      const uint16_t *qs = reinterpret_cast<const uint16_t *>(stage + C::Q_OFF);
#pragma unroll
      for (int h = 0; h < HC; ++h) {
        const uint4 c0 = *reinterpret_cast<const uint4 *>(qs + h * D + sub * 16);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(qs + h * D + sub * 16 + 8);
        const uint32_t wq[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        float x[16];
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          x[2 * k] = bf16lo(wq[k]) * a.qscale;
          x[2 * k + 1] = bf16hi(wq[k]) * a.qscale;
          amax = fmaxf(amax, fmaxf(fabsf(x[2 * k]), fabsf(x[2 * k + 1])));
        }
#pragma unroll
        for (int o = L / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        // step 2^E with amax / 2^E < 2^15: E = floor(log2 amax) + 1 - 15
        int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127 + 1 - 15;
        E = E < -126 ? -126 : E;
        const float inv = __uint_as_float(static_cast<uint32_t>(127 - E) << 23);  // 2^-E (E in [-126, 113])
        escale[h] = __uint_as_float(static_cast<uint32_t>(127 + E) << 23);       // 2^E
        int s = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t hw = 0, lw = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // byte j of word k pairs with the code of dim 4k + j; unpacked TQ4
            // nibbles come as (0,2,4,6), (1,3,5,7), (8,10,12,14), (9,11,13,15)
            const int dim = C::Q4 ? (k >> 1) * 8 + (k & 1) + 2 * j : 4 * k + j;
            int n = __float2int_rn(x[dim] * inv);
            n = n > 32767 ? 32767 : (n < -32767 ? -32767 : n);
            s += n;
            hw |= (static_cast<uint32_t>(n >> 8) & 0xFFu) << (8 * j);
            lw |= (static_cast<uint32_t>(n) & 0xFFu) << (8 * j);
          }
          qhi[h][k] = hw;
          qlo[h][k] = lw;
        }
#pragma unroll
        for (int o = L / 2; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        nsum[h] = s;
        m[h] = -INFINITY;
        lsum[h] = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) o2[h][k] = make_float2(0.0f, 0.0f);
      }
    }

    const int s0 = t * TS;
    const int wbase = warp * 32;
    if (ok && s0 + wbase < kv_u) {
      // ---- q . k on dp4a for the L slots of this lane group (slot = wbase + g + NG*jj)
      int part[L][HC];
#pragma unroll
      for (int jj = 0; jj < L; ++jj) {
        const int sl = wbase + g + NG * jj;
        if constexpr (C::Q4) {
          const uint2 cw = *reinterpret_cast<const uint2 *>(stage + C::K_OFF + sl * C::CB + sub * 8);
          uint4 c;
          unpack_nibbles(cw.x, c.x, c.y);
          unpack_nibbles(cw.y, c.z, c.w);
#pragma unroll
          for (int h = 0; h < HC; ++h) {
            int acc = dp4a_su(qhi[h][0], c.x, 0);
            acc = dp4a_su(qhi[h][1], c.y, acc);
            acc = dp4a_su(qhi[h][2], c.z, acc);
            acc = dp4a_su(qhi[h][3], c.w, acc);
            acc *= 256;
            acc = dp4a_uu(qlo[h][0], c.x, acc);
            acc = dp4a_uu(qlo[h][1], c.y, acc);
            acc = dp4a_uu(qlo[h][2], c.z, acc);
            acc = dp4a_uu(qlo[h][3], c.w, acc);
            part[jj][h] = acc;
          }
        } else {
          const uint4 c = *reinterpret_cast<const uint4 *>(stage + C::K_OFF + sl * D + sub * 16);
#pragma unroll
          for (int h = 0; h < HC; ++h) {
            int acc = dp4a_ss(qhi[h][0], c.x, 0);
            acc = dp4a_ss(qhi[h][1], c.y, acc);
            acc = dp4a_ss(qhi[h][2], c.z, acc);
            acc = dp4a_ss(qhi[h][3], c.w, acc);
            acc *= 256;
            acc = dp4a_us(qlo[h][0], c.x, acc);
            acc = dp4a_us(qlo[h][1], c.y, acc);
            acc = dp4a_us(qlo[h][2], c.z, acc);
            acc = dp4a_us(qlo[h][3], c.w, acc);
            part[jj][h] = acc;
          }
        }
      }
      // ---- butterfly reduce-scatter: lane `sub` ends with slot jj = sub
#pragma unroll
      for (int o = L / 2; o >= 1; o >>= 1) {
        const bool upper = (sub & o) != 0;
#pragma unroll
        for (int j = 0; j < o; ++j)
#pragma unroll
          for (int h = 0; h < HC; ++h) {
            const int keep = upper ? part[j + o][h] : part[j][h];
            const int send = upper ? part[j][h] : part[j + o][h];
            part[j][h] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
      }
      // ---- scores (log2 domain) for this lane's slot
      const int sl_own = wbase + own;
      const bool valid = s0 + sl_own < kv_u;
      const int kzp = static_cast<int8_t>(stage[C::KZ_OFF + sl_own]);
      const float ksc = reinterpret_cast<const float *>(stage + C::KS_OFF)[sl_own];
      const float vsc = reinterpret_cast<const float *>(stage + C::VS_OFF)[sl_own];
      const float madd = a.mask ? reinterpret_cast<const float *>(stage + C::M_OFF)[sl_own] * kLog2e : 0.0f;
      float sc[HC], mt[HC];
      bool need = false;
#pragma unroll
      for (int h = 0; h < HC; ++h) {
        // exact: |sum n (c - zp)| < 2^31 for D <= 256 (computed modulo 2^32)
        const int dz = static_cast<int>(static_cast<uint32_t>(part[0][h]) -
                                        static_cast<uint32_t>(kzp) * static_cast<uint32_t>(nsum[h]));
        sc[h] = valid ? fmaf(static_cast<float>(dz), escale[h] * ksc, madd) : -INFINITY;
        mt[h] = sc[h];
#pragma unroll
        for (int o = L / 2; o >= 1; o >>= 1) mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], o));
        need |= mt[h] > m[h] + kRescaleThreshold;
      }
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int h = 0; h < HC; ++h) {
          const float mnew = fmaxf(m[h], mt[h]);
          if (mnew > m[h]) {
            const float alpha = m[h] == -INFINITY ? 0.0f : ex2(m[h] - mnew);
            lsum[h] *= alpha;
            const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
            for (int k = 0; k < 8; ++k) o2[h][k] = __fmul2_rn(o2[h][k], al2);
            m[h] = mnew;
          }
        }
      }
      float wv[4];
#pragma unroll
      for (int h = 0; h < HC; ++h) {
        const float p = sc[h] == -INFINITY ? 0.0f : ex2(sc[h] - m[h]);
        lsum[h] += p;
        wv[h] = p > 0.0f ? p * vsc : 0.0f;
      }
#pragma unroll
      for (int h = HC; h < 4; ++h) wv[h] = 0.0f;
      *reinterpret_cast<float4 *>(wbuf + own * 4) = make_float4(wv[0], wv[1], wv[2], wv[3]);
      __syncwarp();
      // ---- p . v over the same L slots
#pragma unroll
      for (int jj = 0; jj < L; ++jj) {
        const int sl = g + NG * jj;
        const float4 w4 = *reinterpret_cast<const float4 *>(wbuf + sl * 4);
        const float wj[4] = {w4.x, w4.y, w4.z, w4.w};
        const int zp = static_cast<int8_t>(stage[C::VZ_OFF + wbase + sl]);
        const float mz = neg_magic_zp(zp);
        const float2 mz2 = make_float2(mz, mz);
        uint4 c;
        if constexpr (C::Q4) {  // nibbles back to element order: bytes (0,1,2,3), (4,5,6,7), ...
          const uint2 cw = *reinterpret_cast<const uint2 *>(stage + C::V_OFF + (wbase + sl) * C::CB + sub * 8);
          uint32_t e0, o0, e1, o1;
          unpack_nibbles(cw.x, e0, o0);
          unpack_nibbles(cw.y, e1, o1);
          c = make_uint4(__byte_perm(e0, o0, 0x5140), __byte_perm(e0, o0, 0x7362), __byte_perm(e1, o1, 0x5140),
                         __byte_perm(e1, o1, 0x7362));
        } else {
          c = *reinterpret_cast<const uint4 *>(stage + C::V_OFF + (wbase + sl) * D + sub * 16);
        }
        float2 vv2[8];
        codes4_to_f2(c.x, mz2, vv2[0], vv2[1]);
        codes4_to_f2(c.y, mz2, vv2[2], vv2[3]);
        codes4_to_f2(c.z, mz2, vv2[4], vv2[5]);
        codes4_to_f2(c.w, mz2, vv2[6], vv2[7]);
#pragma unroll
        for (int h = 0; h < HC; ++h) {
          const float2 w2 = make_float2(wj[h], wj[h]);
#pragma unroll
          for (int k = 0; k < 8; ++k) o2[h][k] = __ffma2_rn(w2, vv2[k], o2[h][k]);
        }
      }
      __syncwarp();
    }
    if (lane == 0) mbar_arrive(&empty[st]);
    if (++t == ntiles) {
      t = 0;
      ++u;
    }
    if (++st == NST) {
      st = 0;
      fphase ^= 1u;
    }
  }
  if (cur_u >= 0) close_segment(cur_u, seg);
}

// ----------------------------------------------------------------------------
// Merge of split units: one CTA per unit.  Launched right after the decode
// kernel (programmatic dependent launch: it may start while the decode grid
// drains and waits for its completion, so all partials are visible); a unit
// whose tiles one CTA owned alone was written by the decode kernel already.
// Partials are combined in owner (CTA) order.
// ----------------------------------------------------------------------------
template <class C>
__global__ void __launch_bounds__(256) merge_kernel(const DecodeArgs a, int decode_ctas) {
  constexpr int D = C::D, HC = C::HC, TS = C::TS;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int32_t recs[1024];
  __shared__ float mls[1024 * 2];
  __shared__ int32_t red;
  const int kv = max_kv_len(a, &red, false);
  const int64_t ntl = (kv + TS - 1) / TS;
  if (ntl == 0) return;
  const int64_t U = static_cast<int64_t>(a.B) * a.Hkv * a.nhc;
  const int64_t W = U * ntl, CT = decode_ctas;
  for (int64_t u = blockIdx.x; u < U; u += gridDim.x) {
    const int64_t last_tile = u * ntl + ntl - 1;
    const int64_t c_first = cta_of(u * ntl, W, CT);
    const int64_t c_last = cta_of(last_tile, W, CT);
    if (c_first == c_last) continue;
    __syncthreads();  // recs / mls reuse across units
    int owners;
    if (W >= CT) {  // no CTA has an empty range: the owners are c_first..c_last
      owners = static_cast<int>(c_last - c_first + 1);
      for (int i = threadIdx.x; i < owners; i += blockDim.x) {
        const int64_t c = c_first + i;
        recs[i] = static_cast<int32_t>(c * a.smax + (u - range_start(c, W, CT) / ntl));
      }
    } else {
      owners = 0;
      for (int64_t c = c_first; c >= 0; c = next_owner(c, last_tile, W, CT)) {
        if (threadIdx.x == 0) recs[owners] = static_cast<int32_t>(c * a.smax + (u - range_start(c, W, CT) / ntl));
        ++owners;
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < owners * HC; i += blockDim.x) {
      const int o = i / HC, h = i - o * HC;
      const int64_t r = static_cast<int64_t>(recs[o]) * HC + h;
      mls[i * 2] = a.ws_ml[r * 2];
      mls[i * 2 + 1] = a.ws_ml[r * 2 + 1];
    }
    __syncthreads();
    const int hc = static_cast<int>(u % a.nhc);
    const int64_t bhk = u / a.nhc;
    const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
    for (int e = threadIdx.x; e < HC * D; e += blockDim.x) {
      const int h = e / D, d = e - h * D;
      float M = -INFINITY;
      for (int o = 0; o < owners; ++o) M = fmaxf(M, mls[(o * HC + h) * 2]);
      float Lt = 0.0f, O = 0.0f;
      if (M != -INFINITY) {
#pragma unroll 4
        for (int o = 0; o < owners; ++o) {
          const float oc = a.ws_o[(static_cast<int64_t>(recs[o]) * HC + h) * D + d];
          const float mc = mls[(o * HC + h) * 2];
          const float f = mc == -INFINITY ? 0.0f : ex2(mc - M);
          Lt = fmaf(f, mls[(o * HC + h) * 2 + 1], Lt);
          O = fmaf(f, oc, O);
        }
      }
      const int hq = hk * a.G + hc * HC + h;
      const float r = Lt > 0.0f ? O / Lt : 0.0f;
      a.out[(static_cast<int64_t>(b) * a.Hq + hq) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    }
  }
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
int head_chunk(int G) { return G % 4 == 0 ? 4 : (G % 3 == 0 ? 3 : (G % 2 == 0 ? 2 : 1)); }

// Tile geometry per head dim: (consumer warps, ring stages).
template <int D>
struct DTune;
template <>
struct DTune<64> { static constexpr int NW = 11, NST = 3; };
template <>
struct DTune<128> { static constexpr int NW = 11, NST = 2; };
template <>
struct DTune<256> { static constexpr int NW = 4, NST = 3; };

struct WsLayout {
  size_t ml, o, total;
  int smax;
};

// Partials of split units: one record per (CTA, segment) slot; a CTA touches
// at most ceil(U / ctas) + 2 units.
WsLayout ws_layout(int B, int Hkv, int D, int nhc, int HC, int ctas) {
  WsLayout w;
  const int64_t U = static_cast<int64_t>(B) * Hkv * nhc;
  w.smax = static_cast<int>((U + ctas - 1) / ctas + 2);
  const size_t recs = static_cast<size_t>(ctas) * w.smax;
  w.ml = 0;
  w.o = (recs * HC * 2 * 4 + 255) / 256 * 256;
  w.total = w.o + recs * HC * D * 4;
  return w;
}

template <class C, bool VARLEN>
struct KernelTag {};  // names one decode_kernel instantiation for ensure_smem

template <int D, int HC, bool Q4>
int launch_decode(DecodeArgs a, int ctas, cudaStream_t stream) {
  using C = Cfg<D, HC, DTune<D>::NW, DTune<D>::NST, Q4>;
  if (a.kv_per_batch) {
    if (const int st = ensure_smem<KernelTag<C, true>>(decode_kernel<C, true>, C::SMEM)) return st;
    decode_kernel<C, true><<<ctas, C::THREADS, C::SMEM, stream>>>(a);
  } else {
    if (const int st = ensure_smem<KernelTag<C, false>>(decode_kernel<C, false>, C::SMEM)) return st;
    decode_kernel<C, false><<<ctas, C::THREADS, C::SMEM, stream>>>(a);
  }
  if (cudaGetLastError() != cudaSuccess) return KVQ_ECUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.merge_ctas));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, merge_kernel<C>, a, ctas) != cudaSuccess) return KVQ_ECUDA;
  return launch_status();
}

template <int D, bool Q4>
int dispatch_hc(const DecodeArgs &a, int hc, int ctas, cudaStream_t s) {
  switch (hc) {
    case 1: return launch_decode<D, 1, Q4>(a, ctas, s);
    case 2: return launch_decode<D, 2, Q4>(a, ctas, s);
    case 3: return launch_decode<D, 3, Q4>(a, ctas, s);
    default: return launch_decode<D, 4, Q4>(a, ctas, s);
  }
}

}  // namespace
}  // namespace kvq

extern "C" size_t kvq_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t S) {
  using namespace kvq;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S % 16 != 0) return 0;
  if (D != 64 && D != 128 && D != 256) return 0;
  const int G = Hq / Hkv, hc = head_chunk(G);
  return ws_layout(B, Hkv, D, G / hc, hc, sm_count()).total;
}

namespace kvq {
namespace {
int decode_impl(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k, const float *k_scale,
                const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp, int64_t S,
                const int32_t *kv_len, int kv_per_batch, bool q4, const float *mask, float sm_scale, void *out,
                void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S > INT32_MAX) return KVQ_EINVAL;
  if (D != 64 && D != 128 && D != 256) return KVQ_EUNSUPPORTED;
  if (S % 16 != 0) return KVQ_EUNSUPPORTED;
  if (B == 0) return KVQ_OK;
  if (!q || !k || !k_scale || !k_zp || !v || !v_scale || !v_zp || !kv_len || !out) return KVQ_EINVAL;
  const void *ptrs[] = {q, k, k_scale, k_zp, v, v_scale, v_zp, out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return KVQ_EINVAL;
  if (mask && !aligned16(mask)) return KVQ_EINVAL;
  if (!(sm_scale == sm_scale)) return KVQ_EINVAL;
  const int G = Hq / Hkv;
  const int hc = head_chunk(G);
  const int nhc = G / hc;
  const int ctas = sm_count();
  const WsLayout w = ws_layout(B, Hkv, D, nhc, hc, ctas);
  if (ctas > 256) return KVQ_EUNSUPPORTED;  // merge staging holds 256 owners x 4 heads
  if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return KVQ_EINVAL;
  DecodeArgs a;
  a.q = static_cast<const uint16_t *>(q);
  a.k = k;
  a.ks = k_scale;
  a.kz = k_zp;
  a.v = v;
  a.vs = v_scale;
  a.vz = v_zp;
  a.mask = mask;
  a.kv_len = kv_len;
  a.kv_per_batch = kv_per_batch;
  a.out = static_cast<uint16_t *>(out);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  a.ws_ml = reinterpret_cast<float *>(ws + w.ml);
  a.ws_o = reinterpret_cast<float *>(ws + w.o);
  a.err = err_word;
  a.S = S;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = G;
  a.nhc = nhc;
  a.smax = w.smax;
  {
    const int64_t U = static_cast<int64_t>(B) * Hkv * nhc;
    a.merge_ctas = static_cast<int>(U < 4 * ctas ? U : 4 * ctas);
  }
  a.qscale = sm_scale * kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q4) {
    switch (D) {
      case 64: return dispatch_hc<64, true>(a, hc, ctas, s);
      case 128: return dispatch_hc<128, true>(a, hc, ctas, s);
      default: return dispatch_hc<256, true>(a, hc, ctas, s);
    }
  }
  switch (D) {
    case 64: return dispatch_hc<64, false>(a, hc, ctas, s);
    case 128: return dispatch_hc<128, false>(a, hc, ctas, s);
    default: return dispatch_hc<256, false>(a, hc, ctas, s);
  }
}
}  // namespace
}  // namespace kvq

extern "C" int kvq_decode_attn(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k, const float *k_scale,
                               const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp,
                               int64_t S, const int32_t *kv_len, const float *mask, float sm_scale, void *out,
                               void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream) {
  return kvq::decode_impl(q, B, Hq, Hkv, D, k, k_scale, k_zp, v, v_scale, v_zp, S, kv_len, 0, false, mask, sm_scale,
                          out, workspace, workspace_bytes, err_word, stream);
}

extern "C" int kvq_decode_attn_tq4(const void *q, int B, int Hq, int Hkv, int D, const uint8_t *k,
                                   const float *k_scale, const uint8_t *k_zp, const uint8_t *v, const float *v_scale,
                                   const uint8_t *v_zp, int64_t S, const int32_t *kv_len, const float *mask,
                                   float sm_scale, void *out, void *workspace, size_t workspace_bytes,
                                   int32_t *err_word, void *stream) {
  return kvq::decode_impl(q, B, Hq, Hkv, D, reinterpret_cast<const int8_t *>(k), k_scale,
                          reinterpret_cast<const int8_t *>(k_zp), reinterpret_cast<const int8_t *>(v), v_scale,
                          reinterpret_cast<const int8_t *>(v_zp), S, kv_len, 0, true, mask, sm_scale, out, workspace,
                          workspace_bytes, err_word, stream);
}

extern "C" int kvq_decode_attn_varlen(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k,
                                      const float *k_scale, const int8_t *k_zp, const int8_t *v,
                                      const float *v_scale, const int8_t *v_zp, int64_t S, const int32_t *kv_lens,
                                      const float *mask, float sm_scale, void *out, void *workspace,
                                      size_t workspace_bytes, int32_t *err_word, void *stream) {
  return kvq::decode_impl(q, B, Hq, Hkv, D, k, k_scale, k_zp, v, v_scale, v_zp, S, kv_lens, 1, false, mask,
                          sm_scale, out, workspace, workspace_bytes, err_word, stream);
}

// ----------------------------------------------------------------------------
// Decode without a caller-supplied workspace (for callers that cannot
// allocate device memory): the partials go to a buffer that is part of the
// library image.  In host code the symbol is only a handle; its device address
// is looked up once per device, with that device current.
// ----------------------------------------------------------------------------
namespace kvq {
namespace {
static __device__ __align__(256) uint8_t g_static_scratch[KVQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mu;
void *g_static_scratch_addr[kMaxDevices] = {};

int static_scratch_address(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return KVQ_ECUDA;
    g_static_scratch_addr[dev] = p;
  }
  *addr = g_static_scratch_addr[dev];
  return KVQ_OK;
}
}  // namespace
}  // namespace kvq

extern "C" int kvq_decode_attn_static(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k,
                                      const float *k_scale, const int8_t *k_zp, const int8_t *v,
                                      const float *v_scale, const int8_t *v_zp, int64_t S, const int32_t *kv_len,
                                      const float *mask, float sm_scale, void *out, int32_t *err_word,
                                      void *stream) {
  const size_t need = kvq_decode_workspace_bytes(B > 0 ? B : 1, Hq, Hkv, D, S);
  if (need > KVQ_STATIC_SCRATCH_BYTES) return KVQ_ESCRATCH;
  void *scratch = nullptr;
  const int st = kvq::static_scratch_address(&scratch);
  if (st != KVQ_OK) return st;
  return kvq_decode_attn(q, B, Hq, Hkv, D, k, k_scale, k_zp, v, v_scale, v_zp, S, kv_len, mask, sm_scale, out,
                         scratch, KVQ_STATIC_SCRATCH_BYTES, err_word, stream);
}
