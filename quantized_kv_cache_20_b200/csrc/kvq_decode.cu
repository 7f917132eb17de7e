// kvq_decode.cu -- one-query (decode) attention over the int8 KV cache.
//
// What it computes (abaddon src/attention_cache/mod.rs, trait KvCache,
// forward_attention; ExecuTorch PR 20351 commit notes on the kv_len bound;
// ExecuTorch PR 24473, Summary, on the additive mask):
//   out[b,h] = softmax_j(sm_scale * q[b,h] . K[b,hk,j] + mask[j]) . V[b,hk,j],
//   j in [0, kv_len), hk = h / G, K = (k - k_zp) * k_scale, V likewise.
//
// Design (HBM-bound; B200 sm_100a):
//  - Grid (split * head_chunks, Hkv, B).  Each CTA streams a contiguous slot
//    range of one (b, kv head) and serves HC query heads of its GQA group, so
//    every K/V byte is read once for all of them.  The split length is derived
//    on the device from *kv_len (no host sync, graph-replayable).
//  - One producer warp issues 1-D bulk async copies (TMA, cp.async.bulk) of
//    K/V code tiles, scales, zero points and mask into an NST-stage ring of
//    shared memory, synchronised by mbarriers (full: tx bytes; empty: one
//    arrival per consumer warp).  Every wait is bounded.
//  - NW consumer warps each own 32 slots of a tile.  A lane owns 16 dims
//    (16 code bytes = one 128-bit shared load) of L = D/16 slots in turn; the
//    codes become exact floats (c - zp) through a byte-permute into the
//    mantissa of 2^23 and one packed subtract, and q.k runs on packed fp32 FMA
//    (fma.rn.f32x2).  A butterfly reduce-scatter across the L lanes leaves each
//    lane with the full dot products of one slot, so the online-softmax state
//    is per lane-group and PV reuses the same lane/dim ownership.
//  - The CTA combines its groups in a fixed order; split partials go to the
//    workspace and the last CTA of a (b, kv head, head chunk) to finish (an
//    atomic counter it then resets) merges them in split order.  No atomics
//    touch the output, so results are deterministic.
#include <cuda_bf16.h>

#include "kvq_common.cuh"

namespace kvq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  const uint16_t *q;
  const int8_t *k;
  const float *ks;
  const int8_t *kz;
  const int8_t *v;
  const float *vs;
  const int8_t *vz;
  const float *mask;
  const int32_t *kv_len;
  uint16_t *out;
  float *ws_ml;  // [B, Hkv, nsplit, G, 2]
  float *ws_o;   // [B, Hkv, nsplit, G, D]
  int32_t *counters;  // [B, Hkv, nhc]
  int32_t *err;
  int64_t S;
  int B, Hq, Hkv, G, nsplit, nhc;
  float qscale;  // sm_scale * log2(e)
};

template <int D_, int HC_, int NW_, int NST_>
struct Cfg {
  static constexpr int D = D_, HC = HC_, NW = NW_, NST = NST_;
  static constexpr int DPL = 16;       // dims per lane
  static constexpr int L = D / DPL;    // lanes per slot group
  static constexpr int NG = 32 / L;    // slot groups per warp
  static constexpr int TS = 32 * NW;   // slots per tile
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TS * D;
  static constexpr int KS_OFF = 2 * TS * D;
  static constexpr int VS_OFF = KS_OFF + 4 * TS;
  static constexpr int M_OFF = VS_OFF + 4 * TS;
  static constexpr int KZ_OFF = M_OFF + 4 * TS;
  static constexpr int VZ_OFF = KZ_OFF + TS;
  static constexpr int STAGE = VZ_OFF + TS;
  static constexpr int RING = NST * STAGE;
  // combine scratch (reuses the ring once it is drained)
  static constexpr int OBUF = NW * NG * HC * D * 4;
  static constexpr int MLBUF = NW * NG * HC * 2 * 4;
  static_assert(OBUF + MLBUF <= RING, "combine scratch must fit in the ring");
  static constexpr int BAR_OFF = RING;
  static constexpr int SMEM = RING + 2 * NST * 8 + 16;
  static constexpr int THREADS = (NW + 1) * 32;
};

template <class C>
__global__ void __launch_bounds__(C::THREADS) decode_kernel(const DecodeArgs a) {
  constexpr int D = C::D, HC = C::HC, NW = C::NW, NST = C::NST, L = C::L, NG = C::NG, TS = C::TS;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + NST;
  int32_t *sh = reinterpret_cast<int32_t *>(empty + NST);  // [0] kv_len, [1] abort, [2] last

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hc = blockIdx.x % a.nhc, split = blockIdx.x / a.nhc;
  const int hk = blockIdx.y, b = blockIdx.z;

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    fence_mbar_init();
    int kv = *a.kv_len;
    if (kv < 0 || kv > a.S) {
      if (blockIdx.x == 0 && hk == 0 && b == 0) report(a.err, KVQ_ERR_KV_LEN_RANGE);
      kv = kv < 0 ? 0 : static_cast<int>(a.S);
    }
    sh[0] = kv;
    sh[1] = 0;
  }
  __syncthreads();

  const int kv = sh[0];
  int chunk = (kv + a.nsplit - 1) / a.nsplit;
  chunk = (chunk + TS - 1) / TS * TS;
  const int start = split * chunk;
  const int end = min(kv, start + chunk);
  const int ntiles = start < end ? (end - start + TS - 1) / TS : 0;
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;

  // ---------------------------------------------------------------- producer
  if (warp == NW) {
    if (lane == 0 && ntiles > 0) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % NST;
        if (i >= NST && !mbar_wait_bounded(&empty[st], ((i / NST) - 1) & 1)) {
          report(a.err, KVQ_ERR_TIMEOUT);
          sh[1] = 1;
          break;
        }
        const int s0 = start + i * TS;
        const int n = min(TS, end - s0);
        const int n16 = (n + 15) & ~15;  // S % 16 == 0 keeps this inside the (b, hk) slab
        uint8_t *stage = smem + st * C::STAGE;
        const uint32_t bytes = static_cast<uint32_t>(n16) * (2 * D + 10) + (a.mask ? 4u * n16 : 0u);
        mbar_arrive_expect_tx(&full[st], bytes);
        const int64_t row = bh * a.S + s0;
        bulk_g2s_hint(stage + C::K_OFF, a.k + row * D, n16 * D, &full[st], pol);
        bulk_g2s_hint(stage + C::V_OFF, a.v + row * D, n16 * D, &full[st], pol);
        bulk_g2s(stage + C::KS_OFF, a.ks + row, n16 * 4, &full[st]);
        bulk_g2s(stage + C::VS_OFF, a.vs + row, n16 * 4, &full[st]);
        bulk_g2s(stage + C::KZ_OFF, a.kz + row, n16, &full[st]);
        bulk_g2s(stage + C::VZ_OFF, a.vz + row, n16, &full[st]);
        if (a.mask) bulk_g2s(stage + C::M_OFF, a.mask + s0, n16 * 4, &full[st]);
        issued = i + 1;
      }
      // Drain: the last copy issued into each stage must have landed before
      // shared memory is reused or the CTA exits.
      for (int i = max(0, issued - NST); i < issued; ++i)
        if (!mbar_wait_bounded(&full[i % NST], (i / NST) & 1)) report(a.err, KVQ_ERR_TIMEOUT);
    }
  }

  // ---------------------------------------------------------------- consumers
  float m[HC], lsum[HC];
  float2 o2[HC][8];
  const int g = lane / L, sub = lane % L;
  if (warp < NW) {
    float2 q2[HC][8];
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      const int hq = hk * a.G + hc * HC + h;
      const uint16_t *qp = a.q + (static_cast<int64_t>(b) * a.Hq + hq) * D + sub * 16;
      const uint4 c0 = *reinterpret_cast<const uint4 *>(qp);
      const uint4 c1 = *reinterpret_cast<const uint4 *>(qp + 8);
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k)
        q2[h][k] = make_float2(bf16lo(w[k]) * a.qscale, bf16hi(w[k]) * a.qscale);
      m[h] = -INFINITY;
      lsum[h] = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) o2[h][k] = make_float2(0.0f, 0.0f);
    }

    for (int i = 0; i < ntiles; ++i) {
      const int st = i % NST;
      if (!mbar_wait_bounded(&full[st], (i / NST) & 1)) {
        if (lane == 0) report(a.err, KVQ_ERR_TIMEOUT);
        break;
      }
      const int s0 = start + i * TS;
      const uint8_t *stage = smem + st * C::STAGE;
      const int wbase = warp * 32;
      if (s0 + wbase < end) {
        // ---- q . k for the L slots of this lane group (slot = wbase + g + NG*jj)
        float part[L][HC];
#pragma unroll
        for (int jj = 0; jj < L; ++jj) {
          const int sl = wbase + g + NG * jj;
          const int zp = static_cast<int8_t>(stage[C::KZ_OFF + sl]);
          const float mz = neg_magic_zp(zp);
          const float2 mz2 = make_float2(mz, mz);
          const uint4 c = *reinterpret_cast<const uint4 *>(stage + C::K_OFF + sl * D + sub * 16);
          float2 kv2[8];
          codes4_to_f2(c.x, mz2, kv2[0], kv2[1]);
          codes4_to_f2(c.y, mz2, kv2[2], kv2[3]);
          codes4_to_f2(c.z, mz2, kv2[4], kv2[5]);
          codes4_to_f2(c.w, mz2, kv2[6], kv2[7]);
#pragma unroll
          for (int h = 0; h < HC; ++h) {
            float2 acc = __fmul2_rn(q2[h][0], kv2[0]);
#pragma unroll
            for (int k = 1; k < 8; ++k) acc = __ffma2_rn(q2[h][k], kv2[k], acc);
            part[jj][h] = acc.x + acc.y;
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
              const float keep = upper ? part[j + o][h] : part[j][h];
              const float send = upper ? part[j][h] : part[j + o][h];
              part[j][h] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        // ---- scores (log2 domain) and online softmax per lane group
        const int own = wbase + g + NG * sub;
        const bool valid = s0 + own < end;
        const float ksc = reinterpret_cast<const float *>(stage + C::KS_OFF)[own];
        const float vsc = reinterpret_cast<const float *>(stage + C::VS_OFF)[own];
        const float madd = a.mask ? reinterpret_cast<const float *>(stage + C::M_OFF)[own] * kLog2e : 0.0f;
        float w[HC];
#pragma unroll
        for (int h = 0; h < HC; ++h) {
          const float s = valid ? fmaf(part[0][h], ksc, madd) : -INFINITY;
          float mt = s;
#pragma unroll
          for (int o = L / 2; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
          const float mnew = fmaxf(m[h], mt);
          const float muse = mnew == -INFINITY ? 0.0f : mnew;
          const float alpha = exp2f(m[h] - muse);
          const float p = exp2f(s - muse);
          lsum[h] = fmaf(lsum[h], alpha, p);
          m[h] = mnew;
          const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
          for (int k = 0; k < 8; ++k) o2[h][k] = __fmul2_rn(o2[h][k], al2);
          w[h] = p > 0.0f ? p * vsc : 0.0f;
        }
        // ---- p . v over the same L slots
#pragma unroll
        for (int jj = 0; jj < L; ++jj) {
          const int sl = wbase + g + NG * jj;
          const int zp = static_cast<int8_t>(stage[C::VZ_OFF + sl]);
          const float mz = neg_magic_zp(zp);
          const float2 mz2 = make_float2(mz, mz);
          const uint4 c = *reinterpret_cast<const uint4 *>(stage + C::V_OFF + sl * D + sub * 16);
          float2 vv2[8];
          codes4_to_f2(c.x, mz2, vv2[0], vv2[1]);
          codes4_to_f2(c.y, mz2, vv2[2], vv2[3]);
          codes4_to_f2(c.z, mz2, vv2[4], vv2[5]);
          codes4_to_f2(c.w, mz2, vv2[6], vv2[7]);
#pragma unroll
          for (int h = 0; h < HC; ++h) {
            const float wj = __shfl_sync(0xffffffffu, w[h], g * L + jj);
            const float2 w2 = make_float2(wj, wj);
#pragma unroll
            for (int k = 0; k < 8; ++k) o2[h][k] = __ffma2_rn(w2, vv2[k], o2[h][k]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // per-group denominator
#pragma unroll
    for (int h = 0; h < HC; ++h)
#pragma unroll
      for (int o = L / 2; o >= 1; o >>= 1) lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
  }
  __syncthreads();  // ring drained (producer waited on every outstanding copy)

  // ---------------------------------------------------------------- CTA combine
  float *obuf = reinterpret_cast<float *>(smem);                     // [NW*NG][HC][D]
  float *mlbuf = reinterpret_cast<float *>(smem + C::OBUF);          // [NW*NG][HC][2]
  if (warp < NW) {
    const int gid = warp * NG + g;
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      float4 *dst = reinterpret_cast<float4 *>(obuf + (gid * HC + h) * D + sub * 16);
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = make_float4(o2[h][2 * k].x, o2[h][2 * k].y, o2[h][2 * k + 1].x, o2[h][2 * k + 1].y);
      if (sub == 0) {
        mlbuf[(gid * HC + h) * 2 + 0] = m[h];
        mlbuf[(gid * HC + h) * 2 + 1] = lsum[h];
      }
    }
  }
  __syncthreads();

  const bool single = a.nsplit == 1;
  const int64_t part_idx = (bh * a.nsplit + split) * a.G + hc * HC;  // first head row of this CTA
  for (int e = tid; e < HC * D; e += C::THREADS) {
    const int h = e / D, d = e - h * D;
    float M = -INFINITY;
    for (int gi = 0; gi < NW * NG; ++gi) M = fmaxf(M, mlbuf[(gi * HC + h) * 2]);
    float Ltot = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
      for (int gi = 0; gi < NW * NG; ++gi) {
        const float mg = mlbuf[(gi * HC + h) * 2];
        if (mg == -INFINITY) continue;
        const float f = exp2f(mg - M);
        Ltot = fmaf(f, mlbuf[(gi * HC + h) * 2 + 1], Ltot);
        O = fmaf(f, obuf[(gi * HC + h) * D + d], O);
      }
    }
    if (single) {
      const int hq = hk * a.G + hc * HC + h;
      const float r = Ltot > 0.0f ? O / Ltot : 0.0f;
      a.out[(static_cast<int64_t>(b) * a.Hq + hq) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    } else {
      a.ws_o[(part_idx + h) * D + d] = O;
      if (d == 0) {
        a.ws_ml[(part_idx + h) * 2 + 0] = M;
        a.ws_ml[(part_idx + h) * 2 + 1] = Ltot;
      }
    }
  }
  if (single) return;

  // ---------------------------------------------------------------- split merge
  __threadfence();
  __syncthreads();
  int32_t *counter = a.counters + bh * a.nhc + hc;
  if (tid == 0) sh[2] = (atomicAdd(counter, 1) == a.nsplit - 1);
  __syncthreads();
  if (!sh[2]) return;
  __threadfence();
  for (int e = tid; e < HC * D; e += C::THREADS) {
    const int h = e / D, d = e - h * D;
    float M = -INFINITY;
    for (int sp = 0; sp < a.nsplit; ++sp)
      M = fmaxf(M, __ldcg(a.ws_ml + ((bh * a.nsplit + sp) * a.G + hc * HC + h) * 2));
    float Ltot = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
      for (int sp = 0; sp < a.nsplit; ++sp) {
        const int64_t pi = (bh * a.nsplit + sp) * a.G + hc * HC + h;
        const float ms = __ldcg(a.ws_ml + pi * 2);
        if (ms == -INFINITY) continue;
        const float f = exp2f(ms - M);
        Ltot = fmaf(f, __ldcg(a.ws_ml + pi * 2 + 1), Ltot);
        O = fmaf(f, __ldcg(a.ws_o + pi * D + d), O);
      }
    }
    const int hq = hk * a.G + hc * HC + h;
    const float r = Ltot > 0.0f ? O / Ltot : 0.0f;
    a.out[(static_cast<int64_t>(b) * a.Hq + hq) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
  }
  if (tid == 0) *counter = 0;  // leave the workspace ready for the next call
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
int head_chunk(int G) { return G % 4 == 0 ? 4 : (G % 3 == 0 ? 3 : (G % 2 == 0 ? 2 : 1)); }

template <int D>
struct DCfgFor;
template <>
struct DCfgFor<64> { static constexpr int NW = 8, NST = 3; };
template <>
struct DCfgFor<128> { static constexpr int NW = 4, NST = 3; };
template <>
struct DCfgFor<256> { static constexpr int NW = 2, NST = 3; };

int tile_slots(int D) { return 32 * (D == 64 ? DCfgFor<64>::NW : D == 128 ? DCfgFor<128>::NW : DCfgFor<256>::NW); }

// Split count: enough CTAs for ~4 per SM (two resident rounds of two), never
// more than one tile per split at full S.
int choose_nsplit(int B, int Hkv, int nhc, int D, int64_t S) {
  const int64_t units = static_cast<int64_t>(B) * Hkv * nhc;
  const int64_t target = static_cast<int64_t>(sm_count()) * 4;
  int64_t ns = (target + units - 1) / units;
  const int64_t max_split = (S + tile_slots(D) - 1) / tile_slots(D);
  if (ns > max_split) ns = max_split;
  if (ns < 1) ns = 1;
  if (ns > 1024) ns = 1024;
  return static_cast<int>(ns);
}

struct WsLayout {
  size_t counters, ml, o, total;
};

WsLayout ws_layout(int B, int Hq, int Hkv, int D, int nsplit, int nhc) {
  WsLayout w;
  const size_t nc = static_cast<size_t>(B) * Hkv * nhc;
  w.counters = 0;
  w.ml = (nc * 4 + 255) / 256 * 256;
  const size_t rows = static_cast<size_t>(B) * Hkv * nsplit * (Hq / Hkv);
  w.o = w.ml + (rows * 2 * 4 + 255) / 256 * 256;
  w.total = nsplit > 1 ? w.o + rows * D * 4 : 0;
  return w;
}

template <int D, int HC>
int launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  using C = Cfg<D, HC, DCfgFor<D>::NW, DCfgFor<D>::NST>;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(decode_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return KVQ_ECUDA;
    configured = true;
  }
  dim3 grid(a.nsplit * a.nhc, a.Hkv, a.B);
  decode_kernel<C><<<grid, C::THREADS, C::SMEM, stream>>>(a);
  return launch_status();
}

template <int D>
int dispatch_hc(const DecodeArgs &a, int hc, cudaStream_t s) {
  switch (hc) {
    case 1: return launch_decode<D, 1>(a, s);
    case 2: return launch_decode<D, 2>(a, s);
    case 3: return launch_decode<D, 3>(a, s);
    default: return launch_decode<D, 4>(a, s);
  }
}

}  // namespace
}  // namespace kvq

extern "C" size_t kvq_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t S) {
  using namespace kvq;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S % 16 != 0) return 0;
  if (D != 64 && D != 128 && D != 256) return 0;
  const int nhc = (Hq / Hkv) / head_chunk(Hq / Hkv);
  const int ns = choose_nsplit(B, Hkv, nhc, D, S);
  const WsLayout w = ws_layout(B, Hq, Hkv, D, ns, nhc);
  return w.total > 0 ? w.total : 256;
}

extern "C" int kvq_decode_attn(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k, const float *k_scale,
                               const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp,
                               int64_t S, const int32_t *kv_len, const float *mask, float sm_scale, void *out,
                               void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream) {
  using namespace kvq;
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
  if (static_cast<int64_t>(B) * Hkv > 65535 * 65535LL || Hkv > 65535 || B > 65535) return KVQ_EUNSUPPORTED;
  const int ns = choose_nsplit(B, Hkv, nhc, D, S);
  const WsLayout w = ws_layout(B, Hq, Hkv, D, ns, nhc);
  if (ns > 1) {
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return KVQ_EINVAL;
  }
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
  a.out = static_cast<uint16_t *>(out);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  a.counters = ns > 1 ? reinterpret_cast<int32_t *>(ws + w.counters) : nullptr;
  a.ws_ml = ns > 1 ? reinterpret_cast<float *>(ws + w.ml) : nullptr;
  a.ws_o = ns > 1 ? reinterpret_cast<float *>(ws + w.o) : nullptr;
  a.err = err_word;
  a.S = S;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = G;
  a.nsplit = ns;
  a.nhc = nhc;
  a.qscale = sm_scale * kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (D) {
    case 64: return dispatch_hc<64>(a, hc, s);
    case 128: return dispatch_hc<128>(a, hc, s);
    default: return dispatch_hc<256>(a, hc, s);
  }
}
