// kvq_prefill_tc.cuh -- chunked-prefill attention over the int8 cache on the
// 5th-generation tensor cores (tcgen05, sm_100a).
//
// What it computes (abaddon src/attention_cache/mod.rs, trait KvCache,
// forward_attention; ExecuTorch PR 20351 commit notes on kv_len and on the
// per-tile causal upper bound; ExecuTorch PR 24473, Summary, on the additive
// mask):  out = softmax(sm_scale * Q K^T + mask) V  with K = (k - k_zp) * k_scale,
// V = (v - v_zp) * v_scale, for the chunk's Lq query rows at positions
// kv_len - Lq + i.
//
// Design:
//  - One CTA = one warpgroup (128 threads) = 128 query rows.  With GQA the rows
//    are HPT heads x RPH positions of the same kv head, so every K/V tile is
//    dequantized once for all of them.  Thread t owns row t: TMEM lane t.
//  - K/V tiles of 64 slots: int8 codes are turned into the exact bf16 values
//    (c - zp) (|c - zp| <= 255, exact in bf16) and written into 128-byte
//    swizzled shared memory, the layout the tensor core reads; the per-slot
//    scales are applied outside the MMAs: k_scale to the score columns, v_scale
//    folded into P.
//  - S = Q K^T: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M=128, N=64, into
//    TMEM; the softmax warpgroup reads S with tcgen05.ld, keeps an online
//    softmax in the log2 domain (running max raised only when a score exceeds
//    it by more than 8), and writes P = p * v_scale to swizzled shared memory as
//    two bf16 terms, P_hi = bf16(P) and P_lo = bf16(P - P_hi), so the product
//    keeps about 16 significant bits (a single bf16 P would cost up to 2^-9 of
//    max|V| in the output); then O += P_hi V + P_lo V: tcgen05.mma M=128, N=D
//    into TMEM.  V = (c - zp) is exact in bf16.  O is rescaled in TMEM only when
//    the running max moves.
//  - Per-tile causal bound: with mask_is_causal the tile loop stops at
//    min(kv_len, kv_len - Lq + (last row of the CTA) + 1); later tiles would be
//    fully masked, so the output is bit-identical with or without the skip.
//  - Two or more CTAs per SM (D <= 128) overlap one CTA's CUDA-core phases with
//    another's tensor-core phases.
#pragma once

#include <cuda_bf16.h>

#include "kvq_common.cuh"

namespace kvq {
namespace tc {

constexpr int kRows = 128;  // query rows per CTA (tcgen05 M)
constexpr int kTile = 64;   // slots per K/V tile (tcgen05 N of S, K of P.V)
constexpr int kThreads = 128;

struct PrefillArgs {
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
  int32_t *err;
  int64_t S;
  int B, Hq, Hkv, G, Lq, nhc;  // nhc: head chunks of HPT heads per kv head
  int is_causal, mask_is_causal;
  float qscale;  // sm_scale * log2(e)
};

template <int D_, int HPT_>
struct Cfg {
  static constexpr int D = D_, HPT = HPT_, RPH = kRows / HPT;
  static constexpr int KB = D / 64;  // 64-element (128-byte) blocks along D
  // shared memory (operand regions 1024-byte aligned for the 128-byte swizzle)
  static constexpr int Q_OFF = 0;                        // KB x [128 rows x 128 B]
  static constexpr int K_OFF = Q_OFF + KB * kRows * 128;  // KB x [64 slots x 128 B]
  static constexpr int V_OFF = K_OFF + KB * kTile * 128;  // KB x [64 slots x 128 B]
  static constexpr int P_OFF = V_OFF + KB * kTile * 128;  // 2 x [128 rows x 128 B]: P_hi, P_lo
  static constexpr int KS_OFF = P_OFF + 2 * kRows * 128;  // float[64]
  static constexpr int VS_OFF = KS_OFF + kTile * 4;       // float[64]
  static constexpr int BAR_OFF = VS_OFF + kTile * 4;      // 2 mbarriers
  static constexpr int TM_OFF = BAR_OFF + 16;             // TMEM base address
  static constexpr int SMEM = TM_OFF + 16 + 1024;         // + slack to align the base to 1024
  static constexpr int S_COL = 0, O_COL = kTile;
  static constexpr int TMEM_COLS = (kTile + D) <= 128 ? 128 : ((kTile + D) <= 256 ? 256 : 512);
  static_assert(kTile + D <= TMEM_COLS, "TMEM budget");
};

// ---- descriptors -------------------------------------------------------------
// Shared-memory matrix descriptor (tcgen05): start address >> 4 in bits 0-13,
// leading byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45,
// descriptor version 1 in bits 46-47, swizzle mode in 61-63 (2 = 128-byte).
KVQ_DEVINL uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: f32 accumulator (bits 4-5 = 1), bf16 A and
// B (bits 7-9, 10-12 = 1), A/B major in bits 15/16 (0 = K-major), N >> 3 in
// bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

KVQ_DEVINL void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
KVQ_DEVINL void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
KVQ_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
KVQ_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
KVQ_DEVINL void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
KVQ_DEVINL void tmem_ld32(uint32_t taddr, float (&r)[32]) {
  uint32_t u[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]), "=r"(u[8]),
        "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]),
        "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
        "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(u[i]);
}
KVQ_DEVINL void tmem_st32(uint32_t taddr, const float (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(r[0])), "r"(__float_as_uint(r[1])), "r"(__float_as_uint(r[2])), "r"(__float_as_uint(r[3])),
      "r"(__float_as_uint(r[4])), "r"(__float_as_uint(r[5])), "r"(__float_as_uint(r[6])), "r"(__float_as_uint(r[7])),
      "r"(__float_as_uint(r[8])), "r"(__float_as_uint(r[9])), "r"(__float_as_uint(r[10])),
      "r"(__float_as_uint(r[11])), "r"(__float_as_uint(r[12])), "r"(__float_as_uint(r[13])),
      "r"(__float_as_uint(r[14])), "r"(__float_as_uint(r[15])), "r"(__float_as_uint(r[16])),
      "r"(__float_as_uint(r[17])), "r"(__float_as_uint(r[18])), "r"(__float_as_uint(r[19])),
      "r"(__float_as_uint(r[20])), "r"(__float_as_uint(r[21])), "r"(__float_as_uint(r[22])),
      "r"(__float_as_uint(r[23])), "r"(__float_as_uint(r[24])), "r"(__float_as_uint(r[25])),
      "r"(__float_as_uint(r[26])), "r"(__float_as_uint(r[27])), "r"(__float_as_uint(r[28])),
      "r"(__float_as_uint(r[29])), "r"(__float_as_uint(r[30])), "r"(__float_as_uint(r[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// MMA completion arrives within microseconds; give up after 100 ms.
KVQ_DEVINL bool wait_mma(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > 100000000ull) return false;
  }
}

KVQ_DEVINL float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of the 16-byte chunk `c` (8 bf16) of row `r` inside a 128-byte
// swizzled region (rows of 128 B, chunks XOR-permuted by r % 8).
KVQ_DEVINL uint32_t swz(int r, int c) { return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4)); }

// 16 int8 codes -> 16 bf16 values (c - zp), exact, as two 16-byte chunks.
KVQ_DEVINL void codes16_to_bf16(const uint4 &w, int zp, uint4 &lo, uint4 &hi) {
  const float mz = neg_magic_zp(zp);
  const float2 mz2 = make_float2(mz, mz);
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  uint32_t outw[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float2 a, b;
    codes4_to_f2(words[k], mz2, a, b);
    const __nv_bfloat162 ba = __float22bfloat162_rn(a);
    const __nv_bfloat162 bb = __float22bfloat162_rn(b);
    outw[2 * k] = *reinterpret_cast<const uint32_t *>(&ba);
    outw[2 * k + 1] = *reinterpret_cast<const uint32_t *>(&bb);
  }
  lo = make_uint4(outw[0], outw[1], outw[2], outw[3]);
  hi = make_uint4(outw[4], outw[5], outw[6], outw[7]);
}

template <class C>
__global__ void __launch_bounds__(kThreads, 2) prefill_tc_kernel(const PrefillArgs a) {
  constexpr int D = C::D, HPT = C::HPT, RPH = C::RPH;
  constexpr int CH = D / 16;  // 16-code chunks per slot row
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (the 128-byte swizzle is a function of address bits 4-9)
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bar_s = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *bar_o = bar_s + 1;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::TM_OFF);
  float *ks_s = reinterpret_cast<float *>(smem + C::KS_OFF);
  float *vs_s = reinterpret_cast<float *>(smem + C::VS_OFF);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int xrow = blockIdx.x;  // row block
  const int hkc = blockIdx.y;   // kv head x head chunk
  const int b = blockIdx.z;
  const int hk = hkc / a.nhc, hc = hkc - hk * a.nhc;
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;

  // ---- set-up: barriers, TMEM, kv_len
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  int kv = *a.kv_len;
  if (kv < a.Lq || kv > a.S) {
    if (tid == 0 && xrow == 0 && hkc == 0 && b == 0) report(a.err, KVQ_ERR_KV_LEN_RANGE);
    kv = kv < a.Lq ? a.Lq : static_cast<int>(a.S);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tm_s = tmem + C::S_COL, tm_o = tmem + C::O_COL;

  // ---- this thread's query row
  const int g = tid / RPH;
  const int pos = xrow * RPH + (tid - g * RPH);  // row index in the chunk
  const int hq = hk * a.G + hc * HPT + g;
  const bool row_ok = pos < a.Lq;
  const int row_limit = kv - a.Lq + pos;  // last visible slot under the causal rule

  // ---- Q tile -> swizzled smem (bf16 as given; scales are applied in fp32 later)
  {
    const uint4 *qp = reinterpret_cast<const uint4 *>(a.q + ((static_cast<int64_t>(b) * a.Hq + hq) * a.Lq + pos) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 w = row_ok ? __ldg(qp + c) : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4 *>(smem + C::Q_OFF + (c >> 3) * (kRows * 128) + swz(tid, c & 7)) = w;
    }
  }

  // ---- tile loop bound (per-tile causal upper bound)
  const int last_pos = min(xrow * RPH + RPH, a.Lq) - 1;
  const int loop_end = a.mask_is_causal ? min(kv, kv - a.Lq + last_pos + 1) : kv;
  const int ntiles = (loop_end + kTile - 1) / kTile;

  constexpr uint32_t ID_QK = idesc_bf16(kRows, kTile, 0);
  constexpr uint32_t ID_PV = idesc_bf16(kRows, D, 1);
  const uint32_t q_base = smem_u32(smem + C::Q_OFF), k_base = smem_u32(smem + C::K_OFF);
  const uint32_t v_base = smem_u32(smem + C::V_OFF), p_base = smem_u32(smem + C::P_OFF);

  float m = -INFINITY, l = 0.0f;
  uint32_t phase = 0;
  // `good`: this thread's last MMA wait completed.  The decision to stop is
  // taken at the CTA barriers, so every thread leaves the loop at the same point.
  bool good = true, failed = false;

  for (int it = 0; it < ntiles; ++it) {
    const int t0 = it * kTile;
    const int n = min(kTile, loop_end - t0);
    // ---- K / V tile: int8 -> exact bf16 (c - zp) in swizzled smem; zero rows past n
#pragma unroll 2
    for (int c = tid; c < kTile * CH; c += kThreads) {
      const int s = c / CH, part = c - s * CH;
      uint4 klo = make_uint4(0u, 0u, 0u, 0u), khi = klo, vlo = klo, vhi = klo;
      if (s < n) {
        const int64_t row = bh * a.S + t0 + s;
        const uint4 kw = __ldg(reinterpret_cast<const uint4 *>(a.k + row * D) + part);
        const uint4 vw = __ldg(reinterpret_cast<const uint4 *>(a.v + row * D) + part);
        codes16_to_bf16(kw, __ldg(a.kz + row), klo, khi);
        codes16_to_bf16(vw, __ldg(a.vz + row), vlo, vhi);
      }
      const int e0 = part * 16;  // first element of the 16 codes
      const uint32_t reg = static_cast<uint32_t>(e0 >> 6) * (kTile * 128);
      const int ch = (e0 & 63) >> 3;
      *reinterpret_cast<uint4 *>(smem + C::K_OFF + reg + swz(s, ch)) = klo;
      *reinterpret_cast<uint4 *>(smem + C::K_OFF + reg + swz(s, ch + 1)) = khi;
      *reinterpret_cast<uint4 *>(smem + C::V_OFF + reg + swz(s, ch)) = vlo;
      *reinterpret_cast<uint4 *>(smem + C::V_OFF + reg + swz(s, ch + 1)) = vhi;
    }
    if (tid < kTile) {
      const bool in = tid < n;
      ks_s[tid] = in ? __ldg(a.ks + bh * a.S + t0 + tid) : 0.0f;
      vs_s[tid] = in ? __ldg(a.vs + bh * a.S + t0 + tid) : 0.0f;
    }
    proxy_fence();
    tc_fence_before();
    if (__syncthreads_or(!good)) {
      failed = true;
      break;
    }
    tc_fence_after();

    // ---- S = Q K^T
    if (tid == 0) {
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t aoff = static_cast<uint32_t>(k >> 2) * (kRows * 128) + (k & 3) * 32;
        const uint32_t boff = static_cast<uint32_t>(k >> 2) * (kTile * 128) + (k & 3) * 32;
        mma_bf16(tm_s, sdesc(q_base + aoff, 16, 1024), sdesc(k_base + boff, 16, 1024), ID_QK, k > 0);
      }
      mma_commit(bar_s);
    }
    good = wait_mma(bar_s, phase);
    if (!good && tid == 0) wait_mma(bar_s, phase);  // the issuer lets its MMAs finish (bounded)
    tc_fence_after();

    // ---- online softmax on this row's 64 scores
    float sc[kTile];
    {
      float r32[32];
      tmem_ld32(tm_s + lane_base, r32);
#pragma unroll
      for (int j = 0; j < 32; ++j) sc[j] = r32[j];
      tmem_ld32(tm_s + lane_base + 32, r32);
#pragma unroll
      for (int j = 0; j < 32; ++j) sc[32 + j] = r32[j];
    }
    float mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < kTile; ++j) {
      const int slot = t0 + j;
      bool vis = row_ok && j < n;
      if (a.is_causal && slot > row_limit) vis = false;
      float s = sc[j] * (a.qscale * ks_s[j]);
      if (a.mask && vis) s += a.mask[static_cast<int64_t>(pos) * a.S + slot] * 1.4426950408889634f;
      sc[j] = vis ? s : -INFINITY;
      mt = fmaxf(mt, sc[j]);
    }
    // raise the running max only when a score exceeds it by more than 8
    const bool raise = mt > m + 8.0f;
    const float mnew = raise ? mt : m;
    const float alpha = (raise && m != -INFINITY) ? ex2f(m - mnew) : 1.0f;
    if (it > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {  // rescale O (warp-collective TMEM access)
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tm_o + lane_base + c * 32, o);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] *= alpha;
        tmem_st32(tm_o + lane_base + c * 32, o);
      }
    }
    l *= alpha;
    m = mnew;
#pragma unroll
    for (int c = 0; c < kTile / 8; ++c) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = c * 8 + 2 * u;
        const float p0 = sc[j] == -INFINITY ? 0.0f : ex2f(sc[j] - m);
        const float p1 = sc[j + 1] == -INFINITY ? 0.0f : ex2f(sc[j + 1] - m);
        l += p0 + p1;
        const float x0 = p0 * vs_s[j], x1 = p1 * vs_s[j + 1];
        const __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
        const float2 hf = __bfloat1622float2(hb);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
        hw[u] = *reinterpret_cast<const uint32_t *>(&hb);
        lw[u] = *reinterpret_cast<const uint32_t *>(&lb);
      }
      *reinterpret_cast<uint4 *>(smem + C::P_OFF + swz(tid, c)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4 *>(smem + C::P_OFF + kRows * 128 + swz(tid, c)) =
          make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    proxy_fence();
    tc_fence_before();
    if (__syncthreads_or(!good)) {
      failed = true;
      break;
    }
    tc_fence_after();

    // ---- O += P V
    if (tid == 0) {
#pragma unroll
      for (int k = 0; k < kTile / 16; ++k) {
        const uint64_t vd = sdesc(v_base + k * 2048, kTile * 128, 1024);
        mma_bf16(tm_o, sdesc(p_base + k * 32, 16, 1024), vd, ID_PV, (it > 0 || k > 0) ? 1u : 0u);
        mma_bf16(tm_o, sdesc(p_base + kRows * 128 + k * 32, 16, 1024), vd, ID_PV, 1u);
      }
      mma_commit(bar_o);
    }
    good = wait_mma(bar_o, phase);
    if (!good && tid == 0) wait_mma(bar_o, phase);
    tc_fence_after();
    phase ^= 1u;
  }
  // every thread reaches this barrier (a break above is taken by all of them)
  failed = __syncthreads_or(failed || !good) != 0;
  if (failed) {
    if (tid == 0) report(a.err, KVQ_ERR_TIMEOUT);
  } else
  // ---- epilogue: O / l -> bf16.  The TMEM loads are warp-collective, so every
  // lane runs them; only rows inside the chunk store.
  {
    uint16_t *op = a.out + ((static_cast<int64_t>(b) * a.Hq + hq) * a.Lq + (row_ok ? pos : 0)) * D;
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      tmem_ld32(tm_o + lane_base + c * 32, o);
      if (row_ok) {
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(o[2 * j] * inv, o[2 * j + 1] * inv);
          w[j] = *reinterpret_cast<const uint32_t *>(&v2);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(op + c * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

inline int hpt_for(int G) { return G % 4 == 0 ? 4 : (G % 2 == 0 ? 2 : 1); }

template <int D, int HPT>
int launch_prefill_tc(PrefillArgs a, cudaStream_t stream) {
  using C = Cfg<D, HPT>;
  if (const int st = ensure_smem<C>(prefill_tc_kernel<C>, C::SMEM)) return st;
  a.nhc = a.G / HPT;
  dim3 grid((a.Lq + C::RPH - 1) / C::RPH, a.Hkv * a.nhc, a.B);
  prefill_tc_kernel<C><<<grid, kThreads, C::SMEM, stream>>>(a);
  return launch_status();
}

template <int D>
int dispatch_prefill_tc(const PrefillArgs &a, cudaStream_t s) {
  switch (hpt_for(a.G)) {
    case 4: return launch_prefill_tc<D, 4>(a, s);
    case 2: return launch_prefill_tc<D, 2>(a, s);
    default: return launch_prefill_tc<D, 1>(a, s);
  }
}

}  // namespace tc
}  // namespace kvq
