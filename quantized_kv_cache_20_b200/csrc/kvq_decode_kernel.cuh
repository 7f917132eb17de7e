// kvq_decode_kernel.cuh -- one-query (decode) attention over the quantized KV cache:
// the kernel, its cores and its launch (the entry points are in kvq_decode.cu and
// kvq_decode_block.cu).
//
// What it computes (abaddon src/attention_cache/mod.rs, trait KvCache,
// forward_attention; ExecuTorch PR 20351 commit notes on the kv_len bound;
// ExecuTorch PR 24473, Summary, on the additive mask):
//   out[b,h] = softmax_j(sm_scale * q[b,h] . K[b,hk,j] + mask[j]) . V[b,hk,j],
//   j in [0, kv_len), hk = h / G, K = (k - k_zp) * k_scale, V likewise.
//
// Design (B200, sm_100a).  Decode is HBM-bound in bytes, but with GQA every
// K/V byte feeds G q heads: at G = 4 and D = 128 a 32-slot chunk needs 32 K
// multiply-adds for q.K and as many for P.V.  On this part the CUDA-core pipes
// that do them (integer dot products, packed fp32 FMA, byte permutes) issue
// every other cycle, so those multiply-adds alone take about as long as HBM
// takes to deliver the bytes.  The int8 cache is therefore contracted on the
// tensor cores (warp-level mma.sync; the tiles are M = 16 rows of q heads, far
// too small for tcgen05's 64/128-row tiles), leaving the CUDA cores the
// softmax bookkeeping:
//  - Persistent grid: one CTA per SM.  The work -- units (b, kv head, head
//    chunk of HC q heads) x chunks of CS slots, with the chunk count derived
//    on the device from *kv_len -- is flattened and cut into equal contiguous
//    ranges, one per CTA, so every SM streams the same bytes (to one chunk)
//    whatever B, Hkv and kv_len are.  With one kv_len per batch row the
//    flattening uses each row's own length (a prefix of the rows' chunk counts
//    in shared memory).  With one kv_len, when the units divide the grid into
//    k >= 1 CTAs each at no cost in rounds of chunks per warp, only those U k
//    CTAs stream, each a k-th of one unit: a warp's time is set by its rounds
//    of chunks (copy latency, then compute), and a CTA confined to one unit
//    skips the second combine and the three-owner merges of the flattened cut.
//  - Every warp is its own pipeline: chunk i of the CTA's range belongs to
//    warp i mod NW, whose R-deep ring of chunk buffers is filled by async
//    copies -- K and V tiles by 2-D TMA with the 128-byte (64-byte for D = 64)
//    swizzle, so that ldmatrix reads them without bank conflicts; scales, zero
//    points and mask by 1-D bulk copies -- counted on the buffer's mbarrier.
//    The warp computes every q head of the unit on each chunk.  No producer
//    warp, no cross-warp hand-off in the main loop; every wait is bounded.
//  - q.K (tensor cores, exact): q is rounded once per unit onto a 16-bit
//    fixed-point grid per head (n = rne(q * sm_scale * log2e / 2^E), a
//    power-of-two step, |n| <= 32639) and split exactly into two signed bytes,
//    n = 256 hi + lo.  One int8 MMA (m16n8k32, int32 accumulate) takes hi in
//    rows 0..7 and lo in rows 8..15, so a lane ends with both halves of its
//    head's dot products: sum n k = 256 (hi . k) + (lo . k), exact.  The zero
//    point enters as - zp * sum(n).  The only rounding is q's, below 2^-15 of
//    max|q|, far below bf16's own resolution of q.
//  - softmax: online, in the log2 domain; the running maximum of a head is
//    raised only when a score exceeds it by more than 8.
//  - P.V (tensor cores, fp32 accumulate): O^T = V^T P^T with m16n8k16 fp16
//    MMAs.  The q.K accumulator fragment of a lane holds exactly the weights
//    its P^T fragment needs, so P never leaves the registers.  A weight
//    w = p * v_scale * 2^-E_v (E_v: a per-unit power of two keeping w below
//    2^15) enters as the fp16 pair hi + lo (two MMAs), about 22 significant
//    bits.  V^T fragments come from ldmatrix.trans of the code bytes; one
//    permute makes a pair of codes the exact fp16 values 1152 + c, and the
//    offset and zero point leave as one per-head correction,
//    sum_j w_j (1152 + zp_j).
//  - The TQ4 cache (4-bit codes, two a byte) runs the same core at D = 128 and
//    256: a lane's codes of an ldmatrix row are unpacked to bytes for the int8
//    q.K MMA (q loaded in the matching order), and made the fp16 values 1024 + c
//    for P.V.  At D = 64 (32-byte code rows) it runs the skeleton on the CUDA
//    cores: q.k on dp2a with an exact 16-bit q, p.v on packed fp32 FMA over
//    codes turned into exact subnormal floats.
//  - Unit close: when a CTA spans at most two units, a warp keeps its first
//    unit's state in registers and starts the second; at the end the (idle)
//    rings hold every warp's records and the CTA merges them in warp order.
//    With more units per CTA (short rows), a warp stops prefetching at the end
//    of each unit and the CTA merges each unit through the rings.  A unit a
//    CTA covers alone is written directly; a unit split across CTAs leaves one
//    partial per CTA in the workspace, and the owner that completes the unit
//    (a counter in the workspace, named by the unit's first owner CTA and
//    reset to zero by the completing owner) merges the partials in owner
//    order, so the result does not depend on which CTA finishes last.
//  - The kernel is launched as a programmatic dependent of the kernel before
//    it (typically the cache write of the new token): its launch and barrier
//    set-up overlap that kernel's tail, and it reads nothing before
//    griddepcontrol.wait has seen that kernel complete.
#pragma once

#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched from the driver at run time)
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "kvq_common.cuh"

namespace kvq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest p kept without rescaling
constexpr int kMaxCtas = 256;   // grid size limit (owner records staged per unit; merge counters)
constexpr int kMaxRows = 1024;  // per-row kv_len: batches up to this many rows are flattened by their own lengths

struct DecodeArgs {
  const uint16_t *q;
  const int8_t *k;
  const float *ks;
  const int8_t *kz;
  const int8_t *v;
  const float *vs;
  const int8_t *vz;
  const float *mask;
  int64_t mask_bstride;   // floats between batch rows' masks (0: one mask for every row)
  const int32_t *kv_len;  // one device scalar, or [B] with kv_per_batch
  int kv_per_batch;
  uint16_t *out;
  int32_t *ws_cnt;    // [kMaxCtas] merge counters, one per CTA: the split unit whose first owner it is
  float *ws_ml;       // [C][2][HC][2]: (m, l) of the CTA's first and last unit, when split
  float *ws_o;        // [C][2][HC][D]
  int32_t *err;
  int64_t S;
  int B, Hq, Hkv, G, nhc;
  float qscale;       // sm_scale * log2(e)
  uint64_t wait_ns;   // bound on each main-loop wait
  // block caches (kvq_write modes 1, 2, 4, 5, 6): per-32 scales [rows][D / 32], float
  // or E8M0 bytes (k / v hold the codes; ks, vs, kz, vz unused)
  const void *kscl, *vscl;
};

// 2-D TMA descriptors of the K and V code slabs [B * Hkv * S rows, D bytes]
// (tensor-core path only).
struct __align__(64) KvMaps {
  CUtensorMap k, v;
};

// ---------------------------------------------------------------------------
// Shared-memory layout: NW rings of R buffers.  A buffer is a tile (K codes,
// then V codes of 32 slots) and a small part (k scales, v scales, mask, k zero
// points, v zero points); tiles are 1024-byte aligned for the TMA swizzle.
// ---------------------------------------------------------------------------
template <int D_, int HC_, int NW_, int R_, bool MMA_, bool Q4_, int CS_ = 32, int MODE_ = 0>
struct Cfg {
  static constexpr int D = D_, HC = HC_, NW = NW_, R = R_;
  static constexpr bool MMA = MMA_;          // int8 or block cache on the tensor cores
  static constexpr bool Q4 = Q4_;            // TQ4 cache: 4-bit codes, two per byte
  static_assert(!(MMA && Q4) || D_ >= 128, "the TQ4 cache on the tensor cores from D = 128");
  static constexpr int MODE = MODE_;         // kvq_write mode of the cache: 0 int8 affine, else a block mode
  static constexpr bool BLK = MODE_ != 0;
  static_assert(!BLK || (MMA && MODE_ <= KVQ_MODE_INT8_SYM && (MODE_ != KVQ_MODE_MXFP4 || D_ >= 128)),
                "block caches on the tensor cores (MX-FP4 from D = 128)");
  static constexpr bool F32S = MODE_ == KVQ_MODE_FP8_E4M3 || MODE_ == KVQ_MODE_FP8_E5M2 || MODE_ == KVQ_MODE_INT8_SYM;
  static constexpr int NGS = D / 32;         // scale groups of a slot (block caches)
  static constexpr int SB = F32S ? 4 : 1;    // bytes of one group scale
  static constexpr int CB = Q4 || MODE_ == KVQ_MODE_MXFP4 ? D / 2 : D;  // code bytes per slot
  static constexpr int CS = CS_;             // slots per chunk
  static_assert(CS == 32 || (MMA && CS == 64), "the CUDA-core path maps 32 lanes onto 32 slots");
  static constexpr int KT = CS * CB;         // one tile of codes
  static constexpr int TILE = 2 * KT;        // K tile, V tile
  static constexpr int ROWB = CB < 128 ? CB : 128;  // bytes of a swizzled tile row (tensor-core path)
  static constexpr int SUBT = CS_ * ROWB;         // bytes of one swizzled sub-tile
  // small part of a buffer: int8 cache, k / v scales, mask, k / v zero points;
  // block cache, the k / v scale rows [CS][NG] and the mask
  static constexpr int KS_OFF = 0, VS_OFF = BLK ? CS * NGS * SB : 4 * CS;
  static constexpr int M_OFF = BLK ? 2 * CS * NGS * SB : 8 * CS;
  static constexpr int KZ_OFF = 12 * CS, VZ_OFF = 13 * CS;
  static constexpr int SMALL = BLK ? M_OFF + 4 * CS : 14 * CS;
  static_assert(VS_OFF % 16 == 0 && M_OFF % 16 == 0 && SMALL % 16 == 0, "bulk copy alignment");
  // CUDA-core path geometry
  static constexpr int L = D / 16;           // q.k: lanes per slot (16 dims per lane)
  static constexpr int NG = 32 / L;          // q.k: slot groups per warp
  static constexpr int VPL = D / 32;         // p.v: dims per lane
  // a warp's record of one unit: O [HC][D] float, then (m, l, corr, -) [HC][4] float
  static constexpr int PUB = HC * D * 4 + HC * 16;
  static_assert(2 * PUB <= R * TILE, "two unit records fit a warp's (then idle) ring of tiles");
  static constexpr int SMALL_OFF = NW * R * TILE;
  // per-warp scratch: CUDA-core path, weights [HC][CS]; tensor-core path, per-slot values
  // [CS] float4 + [CS] float
  static constexpr int WBUF_OFF = SMALL_OFF + NW * R * SMALL;
  // block caches: (k factor, -, mask, v factor) [CS] float4, then the group factors
  // of K and V, [NG][CS] float each
  static constexpr int WBUF_W = BLK ? CS * 16 + 2 * NGS * CS * 4 : (MMA ? CS * 20 : HC * CS * 4);  // bytes per warp
  static constexpr int BAR_OFF = WBUF_OFF + NW * WBUF_W;     // [NW][R] mbarrier
  static constexpr int SH_OFF = (BAR_OFF + NW * R * 8 + 15) / 16 * 16;     // 8 ints
  static constexpr int Q_OFF = SH_OFF + 32;                  // [2] q slots of 2 HC D bytes
  static constexpr int QMETA_OFF = Q_OFF + 4 * HC * D;       // [2][HC] (sum n, 2^E)
  static constexpr int RECS_OFF = QMETA_OFF + 2 * HC * 8;    // [2][kMaxCtas] owner records
  static constexpr int PFX_OFF = RECS_OFF + 2 * kMaxCtas * 4;  // [kMaxRows + 1] chunk prefix, [32] scratch
  // cluster pair merge: the half of the unit's O this CTA merges, from either CTA
  // ([2 sources][HC D / 2] float), then every head's (M, L) from either ([2][HC] float2)
  static constexpr int PAIR_OFF = (PFX_OFF + (kMaxRows + 1 + 32) * 4 + 15) / 16 * 16;
  static constexpr int PAIR_BYTES = HC * D * 4 + HC * 16;
  static constexpr int ALIGN = MMA ? 1024 : 0;                 // slack to align the tiles
  static constexpr int SMEM = PAIR_OFF + PAIR_BYTES + ALIGN;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr int THREADS = NW * 32;
};

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
// a (two signed 16-bit values) . bytes {0,1} (lo) or {2,3} (hi) of b, plus c
KVQ_DEVINL int dp2a_lo_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
KVQ_DEVINL int dp2a_hi_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
KVQ_DEVINL float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Add 1 to a merge counter, releasing this CTA's partial (written before the
// barrier that precedes the call) and acquiring the other owners'.
KVQ_DEVINL int count_acq_rel(int32_t *p) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// Work split: CTA c owns flattened chunks [c*W/C, (c+1)*W/C); cta_of is its inverse.
KVQ_DEVINL int64_t range_start(int64_t c, int64_t W, int64_t C) { return c * W / C; }
KVQ_DEVINL int64_t cta_of(int64_t idx, int64_t W, int64_t C) { return ((idx + 1) * C - 1) / W; }
// CTAs that take part when every one of the U units has nch chunks: all CT0 of the
// grid (the flattened split), or U * k of them, k = floor(CT0 / U), when that costs a
// warp no more rounds of chunks (a warp takes every NW-th chunk of its CTA).  With
// U * k CTAs the range of CTA c lies inside unit floor(c / k), so a CTA never combines
// two units and a unit has exactly k owners (none to merge when k = 1).
// Index math in 32 bits (U * nch < 2^31, CT0 <= kMaxCtas): a 64-bit division by a
// run-time value is a long dependent chain, and these sit before the first copy.
KVQ_DEVINL int active_ctas(uint32_t U, uint32_t nch, uint32_t CT0, uint32_t NW) {
  const uint32_t k = CT0 / U;
  if (k < 1) return static_cast<int>(CT0);
  const uint32_t rounds_all = ((U * nch + CT0 - 1) / CT0 + NW - 1) / NW;
  const uint32_t rounds_units = ((nch + k - 1) / k + NW - 1) / NW;
  return static_cast<int>(rounds_units <= rounds_all ? U * k : CT0);
}
// range_start(c, W, C) for 0 <= c <= C <= kMaxCtas, given q = W / C and r = W % C
KVQ_DEVINL int range_start_qr(uint32_t c, uint32_t q, uint32_t r, uint32_t C) { return static_cast<int>(c * q + c * r / C); }

// One probe of the phase, suspending the thread for at most `hint_ns`.
KVQ_DEVINL bool mbar_try_wait_ns(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for a ring buffer, giving up after `limit_ns` or once another warp of
// the CTA has given up (abort_flag).
KVQ_DEVINL bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int32_t *abort_flag, uint64_t limit_ns) {
  if (limit_ns < kNoProbeBelowNs) return false;
  const uint32_t hint = limit_ns < kSuspendNs ? static_cast<uint32_t>(limit_ns) : kSuspendNs;
  if (mbar_try_wait_ns(bar, parity, hint)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_ns(bar, parity, hint)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
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

// Byte e (0..3) of w as the low byte of an otherwise zero word: with w's bytes
// biased by +128 that is the exact subnormal float (c + 128) * 2^-149.
KVQ_DEVINL float byte_as_subnormal(uint32_t w, int e) {
  return __uint_as_float(__byte_perm(w, 0u, 0x4440u + static_cast<uint32_t>(e)));
}

// 2^e as a float for e in [-126, 127].
KVQ_DEVINL float pow2i(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// ---- tensor-core and TMA helpers
KVQ_DEVINL void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
KVQ_DEVINL void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D (16 x 8, int32) += A (16 x 32, s8, row) . B (32 x 8, s8, col)
KVQ_DEVINL void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D (16 x 8, fp32) += A (16 x 16, f16, row) . B (16 x 8, f16, col)
KVQ_DEVINL void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// A load of the word at p whose value is never read: it only starts the first
// access to p's page (translation, line into L2).  Nothing waits for it.
KVQ_DEVINL void touch_translation(const void *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(reinterpret_cast<uintptr_t>(p) & ~uintptr_t(3)));
  asm volatile("" ::"r"(v));
}
// Bring a TMA descriptor (a __grid_constant__ kernel parameter) into the descriptor cache.
KVQ_DEVINL void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// One 2-D TMA box of the map at element (x, y), completion counted on bar.
KVQ_DEVINL void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// Two floats -> f16x2 (x in the low half), round to nearest.
KVQ_DEVINL uint32_t pack_f16x2(float x, float y) {
  const __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<const uint32_t *>(&h);
}
KVQ_DEVINL float2 unpack_f16x2(uint32_t u) { return __half22float2(*reinterpret_cast<const __half2 *>(&u)); }

// ---------------------------------------------------------------------------
// Per-warp math of one unit on the CUDA cores (TQ4 cache at D = 64).
//   q.k: a lane takes 16 dims of L = D/16 slots; lane `sub` visits slot
//   g + NG*(t ^ sub) at step t, which makes the reduce-scatter over the L lanes
//   a plain butterfly that leaves each lane the full dot products of one slot.
//   p.v: lanes own D/32 dims; packed fp32 FMA pairs two consecutive slots of a
//   dim (even slots in .x, odd in .y).  Codes become the exact subnormal floats
//   (c + 128) * 2^-149 and the weights carry 2^96, so the accumulators hold
//   2^-53 of the sums.
// ---------------------------------------------------------------------------
template <class C>
struct SimtCore {
  static constexpr int D = C::D, HC = C::HC, L = C::L, NG = C::NG, CS = C::CS, CB = C::CB, VPL = C::VPL;
  static constexpr float kWScale = 79228162514264337593543950336.0f;  // 2^96
  static constexpr float kWUnscale = 1.2621774483536189e-29f;         // 2^-96
  static constexpr float OSCALE = 9007199254740992.0f;                // 2^53: record O is 2^-53 of the sums

  uint32_t qw[HC][8];
  int qslot;
  float m[HC], lsum[HC], corr[HC];  // corr: sum of p * v_scale * 2^96 * (128 + v_zp)
  float2 o2[HC][VPL];
  float sm_[HC], sl_[HC], sc_[HC], so_[HC][VPL];  // the first unit's state (deferred close)

  // q of one head as the converter gets it: here the row pointer (the loads
  // happen inside convert_q).
  struct QRaw {
    const uint16_t *qg;
  };
  static __device__ __forceinline__ QRaw load_q_raw(const uint16_t *qg, int) { return QRaw{qg}; }

  // warp `h` (< HC): head h of q onto the fixed-point grid, into q slot `slot`.
  //   n = rne(q * qscale / 2^E), |n| <= 32767.  Word w of lane sub pairs (low half,
  //   high half) with bytes {0,1} (w even) or {2,3} (w odd) of the lane's code word
  //   w / 2, which holds the unpacked nibbles of dims (0,2,4,6), (1,3,5,7),
  //   (8,10,12,14), (9,11,13,15) of the lane's 16.
  static __device__ __forceinline__ void convert_q(uint8_t *smem, const QRaw &raw, float qscale, int slot, int h,
                                                   int lane) {
    const uint16_t *qg = raw.qg;
    constexpr int NWD = D / 2;            // words of one head
    constexpr int PER = (NWD + 31) / 32;  // words per lane
    float x[PER][2];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int wd = lane + 32 * i, sb = wd >> 3, w = wd & 7, cw = w >> 1, half = w & 1;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int byte = 2 * half + j;
        const int dim = sb * 16 + (cw >> 1) * 8 + (cw & 1) + 2 * byte;
        x[i][j] = wd < NWD ? __uint_as_float(static_cast<uint32_t>(qg[dim]) << 16) * qscale : 0.0f;
        amax = fmaxf(amax, fabsf(x[i][j]));
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // step 2^E with amax / 2^E < 2^15: E = floor(log2 amax) + 1 - 15
    int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127 + 1 - 15;
    E = E < -126 ? -126 : E;
    const float inv = pow2i(-E);
    uint32_t *qs = reinterpret_cast<uint32_t *>(smem + C::Q_OFF) + (slot * HC + h) * NWD;
    int s = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int wd = lane + 32 * i;
      int n[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        n[j] = __float2int_rn(x[i][j] * inv);
        n[j] = n[j] > 32767 ? 32767 : (n[j] < -32767 ? -32767 : n[j]);
        s += n[j];
      }
      if (wd < NWD) qs[wd] = (static_cast<uint32_t>(n[0]) & 0xFFFFu) | (static_cast<uint32_t>(n[1]) << 16);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      int32_t *meta = reinterpret_cast<int32_t *>(smem + C::QMETA_OFF) + (slot * HC + h) * 2;
      meta[0] = s;
      meta[1] = static_cast<int32_t>(__float_as_uint(pow2i(E)));
    }
  }

  __device__ __forceinline__ void load_q(const uint8_t *smem, int slot, int lane) {
    const int sub = lane % L;
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      const uint32_t *qs = reinterpret_cast<const uint32_t *>(smem + C::Q_OFF) + (slot * HC + h) * (D / 2) + sub * 8;
      const uint4 w0 = *reinterpret_cast<const uint4 *>(qs);
      const uint4 w1 = *reinterpret_cast<const uint4 *>(qs + 4);
      qw[h][0] = w0.x; qw[h][1] = w0.y; qw[h][2] = w0.z; qw[h][3] = w0.w;
      qw[h][4] = w1.x; qw[h][5] = w1.y; qw[h][6] = w1.z; qw[h][7] = w1.w;
    }
    qslot = slot;
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      m[h] = -INFINITY;
      lsum[h] = 0.0f;
      corr[h] = 0.0f;
#pragma unroll
      for (int e = 0; e < VPL; ++e) o2[h][e] = make_float2(0.0f, 0.0f);
    }
  }

  __device__ __forceinline__ void save() {
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      sm_[h] = m[h];
      sl_[h] = lsum[h];
      sc_[h] = corr[h];
#pragma unroll
      for (int e = 0; e < VPL; ++e) so_[h][e] = o2[h][e].x + o2[h][e].y;
    }
  }

  // one chunk: codes in `tile`, scales etc. in `small`, slots [s0, s0 + 32) of the unit
  __device__ __forceinline__ void chunk(const uint8_t *smem, const uint8_t *tile, const uint8_t *small, float *wbuf,
                                        int s0, int kv_u, bool has_mask, int lane) {
    const int g = lane / L, sub = lane % L;
    const int own = g + NG * sub;  // this lane's slot after the reduce-scatter
    int part[L][HC];
#pragma unroll
    for (int t = 0; t < L; ++t) {
      const int sl = g + NG * (t ^ sub);
      const uint2 cw = *reinterpret_cast<const uint2 *>(tile + sl * CB + sub * 8);
      const uint32_t c[4] = {cw.x & 0x0F0F0F0Fu, (cw.x >> 4) & 0x0F0F0F0Fu, cw.y & 0x0F0F0F0Fu,
                             (cw.y >> 4) & 0x0F0F0F0Fu};
#pragma unroll
      for (int h = 0; h < HC; ++h) {
        int acc = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc = dp2a_lo_su(qw[h][2 * i], c[i], acc);
          acc = dp2a_hi_su(qw[h][2 * i + 1], c[i], acc);
        }
        part[t][h] = acc;
      }
    }
    // reduce-scatter: lane sub holds slot t ^ sub at t, so its partner at distance
    // o holds the same slot at t + o (t < o); afterwards part[0] is slot `own`
#pragma unroll
    for (int o = L / 2; o >= 1; o >>= 1)
#pragma unroll
      for (int t = 0; t < o; ++t)
#pragma unroll
        for (int h = 0; h < HC; ++h) part[t][h] += __shfl_xor_sync(0xffffffffu, part[t + o][h], o);
    const bool valid = s0 + own < kv_u;
    const int kzp = static_cast<int8_t>(small[C::KZ_OFF + own]);
    const float ksc = reinterpret_cast<const float *>(small + C::KS_OFF)[own];
    const float vsc = reinterpret_cast<const float *>(small + C::VS_OFF)[own] * kWScale;
    const float zc = static_cast<float>(128 + static_cast<int8_t>(small[C::VZ_OFF + own]));
    const float madd = has_mask ? reinterpret_cast<const float *>(small + C::M_OFF)[own] * kLog2e : 0.0f;
    const int2 *qmeta = reinterpret_cast<const int2 *>(smem + C::QMETA_OFF) + qslot * HC;
    float sc[HC];
    bool need = false;
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      const int2 meta = qmeta[h];  // (sum n, 2^E)
      // exact: |sum n (c - zp)| < 2^31 (computed modulo 2^32)
      const int dz = static_cast<int>(static_cast<uint32_t>(part[0][h]) -
                                      static_cast<uint32_t>(kzp) * static_cast<uint32_t>(meta.x));
      sc[h] = valid ? fmaf(static_cast<float>(dz), __int_as_float(meta.y) * ksc, madd) : -INFINITY;
      need |= sc[h] > m[h] + kRescaleThreshold;
    }
    // the warp maximum is only needed when some score would overflow the lazy bound
    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int h = 0; h < HC; ++h) {
        float mt = sc[h];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
        const float mnew = fmaxf(m[h], mt);
        if (mnew > m[h] + kRescaleThreshold) {
          const float alpha = m[h] == -INFINITY ? 0.0f : ex2(m[h] - mnew);
          lsum[h] *= alpha;
          corr[h] *= alpha;
          const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
          for (int e = 0; e < VPL; ++e) o2[h][e] = __fmul2_rn(o2[h][e], al2);
          m[h] = mnew;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      const float p = sc[h] == -INFINITY ? 0.0f : ex2(sc[h] - m[h]);
      lsum[h] += p;
      const float wt = p > 0.0f ? p * vsc : 0.0f;
      corr[h] = fmaf(wt, zc, corr[h]);
      wbuf[h * CS + own] = wt;
    }
    __syncwarp();
    // p . v: lanes over dims, slots in fours (two packed FMAs per dim and head)
#pragma unroll 2
    for (int j = 0; j < CS; j += 4) {
      float4 w4[HC];
#pragma unroll
      for (int h = 0; h < HC; ++h) w4[h] = *reinterpret_cast<const float4 *>(wbuf + h * CS + j);
      float v[4][VPL];  // [slot j + i][dim lane * VPL + e] as subnormal floats
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint8_t *vrow = tile + C::KT + (j + i) * CB;  // VPL / 2 bytes: dim 2b in the low nibble of byte b
        uint32_t raw;
        if constexpr (VPL == 2) raw = vrow[lane];
        else if constexpr (VPL == 4) raw = reinterpret_cast<const uint16_t *>(vrow)[lane];
        else raw = reinterpret_cast<const uint32_t *>(vrow)[lane];
        const uint32_t lo = (raw & 0x0F0F0F0Fu) | 0x80808080u;
        const uint32_t hi = ((raw >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
#pragma unroll
        for (int e = 0; e < VPL; ++e) v[i][e] = byte_as_subnormal(e & 1 ? hi : lo, e >> 1);
      }
#pragma unroll
      for (int e = 0; e < VPL; ++e) {
        const float2 va = make_float2(v[0][e], v[1][e]), vb = make_float2(v[2][e], v[3][e]);
#pragma unroll
        for (int h = 0; h < HC; ++h) {
          o2[h][e] = __ffma2_rn(make_float2(w4[h].x, w4[h].y), va, o2[h][e]);
          o2[h][e] = __ffma2_rn(make_float2(w4[h].z, w4[h].w), vb, o2[h][e]);
        }
      }
    }
  }

  // write one unit's warp record (O [HC][D], then (m, l, corr, 0) [HC][4]) at dst
  __device__ __forceinline__ void publish(float *dst, bool first, int lane) {
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      float ll = first ? sl_[h] : lsum[h], cc = first ? sc_[h] : corr[h];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        ll += __shfl_xor_sync(0xffffffffu, ll, o);
        cc += __shfl_xor_sync(0xffffffffu, cc, o);
      }
      float oo[VPL];
#pragma unroll
      for (int e = 0; e < VPL; ++e) oo[e] = first ? so_[h][e] : o2[h][e].x + o2[h][e].y;
      float *od = dst + h * D + lane * VPL;
      if constexpr (VPL == 2) {
        *reinterpret_cast<float2 *>(od) = make_float2(oo[0], oo[1]);
      } else {
#pragma unroll
        for (int e = 0; e < VPL; e += 4)
          *reinterpret_cast<float4 *>(od + e) = make_float4(oo[e], oo[e + 1], oo[e + 2], oo[e + 3]);
      }
      if (lane == 0)
        *reinterpret_cast<float4 *>(dst + HC * D + h * 4) =
            make_float4(first ? sm_[h] : m[h], ll, cc * kWUnscale, 0.0f);
    }
  }
};

// ---------------------------------------------------------------------------
// Per-warp math of one unit on the tensor cores (int8 cache).  Lane t is
// (r, c) = (t / 4, t % 4), the MMA fragment coordinates.
//   q.K: A = q planes (row r: hi of head r, row r + 8: lo of head r), B = the K
//   tile (slots as columns); the int32 accumulator of n-tile nt gives lane
//   (r, c) both halves of head r's dot products with slots 8 nt + 2c, + 1.
//   P.V: O^T (16 dims x 8 heads) += V^T (16 dims x 16 slots) . P^T (16 slots x
//   8 heads).  P^T's fragment of lane (r, c) is head r at slots 2c, 2c + 1,
//   2c + 8, 2c + 9 of the k-step -- what its q.K accumulators hold.  The
//   m-tile of dims 16g .. 16g + 15 takes the even dims as rows 0..7 and the odd
//   dims as rows 8..15, which is how ldmatrix.trans hands out byte pairs.  Lane
//   (r, c) accumulates heads 2c, 2c + 1 at dims 16g + 2r, 16g + 2r + 1.
// ---------------------------------------------------------------------------
template <class C>
struct MmaCore {
  static constexpr int D = C::D, HC = C::HC, CS = C::CS, ROWB = C::ROWB, SUBT = C::SUBT;
  static constexpr int KS = D / 32;  // q.K k-steps
  static constexpr int MT = D / 16;  // P.V m-tiles
  static_assert(HC <= 8, "q heads of a unit fit the 8 MMA rows");
  static constexpr float OSCALE = 1.0f;    // records hold O itself
  // TQ4 cache: 4-bit codes 0..15, two a byte (element 2i in the low nibble of byte i)
  static constexpr bool Q4 = C::Q4;
  // a V code c enters as the fp16 value 1152 + c (int8), 1024 + c (TQ4)
  static constexpr float kVOff = Q4 ? 1024.0f : 1152.0f;

  uint32_t qa[KS][4];  // q A fragments
  int qslot;
  int nsum;             // head r: sum of its fixed-point q
  float es;             // head r: the q step 2^E
  float m, lsum, corr;  // head r: running max (same in the 4 lanes of the group), this lane's sums
  int vexp;             // E_v of the unit (weights are p * v_scale * 2^-E_v); warp-uniform
  float o[MT][4];       // O^T accumulators
  float sm_, sl_, sc_;  // the first unit's state (deferred close)
  int sv_;
  float so_[MT][4];

  // Physical address of byte `db` (a multiple of 16) of tile row `row`: TMA
  // wrote the tile in 128-byte (D >= 128: sub-tiles of 128 dims) or 64-byte
  // swizzled rows, which permute the 16-byte units of a row by its row index.
  static __device__ __forceinline__ uint32_t swz(uint32_t tile, int row, int db) {
    const int st = db / ROWB, unit = (db % ROWB) >> 4;
    const int x = ROWB == 128 ? (row & 7) : ((row >> 1) & 3);
    return tile + st * SUBT + row * ROWB + ((unit ^ x) << 4);
  }

  // q of one head as the converter gets it: the lane's D/32 bf16 values (dims
  // [lane * D/32, lane * D/32 + D/32)), loaded with one access so that the load can
  // be issued well before the conversion.
  struct QRaw {
    uint32_t w[D / 64];
  };
  static __device__ __forceinline__ QRaw load_q_raw(const uint16_t *qg, int lane) {
    QRaw r;
    if constexpr (D == 64) {
      r.w[0] = reinterpret_cast<const uint32_t *>(qg)[lane];
    } else if constexpr (D == 128) {
      const uint2 v = reinterpret_cast<const uint2 *>(qg)[lane];
      r.w[0] = v.x;
      r.w[1] = v.y;
    } else {
      const uint4 v = reinterpret_cast<const uint4 *>(qg)[lane];
      r.w[0] = v.x;
      r.w[1] = v.y;
      r.w[2] = v.z;
      r.w[3] = v.w;
    }
    return r;
  }

  // warp `h` (< HC): head h of q onto the fixed-point grid, split into the two
  // signed byte planes n = 256 hi + lo, into q slot `slot` ([plane][HC][D] bytes)
  static __device__ __forceinline__ void convert_q(uint8_t *smem, const QRaw &raw, float qscale, int slot, int h,
                                                   int lane) {
    constexpr int PER = D / 32;  // dims per lane: [lane * PER, lane * PER + PER)
    float x[PER];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const uint32_t w = raw.w[i / 2];
      x[i] = ((i & 1) ? bf16hi(w) : bf16lo(w)) * qscale;
      amax = fmaxf(amax, fabsf(x[i]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // step 2^E with amax / 2^E < 2^15: E = floor(log2 amax) + 1 - 15; one more when
    // some |n| exceeds 32639, so that hi = (n - lo) / 256 stays a signed byte
    int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127 + 1 - 15;
    E = E < -126 ? -126 : E;
    int n[PER];
    bool big = false;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      n[i] = __float2int_rn(x[i] * pow2i(-E));
      big |= n[i] > 32639 || n[i] < -32639;
    }
    if (__any_sync(0xffffffffu, big)) {
      E += 1;
#pragma unroll
      for (int i = 0; i < PER; ++i) n[i] = __float2int_rn(x[i] * pow2i(-E));
    }
    int s = 0;
    constexpr int NWRD = PER >= 4 ? PER / 4 : 1;
    uint32_t hw[NWRD] = {}, lw[NWRD] = {};
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      s += n[i];
      const int lo = ((n[i] + 128) & 255) - 128;
      const int hi = (n[i] - lo) >> 8;
      hw[i / 4] |= (static_cast<uint32_t>(hi) & 0xFFu) << (8 * (i % 4));
      lw[i / 4] |= (static_cast<uint32_t>(lo) & 0xFFu) << (8 * (i % 4));
    }
    uint8_t *hp = smem + C::Q_OFF + slot * 2 * HC * D + h * D + lane * PER;
    uint8_t *lp = hp + HC * D;
    if constexpr (PER == 2) {
      *reinterpret_cast<uint16_t *>(hp) = static_cast<uint16_t>(hw[0]);
      *reinterpret_cast<uint16_t *>(lp) = static_cast<uint16_t>(lw[0]);
    } else {
#pragma unroll
      for (int i = 0; i < PER / 4; ++i) {
        reinterpret_cast<uint32_t *>(hp)[i] = hw[i];
        reinterpret_cast<uint32_t *>(lp)[i] = lw[i];
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      int32_t *meta = reinterpret_cast<int32_t *>(smem + C::QMETA_OFF) + (slot * HC + h) * 2;
      meta[0] = s;
      meta[1] = static_cast<int32_t>(__float_as_uint(pow2i(E)));
    }
  }

  __device__ __forceinline__ void load_q(const uint8_t *smem, int slot, int lane) {
    const int r = lane >> 2, c = lane & 3;
    const bool on = r < HC;
    const uint8_t *hp = smem + C::Q_OFF + slot * 2 * HC * D + (on ? r : 0) * D;
    const uint8_t *lp = hp + HC * D;
    // k-step k: lane c's K bytes are dims 32 k + 4 c .. + 3 and 32 k + 16 + 4 c .. + 3 (int8);
    // TQ4: its 8 codes of one ldmatrix row are dims 32 k + 8 c .. + 7, unpacked in that order
    const int o0 = Q4 ? 8 * c : 4 * c, o1 = Q4 ? 8 * c + 4 : 16 + 4 * c;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      qa[k][0] = on ? *reinterpret_cast<const uint32_t *>(hp + 32 * k + o0) : 0u;
      qa[k][1] = on ? *reinterpret_cast<const uint32_t *>(lp + 32 * k + o0) : 0u;
      qa[k][2] = on ? *reinterpret_cast<const uint32_t *>(hp + 32 * k + o1) : 0u;
      qa[k][3] = on ? *reinterpret_cast<const uint32_t *>(lp + 32 * k + o1) : 0u;
    }
    qslot = slot;
    const int2 meta = reinterpret_cast<const int2 *>(smem + C::QMETA_OFF)[slot * HC + (on ? r : 0)];
    nsum = meta.x;
    es = __int_as_float(meta.y);
  }

  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    lsum = 0.0f;
    corr = 0.0f;
    vexp = -127;
#pragma unroll
    for (int g = 0; g < MT; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[g][i] = 0.0f;
  }

  __device__ __forceinline__ void save() {
    sm_ = m;
    sl_ = lsum;
    sc_ = corr;
    sv_ = vexp;
#pragma unroll
    for (int g = 0; g < MT; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) so_[g][i] = o[g][i];
  }

  __device__ __forceinline__ void chunk(const uint8_t *smem, const uint8_t *tile, const uint8_t *small, float *scr,
                                        int s0, int kv_u, bool has_mask, int lane) {
    constexpr int NT = CS / 8;   // q.K n-tiles (8 slots each)
    constexpr int PK = CS / 16;  // P.V k-steps (16 slots each)
    const int r = lane >> 2, c = lane & 3;
    const uint32_t kt = smem_u32(tile), vt = kt + C::KT;
    // ---- per-slot values, one lane per slot: (k scale, k zero point, mask, v scale),
    // with scales 0 and the mask -inf past kv_len, and 1152 + v zero point
    float4 *s4 = reinterpret_cast<float4 *>(scr);
    float *zcs = scr + 4 * CS;
    float vmax = 0.0f;
#pragma unroll
    for (int i = 0; i < CS / 32; ++i) {
      const int j = lane + 32 * i;
      const bool valid = s0 + j < kv_u;
      const float ks = reinterpret_cast<const float *>(small + C::KS_OFF)[j];
      const float vs = reinterpret_cast<const float *>(small + C::VS_OFF)[j];
      const int kz = static_cast<int8_t>(small[C::KZ_OFF + j]);
      const int vz = static_cast<int8_t>(small[C::VZ_OFF + j]);
      const float mk = has_mask ? reinterpret_cast<const float *>(small + C::M_OFF)[j] * kLog2e : 0.0f;
      float4 f;
      f.x = valid ? ks : 0.0f;
      f.y = __int_as_float(kz);
      f.z = valid ? mk : -INFINITY;
      f.w = valid ? vs : 0.0f;
      s4[j] = f;
      zcs[j] = kVOff + static_cast<float>(vz);
      vmax = fmaxf(vmax, f.w);
    }
    // the chunk's largest v scale (the same in every lane)
#pragma unroll
    for (int sft = 16; sft >= 1; sft >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, sft));
    // ---- q.K: n-tile nt = slots 8 nt .. 8 nt + 7; ldmatrix x4 gives the B
    // fragments of two k-steps (64 dims) for one n-tile
    int sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sacc[nt][i] = 0;
      if constexpr (Q4) {  // 64 bytes of codes = four k-steps; nibbles unpacked to bytes 0..15
#pragma unroll
        for (int kp = 0; kp < KS / 4; ++kp) {
          uint32_t b[4];
          ldsm_x4(b, swz(kt, nt * 8 + (lane & 7), 64 * kp + 16 * (lane >> 3)));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t lo = b[i] & 0x0F0F0F0Fu, hi = (b[i] >> 4) & 0x0F0F0F0Fu;
            mma_s8(sacc[nt], qa[4 * kp + i], __byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
          }
        }
      } else {
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
          uint32_t b[4];
          ldsm_x4(b, swz(kt, nt * 8 + (lane & 7), 64 * kp + 16 * (lane >> 3)));
          mma_s8(sacc[nt], qa[2 * kp], b[0], b[1]);
          mma_s8(sacc[nt], qa[2 * kp + 1], b[2], b[3]);
        }
      }
    }
    __syncwarp();  // the per-slot values are written
    // ---- scores of head r at slots j = 8 nt + 2c + e (log2 domain)
    float sc[NT][2], vv[NT][2], zc[NT][2];
    float mt = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int j = nt * 8 + 2 * c;
      const float2 z2 = *reinterpret_cast<const float2 *>(zcs + j);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float4 f = s4[j + e];
        // exact: 256 (hi . k) + (lo . k) - zp * sum n = sum n (k - zp), |.| < 2^31 (modulo 2^32)
        const uint32_t dot = (static_cast<uint32_t>(sacc[nt][e]) << 8) + static_cast<uint32_t>(sacc[nt][2 + e]);
        const int dz = static_cast<int>(dot - static_cast<uint32_t>(__float_as_int(f.y)) * static_cast<uint32_t>(nsum));
        sc[nt][e] = fmaf(static_cast<float>(dz), es * f.x, f.z);  // -inf past kv_len (k scale 0 there)
        vv[nt][e] = f.w;
        zc[nt][e] = e ? z2.y : z2.x;
        mt = fmaxf(mt, sc[nt][e]);
      }
    }
    // the head's maximum over the chunk (the 4 lanes of group r)
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const bool need = r < HC && mt > m + kRescaleThreshold;
    if (__any_sync(0xffffffffu, need)) {
      const float alpha = need ? (m == -INFINITY ? 0.0f : ex2(m - mt)) : 1.0f;
      if (need) {
        lsum *= alpha;
        corr *= alpha;
        m = mt;
      }
      // lane (r, c) accumulates heads 2c and 2c + 1, whose factors live in groups 2c, 2c + 1
      const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * c);
      const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * c + 4);
#pragma unroll
      for (int g = 0; g < MT; ++g) {
        o[g][0] *= a0;
        o[g][1] *= a1;
        o[g][2] *= a0;
        o[g][3] *= a1;
      }
    }
    // weights w = p * v_scale * 2^-E_v below 2^15 (p <= 2^8); E_v only grows
    if (vmax > 0.0f) {
      int ev = static_cast<int>((__float_as_uint(vmax) >> 23) & 0xFF) - 127 - 6;
      ev = ev < -120 ? -120 : (ev > 120 ? 120 : ev);
      if (ev > vexp) {
        const float f = vexp - ev < -126 ? 0.0f : pow2i(vexp - ev);
        corr *= f;
#pragma unroll
        for (int g = 0; g < MT; ++g)
#pragma unroll
          for (int i = 0; i < 4; ++i) o[g][i] *= f;
        vexp = ev;
      }
    }
    // lanes of rows past HC carry no head: their weights are 0 (the +inf maximum makes p 0)
    const float vsc = r < HC ? pow2i(-vexp) : 0.0f;
    const float mm = r < HC ? (m == -INFINITY ? 0.0f : m) : INFINITY;
    uint32_t ph[NT], pl[NT];  // P^T fragments: [nt] = f16x2 (hi / lo) of head r at slots 8 nt + 2c, + 1
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float w[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float p = ex2(sc[nt][e] - mm);  // 0 for -inf scores
        lsum += p;
        w[e] = p * (vv[nt][e] * vsc);
        corr = fmaf(w[e], zc[nt][e], corr);
      }
      ph[nt] = pack_f16x2(w[0], w[1]);
      const float2 back = unpack_f16x2(ph[nt]);
      pl[nt] = pack_f16x2(w[0] - back.x, w[1] - back.y);
    }
    // ---- P.V: k-step ks = slots 16 ks .. 16 ks + 15; ldmatrix.trans x4 gives the
    // V^T fragments of two m-tiles (32 dims)
    if constexpr (Q4) {
      // 32 bytes of V codes = 64 dims (gp): a 16-bit element of ldmatrix.trans is four
      // dims of one slot; a byte permute and a nibble swap give, per byte j, dim 4 i + j
      // of slots 2c and 2c + 1, made the fp16 pair (1024 + c0, 1024 + c1).  Four MMAs j,
      // m-tile 4 gp + j: row i is dim 64 gp + 4 i + j, row i + 8 is dim 64 gp + 32 + 4 i + j.
#pragma unroll
      for (int ks = 0; ks < PK; ++ks) {
#pragma unroll
        for (int gp = 0; gp < D / 64; ++gp) {
          uint32_t mr[4];
          const int mi = lane >> 3;
          ldsm_x4_trans(mr, swz(vt, 16 * ks + 8 * (mi & 1) + (lane & 7), 32 * gp + 16 * (mi >> 1)));
          uint32_t y[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t x = __byte_perm(mr[i], 0u, 0x3120);  // bytes: s lo, s+1 lo, s hi, s+1 hi
            const uint32_t t = ((x >> 4) ^ x) & 0x00F000F0u;     // swap the middle nibbles of each half
            y[i] = x ^ t ^ (t << 4);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t a[4];
            const int src[4] = {0, 2, 1, 3};  // a0: unit 2gp slots 2c..; a1: unit 2gp+1; a2, a3: slots + 8
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t bj = (y[src[e]] >> (8 * j)) & 0xFFu;
              a[e] = (bj & 0x0Fu) | ((bj & 0xF0u) << 12) | 0x64006400u;
            }
            mma_f16(o[4 * gp + j], a, ph[2 * ks], ph[2 * ks + 1]);
            mma_f16(o[4 * gp + j], a, pl[2 * ks], pl[2 * ks + 1]);
          }
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < PK; ++ks) {
#pragma unroll
        for (int gp = 0; gp < MT / 2; ++gp) {
          uint32_t mr[4];
          const int mi = lane >> 3;  // matrix: rows 16 ks + 8 (mi & 1) .., dim bytes 32 gp + 16 (mi >> 1)
          ldsm_x4_trans(mr, swz(vt, 16 * ks + 8 * (mi & 1) + (lane & 7), 32 * gp + 16 * (mi >> 1)));
          uint32_t af[2][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // bytes: (slot 2c, dim 2n), (2c, 2n + 1), (2c + 1, 2n), (2c + 1, 2n + 1); +128 then fp16 0x64xx
            const uint32_t x = mr[i] ^ 0x80808080u;
            const uint32_t ev = __byte_perm(x, 0x64646464u, 0x4240u);  // dim 2n of slots 2c, 2c + 1
            const uint32_t od = __byte_perm(x, 0x64646464u, 0x4341u);  // dim 2n + 1
            // matrices 0, 1: m-tile 2gp (slots +0, +8); 2, 3: m-tile 2gp + 1
            af[i >> 1][(i & 1) * 2 + 0] = ev;
            af[i >> 1][(i & 1) * 2 + 1] = od;
          }
          // A fragment order: a0 = rows 0..7 (even dims) k 0..7, a1 = rows 8..15 (odd) k 0..7, a2/a3 k 8..15
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t a[4] = {af[t][0], af[t][1], af[t][2], af[t][3]};
            mma_f16(o[2 * gp + t], a, ph[2 * ks], ph[2 * ks + 1]);
            mma_f16(o[2 * gp + t], a, pl[2 * ks], pl[2 * ks + 1]);
          }
        }
      }
    }
  }

  // write one unit's warp record (O [HC][D], then (m, l, corr, 0) [HC][4]) at dst,
  // O and corr scaled back by 2^E_v
  __device__ __forceinline__ void publish(float *dst, bool first, int lane) {
    const int r = lane >> 2, c = lane & 3;
    float ll = first ? sl_ : lsum, cc = first ? sc_ : corr;
    ll += __shfl_xor_sync(0xffffffffu, ll, 1);
    ll += __shfl_xor_sync(0xffffffffu, ll, 2);
    cc += __shfl_xor_sync(0xffffffffu, cc, 1);
    cc += __shfl_xor_sync(0xffffffffu, cc, 2);
    const float sv = pow2i(first ? sv_ : vexp);
#pragma unroll
    for (int g = 0; g < MT; ++g) {
      const float *og = first ? so_[g] : o[g];
      if constexpr (Q4) {  // rows r, r + 8 of m-tile g: dims 64 (g / 4) + 4 r + g % 4, and + 32
        const int d = 64 * (g >> 2) + 4 * r + (g & 3);
        if (2 * c < HC) {
          dst[(2 * c) * D + d] = og[0] * sv;
          dst[(2 * c) * D + d + 32] = og[2] * sv;
        }
        if (2 * c + 1 < HC) {
          dst[(2 * c + 1) * D + d] = og[1] * sv;
          dst[(2 * c + 1) * D + d + 32] = og[3] * sv;
        }
      } else {
        const int d = 16 * g + 2 * r;
        if (2 * c < HC) *reinterpret_cast<float2 *>(dst + (2 * c) * D + d) = make_float2(og[0] * sv, og[2] * sv);
        if (2 * c + 1 < HC)
          *reinterpret_cast<float2 *>(dst + (2 * c + 1) * D + d) = make_float2(og[1] * sv, og[3] * sv);
      }
    }
    if (r < HC && c == 0)
      *reinterpret_cast<float4 *>(dst + HC * D + r * 4) = make_float4(first ? sm_ : m, ll, cc * sv, 0.0f);
  }
};

// ---------------------------------------------------------------------------
// Per-warp math of one unit over a per-32 block cache (kvq_write modes 1, 2, 4,
// 5, 6; IndexerQuantCache, 计算公式: x ~ code * scale_g), on the tensor cores.
//  - Codes become fp16 on the way into the MMAs, exactly (cvt for E4M3, a byte
//    move for E5M2, the 1024-mantissa form for int8), and are multiplied by
//    their group's factor scale_g * 2^-E_s, with 2^E_s one power of two per
//    slot at or above the slot's largest group scale: exact for E8M0 scales
//    (down to 2^-24 of the slot's largest factor), one rounding for float
//    scales.  2^E_s of K multiplies the fp32 score; 2^F_s of V takes v_scale's
//    place in P.  There is no zero point.
//  - q.K: f16 m16n8k16 with q in rows 0..7 as exact fp16 (a power-of-two step
//    per head; the score scale is applied in fp32).  An ldmatrix row of the K
//    tile gives a lane four consecutive codes of one slot, so the MMA's k order
//    is permuted to match: lane c's k pairs (2c, 2c + 1) and (2c + 8, 2c + 9)
//    are dims 4c, 4c + 1 and 4c + 2, 4c + 3 of a 16-dim step, in q's fragments
//    as in K's, which leaves every dot product unchanged.
//  - Softmax and P.V as in MmaCore, the V codes converted and scaled per group.
// ---------------------------------------------------------------------------
template <class C>
struct BlkCore {
  static constexpr int D = C::D, HC = C::HC, CS = C::CS, ROWB = C::ROWB, SUBT = C::SUBT, MODE = C::MODE;
  static constexpr int NG = C::NGS;
  static constexpr int KT16 = D / 16;  // q.K k-steps of 16 dims
  static constexpr int MT = D / 16;    // P.V m-tiles
  static constexpr bool F32S = C::F32S;
  static constexpr bool E5 = MODE == KVQ_MODE_FP8_E5M2 || MODE == KVQ_MODE_MXFP8_E5M2;
  static constexpr bool I8 = MODE == KVQ_MODE_INT8_SYM;
  // MX-FP4: two E2M1 codes a byte (element 2i in the low nibble of byte i), so a
  // 16-byte ldmatrix row holds 32 dims, one scale group
  static constexpr bool FP4 = MODE == KVQ_MODE_MXFP4;
  static_assert(HC <= 8, "q heads of a unit fit the 8 MMA rows");
  static constexpr float OSCALE = 1.0f;  // records hold O itself

  uint32_t qa[KT16][2];  // q A fragment words a0, a2 (rows 8..15 carry no head)
  int qslot;
  float es;              // head r: qscale * the q step 2^E
  float m, lsum, corr;   // corr stays 0 (no zero point)
  int vexp;
  float o[MT][4];
  float sm_, sl_, sc_;
  int sv_;
  float so_[MT][4];

  static __device__ __forceinline__ uint32_t swz(uint32_t tile, int row, int db) {
    const int st = db / ROWB, unit = (db % ROWB) >> 4;
    const int x = ROWB == 128 ? (row & 7) : ((row >> 1) & 3);
    return tile + st * SUBT + row * ROWB + ((unit ^ x) << 4);
  }

  struct QRaw {
    uint32_t w[D / 64];
  };
  static __device__ __forceinline__ QRaw load_q_raw(const uint16_t *qg, int lane) {
    QRaw r;
    if constexpr (D == 64) {
      r.w[0] = reinterpret_cast<const uint32_t *>(qg)[lane];
    } else if constexpr (D == 128) {
      const uint2 v = reinterpret_cast<const uint2 *>(qg)[lane];
      r.w[0] = v.x;
      r.w[1] = v.y;
    } else {
      const uint4 v = reinterpret_cast<const uint4 *>(qg)[lane];
      r.w[0] = v.x;
      r.w[1] = v.y;
      r.w[2] = v.z;
      r.w[3] = v.w;
    }
    return r;
  }

  // warp `h`: head h of q as fp16 times 2^-E, max |q| 2^-E in [2^14, 2^15) (exact for
  // every bf16 element at least 2^-24 of the step), into q slot `slot` ([HC][D] fp16);
  // meta (0, qscale * 2^E)
  static __device__ __forceinline__ void convert_q(uint8_t *smem, const QRaw &raw, float qscale, int slot, int h,
                                                   int lane) {
    constexpr int PER = D / 32;
    float x[PER];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const uint32_t w = raw.w[i / 2];
      x[i] = (i & 1) ? bf16hi(w) : bf16lo(w);
      amax = fmaxf(amax, fabsf(x[i]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int E = amax > 0.0f ? static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127 + 1 - 15 : 0;
    E = E < -126 ? -126 : E;
    const float inv = pow2i(-E);
    uint32_t hw[PER / 2];
#pragma unroll
    for (int i = 0; i < PER / 2; ++i) hw[i] = pack_f16x2(x[2 * i] * inv, x[2 * i + 1] * inv);
    uint8_t *hp = smem + C::Q_OFF + ((slot * HC + h) * D + lane * PER) * 2;
    if constexpr (PER == 2) {
      *reinterpret_cast<uint32_t *>(hp) = hw[0];
    } else if constexpr (PER == 4) {
      *reinterpret_cast<uint2 *>(hp) = make_uint2(hw[0], hw[1]);
    } else {
      *reinterpret_cast<uint4 *>(hp) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
    if (lane == 0) {
      int32_t *meta = reinterpret_cast<int32_t *>(smem + C::QMETA_OFF) + (slot * HC + h) * 2;
      meta[0] = 0;
      meta[1] = static_cast<int32_t>(__float_as_uint(qscale * pow2i(E)));
    }
  }

  __device__ __forceinline__ void load_q(const uint8_t *smem, int slot, int lane) {
    const int r = lane >> 2, c = lane & 3;
    const bool on = r < HC;
    const uint8_t *qp = smem + C::Q_OFF + (slot * HC + (on ? r : 0)) * D * 2;
    if constexpr (FP4) {  // k-steps 2u, 2u + 1 of group u: lane c takes dims 32 u + 8 c .. + 7
#pragma unroll
      for (int u = 0; u < D / 32; ++u) {
        const uint4 v = *reinterpret_cast<const uint4 *>(qp + (32 * u + 8 * c) * 2);
        qa[2 * u][0] = on ? v.x : 0u;
        qa[2 * u][1] = on ? v.y : 0u;
        qa[2 * u + 1][0] = on ? v.z : 0u;
        qa[2 * u + 1][1] = on ? v.w : 0u;
      }
    } else {
#pragma unroll
      for (int t = 0; t < KT16; ++t) {
        const uint2 v = *reinterpret_cast<const uint2 *>(qp + (16 * t + 4 * c) * 2);
        qa[t][0] = on ? v.x : 0u;
        qa[t][1] = on ? v.y : 0u;
      }
    }
    qslot = slot;
    es = __int_as_float(reinterpret_cast<const int2 *>(smem + C::QMETA_OFF)[slot * HC + (on ? r : 0)].y);
  }

  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    lsum = 0.0f;
    corr = 0.0f;
    vexp = -127;
#pragma unroll
    for (int g = 0; g < MT; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[g][i] = 0.0f;
  }

  __device__ __forceinline__ void save() {
    sm_ = m;
    sl_ = lsum;
    sc_ = corr;
    sv_ = vexp;
#pragma unroll
    for (int g = 0; g < MT; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) so_[g][i] = o[g][i];
  }

  // four codes (byte i = code i) -> fp16 pairs (codes 0, 1) and (2, 3), exact
  static __device__ __forceinline__ void codes4(uint32_t w, uint32_t &h01, uint32_t &h23) {
    if constexpr (E5) {
      h01 = __byte_perm(w, 0u, 0x1404);
      h23 = __byte_perm(w, 0u, 0x3424);
    } else if constexpr (I8) {
      const uint32_t u = w ^ 0x80808080u;
      h01 = sub1152(__byte_perm(u, 0x64646464u, 0x4140));
      h23 = sub1152(__byte_perm(u, 0x64646464u, 0x4342));
    } else {
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"(static_cast<uint16_t>(w & 0xFFFFu)));
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"(static_cast<uint16_t>(w >> 16)));
    }
  }
  // codes in bytes 0 and 2 (ev) or 1 and 3 (od) of w -> one fp16 pair, exact
  template <bool ODD>
  static __device__ __forceinline__ uint32_t codes2(uint32_t w) {
    if constexpr (E5) {
      return __byte_perm(w, 0u, ODD ? 0x3414 : 0x2404);
    } else if constexpr (I8) {
      return sub1152(__byte_perm(w ^ 0x80808080u, 0x64646464u, ODD ? 0x4341 : 0x4240));
    } else {
      uint32_t h;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(__byte_perm(w, 0u, ODD ? 0x0031 : 0x0020))));
      return h;
    }
  }
  // the E2M1 codes in the low byte of w -> fp16 pair (low nibble first), exact
  static __device__ __forceinline__ uint32_t e2m1x2(uint32_t w) {
    uint32_t h;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h) : "r"(w));
    return h;
  }
  // ldmatrix.trans word of E2M1 codes: dims 4i .. 4i + 3 of slot s (bytes 0, 1) and
  // of slot s + 1 (bytes 2, 3) -> byte j holds dim 4i + j of slot s (low nibble) and
  // of slot s + 1 (high nibble)
  static __device__ __forceinline__ uint32_t fp4_slot_pairs(uint32_t w) {
    const uint32_t x = __byte_perm(w, 0u, 0x3120);    // bytes: s lo, s+1 lo, s hi, s+1 hi
    const uint32_t t = ((x >> 4) ^ x) & 0x00F000F0u;  // swap the middle nibbles of each half
    return x ^ t ^ (t << 4);
  }
  static __device__ __forceinline__ uint32_t sub1152(uint32_t h) {
    const __half2 r = __hsub2(*reinterpret_cast<const __half2 *>(&h),
                              __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
    return *reinterpret_cast<const uint32_t *>(&r);
  }
  // an fp16 pair times (f0, f1): E8M0 factors are powers of two (exact product);
  // float factors take the pair through fp32 and round once
  static __device__ __forceinline__ uint32_t scale2(uint32_t h, float f0, float f1) {
    if constexpr (F32S) {
      const float2 v = unpack_f16x2(h);
      return pack_f16x2(v.x * f0, v.y * f1);
    } else {
      const __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&h), __floats2half2_rn(f0, f1));
      return *reinterpret_cast<const uint32_t *>(&r);
    }
  }
  // the exponent of a slot and its group factors scale_g * 2^-E, from the slot's
  // scale row (NG floats, or NG E8M0 bytes)
  static __device__ __forceinline__ int slot_factors(const uint8_t *row, float (&f)[NG]) {
    if constexpr (F32S) {
      uint32_t mx = 0u;
      float sg[NG];
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        sg[g] = reinterpret_cast<const float *>(row)[g];
        mx = max(mx, __float_as_uint(sg[g]) & 0x7FFFFFFFu);
      }
      int E = 0;
      if (mx != 0u) {  // ceil(log2) of the largest scale, from its bits
        const int ex = static_cast<int>(mx >> 23);
        E = ex == 0 ? -126 : ex - 127 + ((mx & 0x7FFFFFu) != 0u ? 1 : 0);
        E = E < -126 ? -126 : (E > 126 ? 126 : E);
      }
      const float inv = pow2i(-E);
#pragma unroll
      for (int g = 0; g < NG; ++g) f[g] = sg[g] * inv;
      return E;
    } else {
      int e[NG], mx = 0;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        e[g] = row[g];
        mx = max(mx, e[g]);
      }
      const int E = max(-126, mx - 127);
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const int k = e[g] - 127 - E;  // <= 0
        f[g] = k >= -126 ? pow2i(k) : 0.0f;
      }
      return E;
    }
  }

  __device__ __forceinline__ void chunk(const uint8_t *smem, const uint8_t *tile, const uint8_t *small, float *scr,
                                        int s0, int kv_u, bool has_mask, int lane) {
    constexpr int NT = CS / 8;   // q.K n-tiles (8 slots each)
    constexpr int PK = CS / 16;  // P.V k-steps (16 slots each)
    constexpr int RB = NG * C::SB;
    const int r = lane >> 2, c = lane & 3;
    const uint32_t kt = smem_u32(tile), vt = kt + C::KT;
    float4 *s4 = reinterpret_cast<float4 *>(scr);  // [CS] (k factor, -, mask, v factor)
    float *kf = scr + 4 * CS;                      // [NG][CS] K group factors
    float *vf = kf + NG * CS;                      // [NG][CS] V group factors
    // ---- per-slot factors, one lane per slot (0 past kv_len, where the mask is -inf)
    float vmax = 0.0f;
#pragma unroll
    for (int i = 0; i < CS / 32; ++i) {
      const int j = lane + 32 * i;
      const bool valid = s0 + j < kv_u;
      float fk[NG], fv[NG];
      const int ek = slot_factors(small + C::KS_OFF + j * RB, fk);
      const int ev = slot_factors(small + C::VS_OFF + j * RB, fv);
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        kf[g * CS + j] = valid ? fk[g] : 0.0f;
        vf[g * CS + j] = valid ? fv[g] : 0.0f;
      }
      const float mk = has_mask ? reinterpret_cast<const float *>(small + C::M_OFF)[j] * kLog2e : 0.0f;
      float4 f;
      f.x = valid ? pow2i(ek) : 0.0f;
      f.y = 0.0f;
      f.z = valid ? mk : -INFINITY;
      f.w = valid ? pow2i(ev) : 0.0f;
      s4[j] = f;
      vmax = fmaxf(vmax, f.w);
    }
#pragma unroll
    for (int sft = 16; sft >= 1; sft >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, sft));
    __syncwarp();  // the factors are written
    // ---- q.K: n-tile nt = slots 8 nt .. 8 nt + 7; ldmatrix x4 gives four 16-dim
    // steps (64 dims) of one n-tile, lane (r, c) holding dims 4c .. 4c + 3 of slot r
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sacc[nt][i] = 0.0f;
      if constexpr (FP4) {  // matrix i of an ldmatrix x4: scale group u = 4 kp + i, lane c: dims 8 c .. 8 c + 7
#pragma unroll
        for (int kp = 0; kp < D / 128; ++kp) {
          uint32_t b[4];
          ldsm_x4(b, swz(kt, nt * 8 + (lane & 7), 64 * kp + 16 * (lane >> 3)));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int u = 4 * kp + i;
            const float f = kf[u * CS + nt * 8 + r];
            uint32_t h[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) h[j] = scale2(e2m1x2(b[i] >> (8 * j)), f, f);
            const uint32_t a0[4] = {qa[2 * u][0], 0u, qa[2 * u][1], 0u};
            mma_f16(sacc[nt], a0, h[0], h[1]);
            const uint32_t a1[4] = {qa[2 * u + 1][0], 0u, qa[2 * u + 1][1], 0u};
            mma_f16(sacc[nt], a1, h[2], h[3]);
          }
        }
      } else {
#pragma unroll
        for (int kp = 0; kp < D / 64; ++kp) {
          uint32_t b[4];
          ldsm_x4(b, swz(kt, nt * 8 + (lane & 7), 64 * kp + 16 * (lane >> 3)));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int t = 4 * kp + i;
            const float f = kf[(t >> 1) * CS + nt * 8 + r];
            uint32_t b0, b1;
            codes4(b[i], b0, b1);
            b0 = scale2(b0, f, f);
            b1 = scale2(b1, f, f);
            const uint32_t a[4] = {qa[t][0], 0u, qa[t][1], 0u};
            mma_f16(sacc[nt], a, b0, b1);
          }
        }
      }
    }
    // ---- scores of head r at slots j = 8 nt + 2c + e (log2 domain)
    float sc[NT][2], vv[NT][2];
    float mt = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int j = nt * 8 + 2 * c;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float4 f = s4[j + e];
        sc[nt][e] = fmaf(sacc[nt][e], es * f.x, f.z);  // -inf past kv_len (k factor 0 there)
        vv[nt][e] = f.w;
        mt = fmaxf(mt, sc[nt][e]);
      }
    }
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const bool need = r < HC && mt > m + kRescaleThreshold;
    if (__any_sync(0xffffffffu, need)) {
      const float alpha = need ? (m == -INFINITY ? 0.0f : ex2(m - mt)) : 1.0f;
      if (need) {
        lsum *= alpha;
        m = mt;
      }
      const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * c);
      const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * c + 4);
#pragma unroll
      for (int g = 0; g < MT; ++g) {
        o[g][0] *= a0;
        o[g][1] *= a1;
        o[g][2] *= a0;
        o[g][3] *= a1;
      }
    }
    // weights w = p * 2^F * 2^-E_v below 2^15 (p <= 2^8); E_v only grows
    if (vmax > 0.0f) {
      int evx = static_cast<int>((__float_as_uint(vmax) >> 23) & 0xFF) - 127 - 6;
      evx = evx < -120 ? -120 : (evx > 120 ? 120 : evx);
      if (evx > vexp) {
        const float f = vexp - evx < -126 ? 0.0f : pow2i(vexp - evx);
#pragma unroll
        for (int g = 0; g < MT; ++g)
#pragma unroll
          for (int i = 0; i < 4; ++i) o[g][i] *= f;
        vexp = evx;
      }
    }
    const float vsc = r < HC ? pow2i(-vexp) : 0.0f;
    const float mm = r < HC ? (m == -INFINITY ? 0.0f : m) : INFINITY;
    uint32_t ph[NT], pl[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float w[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float p = ex2(sc[nt][e] - mm);
        lsum += p;
        w[e] = p * (vv[nt][e] * vsc);
      }
      ph[nt] = pack_f16x2(w[0], w[1]);
      const float2 back = unpack_f16x2(ph[nt]);
      pl[nt] = pack_f16x2(w[0] - back.x, w[1] - back.y);
    }
    // ---- P.V: k-step ks = slots 16 ks .. 16 ks + 15, m-tile pair gp = dims 32 gp ..
    // 32 gp + 31 (one scale group)
    if constexpr (FP4) {
      // group pair gp (dims 64 gp .. + 63, two scale groups) of slots 16 ks .. + 15: four
      // MMAs j, m-tile 4 gp + j, whose row i is dim 64 gp + 4 i + j and row i + 8 is
      // dim 64 gp + 32 + 4 i + j
#pragma unroll
      for (int ks = 0; ks < PK; ++ks) {
#pragma unroll
        for (int gp = 0; gp < D / 64; ++gp) {
          uint32_t mr[4];
          const int mi = lane >> 3;
          ldsm_x4_trans(mr, swz(vt, 16 * ks + 8 * (mi & 1) + (lane & 7), 32 * gp + 16 * (mi >> 1)));
          const float2 f00 = *reinterpret_cast<const float2 *>(vf + (2 * gp) * CS + 16 * ks + 2 * c);
          const float2 f01 = *reinterpret_cast<const float2 *>(vf + (2 * gp) * CS + 16 * ks + 8 + 2 * c);
          const float2 f10 = *reinterpret_cast<const float2 *>(vf + (2 * gp + 1) * CS + 16 * ks + 2 * c);
          const float2 f11 = *reinterpret_cast<const float2 *>(vf + (2 * gp + 1) * CS + 16 * ks + 8 + 2 * c);
          uint32_t y[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) y[i] = fp4_slot_pairs(mr[i]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t a[4] = {scale2(e2m1x2(y[0] >> (8 * j)), f00.x, f00.y),
                                   scale2(e2m1x2(y[2] >> (8 * j)), f10.x, f10.y),
                                   scale2(e2m1x2(y[1] >> (8 * j)), f01.x, f01.y),
                                   scale2(e2m1x2(y[3] >> (8 * j)), f11.x, f11.y)};
            mma_f16(o[4 * gp + j], a, ph[2 * ks], ph[2 * ks + 1]);
            mma_f16(o[4 * gp + j], a, pl[2 * ks], pl[2 * ks + 1]);
          }
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < PK; ++ks) {
#pragma unroll
        for (int gp = 0; gp < MT / 2; ++gp) {
          uint32_t mr[4];
          const int mi = lane >> 3;
          ldsm_x4_trans(mr, swz(vt, 16 * ks + 8 * (mi & 1) + (lane & 7), 32 * gp + 16 * (mi >> 1)));
          // factors of slots 16 ks + 2c, + 1 (matrices 0, 2) and 16 ks + 8 + 2c, + 1 (1, 3)
          const float2 fa = *reinterpret_cast<const float2 *>(vf + gp * CS + 16 * ks + 2 * c);
          const float2 fb = *reinterpret_cast<const float2 *>(vf + gp * CS + 16 * ks + 8 + 2 * c);
          uint32_t af[2][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 ff = (i & 1) ? fb : fa;
            af[i >> 1][(i & 1) * 2 + 0] = scale2(codes2<false>(mr[i]), ff.x, ff.y);  // dim 2r of the two slots
            af[i >> 1][(i & 1) * 2 + 1] = scale2(codes2<true>(mr[i]), ff.x, ff.y);   // dim 2r + 1
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t a[4] = {af[t][0], af[t][1], af[t][2], af[t][3]};
            mma_f16(o[2 * gp + t], a, ph[2 * ks], ph[2 * ks + 1]);
            mma_f16(o[2 * gp + t], a, pl[2 * ks], pl[2 * ks + 1]);
          }
        }
      }
    }
  }

  __device__ __forceinline__ void publish(float *dst, bool first, int lane) {
    const int r = lane >> 2, c = lane & 3;
    float ll = first ? sl_ : lsum;
    ll += __shfl_xor_sync(0xffffffffu, ll, 1);
    ll += __shfl_xor_sync(0xffffffffu, ll, 2);
    const float sv = pow2i(first ? sv_ : vexp);
#pragma unroll
    for (int g = 0; g < MT; ++g) {
      const float *og = first ? so_[g] : o[g];
      if constexpr (FP4) {  // rows r, r + 8 of m-tile g: dims 64 (g / 4) + 4 r + g % 4, and + 32
        const int d = 64 * (g >> 2) + 4 * r + (g & 3);
        if (2 * c < HC) {
          dst[(2 * c) * D + d] = og[0] * sv;
          dst[(2 * c) * D + d + 32] = og[2] * sv;
        }
        if (2 * c + 1 < HC) {
          dst[(2 * c + 1) * D + d] = og[1] * sv;
          dst[(2 * c + 1) * D + d + 32] = og[3] * sv;
        }
      } else {
        const int d = 16 * g + 2 * r;
        if (2 * c < HC) *reinterpret_cast<float2 *>(dst + (2 * c) * D + d) = make_float2(og[0] * sv, og[2] * sv);
        if (2 * c + 1 < HC)
          *reinterpret_cast<float2 *>(dst + (2 * c + 1) * D + d) = make_float2(og[1] * sv, og[3] * sv);
      }
    }
    if (r < HC && c == 0)
      *reinterpret_cast<float4 *>(dst + HC * D + r * 4) = make_float4(first ? sm_ : m, ll, 0.0f, 0.0f);
  }
};

// ---------------------------------------------------------------------------
// The kernel: work split, chunk rings, unit close and split merge.
// VARLEN: kv_len is one value per batch row (a.kv_per_batch); the scalar form
// is a separate instantiation so it carries no per-unit state.
// ---------------------------------------------------------------------------
template <class C, bool VARLEN>
__global__ void __launch_bounds__(C::THREADS, 1)
    decode_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ KvMaps maps) {
  using Core = typename std::conditional<C::BLK, BlkCore<C>,
                                         typename std::conditional<C::MMA, MmaCore<C>, SimtCore<C>>::type>::type;
  constexpr int D = C::D, HC = C::HC, NW = C::NW, R = C::R, CS = C::CS, CB = C::CB;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  // the tiles start at the first 1024-byte boundary (TMA swizzle atoms)
  uint8_t *smem = smem_raw + (C::ALIGN ? ((C::ALIGN - (smem_u32(smem_raw) & (C::ALIGN - 1))) & (C::ALIGN - 1)) : 0);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  volatile int32_t *sh = reinterpret_cast<volatile int32_t *>(smem + C::SH_OFF);  // scratch int, abort, merge flags

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < NW * R; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
    sh[1] = 0;
    sh[2] = 0;
  }
  // the TMA descriptors are launch parameters, not data of the kernel before this one:
  // fetch them while that kernel drains
  if constexpr (C::MMA) {
    if (tid == 32) {
      prefetch_tensormap(&maps.k);
      prefetch_tensormap(&maps.v);
    }
  }
  // One relaxed gpu-scope load per buffer, at the rows this CTA is likely to reach,
  // issued before the wait so that the first access to each buffer (its address
  // translation, its line into L2) can overlap the kernel before this one.  The
  // values are never used (and a gpu-scope load is served by L2, never by a stale
  // L1 line).
  if (tid < 16) {
    const int64_t U0 = static_cast<int64_t>(a.B) * a.Hkv * a.nhc;
    const int64_t u = U0 * blockIdx.x / gridDim.x;  // a unit near this CTA's first one
    const int64_t bhk = u / a.nhc, row = bhk * a.S;
    const int64_t b = bhk / a.Hkv;
    const void *p = nullptr;
    switch (tid) {
      case 0: p = a.kv_len; break;
      case 1: p = a.q + (b * a.Hq + (bhk - b * a.Hkv) * a.G) * D; break;
      case 2: p = a.out + (b * a.Hq + (bhk - b * a.Hkv) * a.G) * D; break;
      case 3: p = a.ws_cnt; break;
      case 4: p = a.ws_o + 2 * static_cast<int64_t>(blockIdx.x) * HC * D; break;
      case 5: p = a.ws_ml + 4 * static_cast<int64_t>(blockIdx.x) * HC; break;
      case 6: p = a.k + row * CB; break;
      case 7: p = a.v + row * CB; break;
      case 8: p = C::BLK ? static_cast<const uint8_t *>(a.kscl) + row * C::NGS * C::SB : (const void *)(a.ks + row); break;
      case 9: p = C::BLK ? static_cast<const uint8_t *>(a.vscl) + row * C::NGS * C::SB : (const void *)(a.vs + row); break;
      case 10: p = C::BLK ? nullptr : a.kz + row; break;
      case 11: p = C::BLK ? nullptr : a.vz + row; break;
      case 12: p = a.mask; break;
      default: break;
    }
    if (p) touch_translation(p);
  }
  // everything read below may have been written by the kernel launched before this one
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  // Every unit is cut into ceil(kv_len / 32) chunks.  With one kv_len per batch
  // row (up to kMaxRows rows) the chunks are flattened by each row's own length
  // through a prefix over the rows; above that every unit takes ceil(max
  // kv_len / 32) chunks and a row's chunks past its own kv_len move no bytes.
  const int kv = max_kv_len(a, sh, blockIdx.x == 0);
  asm volatile("griddepcontrol.launch_dependents;");
  const int nch = (kv + CS - 1) / CS;
  const int64_t U = static_cast<int64_t>(a.B) * a.Hkv * a.nhc;
  const int64_t CT0 = gridDim.x, pcta = blockIdx.x;

  if (nch == 0) {  // nothing to attend to: every row is zero
    for (int64_t u = pcta; u < U; u += CT0) {
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
  // chunk indices fit in 32 bits (the host checks U * ceil(S / 32) < 2^31)
  const bool ragged = VARLEN && a.B <= kMaxRows;
  const int UH = a.Hkv * a.nhc;  // units per batch row
  int32_t *pfx = reinterpret_cast<int32_t *>(smem + C::PFX_OFF);  // pfx[b]: first chunk of row b
  const int nch0 = ragged ? (row_kv(a, 0) + CS - 1) / CS : nch;    // row 0's chunks
  bool equal_rows = !ragged;  // every unit has nch0 chunks
  if (ragged) {  // block scan of the rows' chunk counts, rows [b0, b1) per thread
    const int per = (a.B + C::THREADS - 1) / C::THREADS;
    const int b0 = min(a.B, tid * per), b1 = min(a.B, b0 + per);
    int sum = 0;
    bool same = true;
    for (int b = b0; b < b1; ++b) {
      const int n = (row_kv(a, b) + CS - 1) / CS;
      same = same && n == nch0;
      sum += UH * n;
    }
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    int32_t *wsum = pfx + kMaxRows + 1;
    if (lane == 31) wsum[warp] = x;
    equal_rows = __syncthreads_and(same) != 0;
    int off = 0;
    for (int w = 0; w < warp; ++w) off += wsum[w];
    int run = off + x - sum;
    for (int b = b0; b < b1; ++b) {
      pfx[b] = run;
      run += UH * ((row_kv(a, b) + CS - 1) / CS);
    }
    if (tid == C::THREADS - 1) pfx[a.B] = off + x;
    __syncthreads();
  }
  // unit u's chunks: [ustart(u), ustart(u) + ulen(u)); unit_of(chunk)
  auto ulen = [&](int u) -> int {
    if (!ragged) return nch;
    const int b = u / UH;
    return (pfx[b + 1] - pfx[b]) / UH;
  };
  auto ustart = [&](int u) -> int {
    if (!ragged) return u * nch;
    const int b = u / UH;
    return pfx[b] + (u - b * UH) * ((pfx[b + 1] - pfx[b]) / UH);
  };
  auto unit_of = [&](int idx) -> int {
    if (!ragged) return idx / nch;
    int lo = 0, hi = a.B - 1;  // the last row b with pfx[b] <= idx has chunks
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pfx[mid] <= idx) lo = mid;
      else hi = mid - 1;
    }
    return lo * UH + (idx - pfx[lo]) / ((pfx[lo + 1] - pfx[lo]) / UH);
  };
  if (ragged) {  // units of empty rows own no chunks: their rows are zero
    for (int64_t u = pcta; u < U; u += CT0) {
      if (ulen(static_cast<int>(u)) != 0) continue;
      const int hc = static_cast<int>(u % a.nhc);
      const int64_t bhk = u / a.nhc;
      const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
      for (int e = tid; e < HC * D; e += C::THREADS) {
        const int hq = hk * a.G + hc * HC + e / D;
        a.out[(static_cast<int64_t>(b) * a.Hq + hq) * D + e % D] = 0;
      }
    }
  }
  const int W = ragged ? pfx[a.B] : static_cast<int>(U * nch);
  // Rows of different lengths, at most 32 of them and one CTA a unit at least: each
  // row b gets k_b CTAs a unit (one each, then one more at a time to the row with the
  // most chunks a CTA, while the grid lasts), and CTA (b, unit, j) takes the j-th of
  // k_b equal parts of its unit; used when no warp takes more rounds of chunks than
  // with the flattened cut.  A CTA then never spans two units (see active_ctas).
  // kb[b], and Kb[b] the first CTA of row b, sit in the prefix area past pfx[B].
  int32_t *kb = pfx + a.B + 1, *Kb = kb + a.B;
  bool row_aligned = false;
  if (ragged && !equal_rows && a.B <= 32 && static_cast<int64_t>(a.B) * UH <= CT0) {
    if (warp == 0) {
      const int b = lane;
      const int nb = b < a.B ? (pfx[b + 1] - pfx[b]) / UH : 0;
      int k = nb > 0 ? 1 : 0;
      int used = k;  // rows with chunks: one CTA a unit each
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) used += __shfl_xor_sync(0xffffffffu, used, o);
      int rem = static_cast<int>(CT0) / UH - used;  // a row's extra CTA a unit costs UH CTAs
      while (rem > 0) {  // one more CTA a unit to the row with the most chunks a CTA
        int best = k > 0 ? (nb + k - 1) / k : 0, who = b;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          const int ob = __shfl_xor_sync(0xffffffffu, best, o), ow = __shfl_xor_sync(0xffffffffu, who, o);
          if (ob > best || (ob == best && ow < who)) {
            best = ob;
            who = ow;
          }
        }
        if (best <= 1) break;
        if (b == who) ++k;
        --rem;
      }
      const int per = k > 0 ? (nb + k - 1) / k : 0;  // chunks of this row's CTAs, at most
      int mx = (per + NW - 1) / NW;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const int rounds_all = ((W + static_cast<int>(CT0) - 1) / static_cast<int>(CT0) + NW - 1) / NW;
      int run = k * UH;  // exclusive prefix of the rows' CTAs
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, run, o);
        if (lane >= o) run += y;
      }
      if (b < a.B) {
        kb[b] = k;
        Kb[b] = run - k * UH;
      }
      if (lane == 31) sh[4] = mx <= rounds_all ? run : 0;  // CTAs in use, 0: not used
    }
    __syncthreads();
    row_aligned = sh[4] > 0;
  }
  // CTAs with chunks to stream: the first CT of the grid (the same split for equal rows
  // whether kv_len is one scalar or one per row)
  const int CT = row_aligned ? sh[4]
                 : equal_rows ? active_ctas(static_cast<uint32_t>(U), nch0, static_cast<uint32_t>(CT0), NW)
                              : static_cast<int>(CT0);
  const int cta = static_cast<int>(pcta);
  if (cta >= CT) return;
  // Two CTAs a unit, launched as clusters of two: the pair merges its two partials
  // through distributed shared memory.  Uniform over the grid, and then no CTA of a
  // pair returns before the cluster barriers (both halves of a unit hold chunks).
  const bool pair_merge = !row_aligned && CT == 2 * U && nch0 >= 2 && cluster_size() == 2;
  int c_begin, c_end;
  if (row_aligned) {  // CTA cta: row b, unit uu of the row, part j of k_b
    int b = 0;
    while (b + 1 < a.B && Kb[b + 1] <= cta) ++b;
    const int k = kb[b], off = cta - Kb[b], uu = off / k, j = off - uu * k;
    const int n = (pfx[b + 1] - pfx[b]) / UH, us = pfx[b] + uu * n;
    c_begin = us + j * n / k;
    c_end = us + (j + 1) * n / k;
  } else {
    const uint32_t wq = static_cast<uint32_t>(W) / CT, wr = static_cast<uint32_t>(W) % CT;
    c_begin = range_start_qr(cta, wq, wr, CT);
    c_end = range_start_qr(cta + 1, wq, wr, CT);
  }
  if (c_begin >= c_end) return;  // more CTAs than chunks

  // ---- this warp's chunks: c_begin + warp + k * NW for k in [0, nk), chunk k in buffer k % R
  const int nk = c_begin + warp < c_end ? (c_end - 1 - c_begin - warp) / NW + 1 : 0;
  const int u_first = unit_of(c_begin), u_last = unit_of(c_end - 1);  // the CTA's units
  const bool deferred = u_last - u_first <= 1;
  uint8_t *tiles = smem + warp * R * C::TILE;
  uint8_t *smalls = smem + C::SMALL_OFF + warp * R * C::SMALL;
  uint64_t *bars = full + warp * R;

  // Lane 0's issue cursor: the next chunk to issue (ik), the unit it falls in, that
  // unit's chunk range, first code row (b * Hkv + hk) * S and kv_len.
  int ik = 0, iu = u_first - 1, iustart = 0, iuend = 0, ikv = kv;
  int64_t ibase = 0;
  const float *imask = a.mask;  // the unit's batch row of the mask
  const uint64_t pol = policy_evict_first();
  uint32_t outstanding = 0, outpar = 0;  // ring buffers with copies in flight, and their phases (lane 0)
  auto issue = [&](int kk) {
    const int idx = c_begin + warp + kk * NW;
    if (idx >= iuend) {  // the next unit (empty ones are skipped)
      do {
        ++iu;
        iustart = ustart(iu);
        iuend = iustart + ulen(iu);
      } while (idx >= iuend);
      const int bhk = iu / a.nhc;  // = b * Hkv + hk
      ibase = static_cast<int64_t>(bhk) * a.S;
      const int brow = bhk / a.Hkv;
      ikv = VARLEN ? row_kv(a, brow) : kv;
      if (a.mask) imask = a.mask + brow * a.mask_bstride;
    }
    const int s0 = (idx - iustart) * CS;
    const int kvu = ikv;
    const int n = max(0, min(CS, kvu - s0));
    const int n16 = (n + 15) & ~15;  // S % 16 == 0 keeps this inside the slab
    const int rb = kk % R;
    uint8_t *tile = tiles + rb * C::TILE;
    uint8_t *small = smalls + rb * C::SMALL;
    uint64_t *bar = bars + rb;
    const uint32_t code_bytes = n16 == 0 ? 0u : (C::MMA ? 2u * C::KT : static_cast<uint32_t>(n16) * 2 * CB);
    const uint32_t small_bytes = static_cast<uint32_t>(n16) * (C::BLK ? 2 * C::NGS * C::SB : 10);
    mbar_arrive_expect_tx(bar, code_bytes + small_bytes + (a.mask ? 4u * n16 : 0u));
    if (n16 > 0) {  // 0 bytes: the expect_tx above is a plain arrival
      const int64_t row = ibase + s0;
      auto copy_tiles = [&]() {
        if constexpr (C::MMA) {  // full CS-row boxes (rows past the slab read as zeros, past kv_len are masked)
#pragma unroll
          for (int st = 0; st < CB / C::ROWB; ++st) {
            tma_load_2d(tile + st * C::SUBT, &maps.k, st * C::ROWB, static_cast<int>(row), bar, pol);
            tma_load_2d(tile + C::KT + st * C::SUBT, &maps.v, st * C::ROWB, static_cast<int>(row), bar, pol);
          }
        } else {
          bulk_g2s_hint(tile, a.k + row * CB, n16 * CB, bar, pol);
          bulk_g2s_hint(tile + C::KT, a.v + row * CB, n16 * CB, bar, pol);
        }
      };
      auto copy_small = [&]() {
        if constexpr (C::BLK) {
          constexpr int RB = C::NGS * C::SB;  // scale bytes of a slot
          bulk_g2s(small + C::KS_OFF, static_cast<const uint8_t *>(a.kscl) + row * RB, n16 * RB, bar);
          bulk_g2s(small + C::VS_OFF, static_cast<const uint8_t *>(a.vscl) + row * RB, n16 * RB, bar);
        } else {
          bulk_g2s(small + C::KS_OFF, a.ks + row, n16 * 4, bar);
          bulk_g2s(small + C::VS_OFF, a.vs + row, n16 * 4, bar);
          bulk_g2s(small + C::KZ_OFF, a.kz + row, n16, bar);
          bulk_g2s(small + C::VZ_OFF, a.vz + row, n16, bar);
        }
        if (a.mask) bulk_g2s(small + C::M_OFF, imask + s0, n16 * 4, bar);
      };
      // With one buffer per warp the small copies (scales, zero points, mask) go
      // first: queued behind the 16 KB of tiles they land last and hold up the
      // buffer (measured: 0.5 us of an 18 us decode-workload launch).  With two
      // buffers per warp (D = 256) the tiles first are faster (8% on the long
      // workload).  No evict-first hint on the small copies: two chunks share a
      // 128-byte line of zero points.
      if constexpr (R == 1) {
        copy_small();
        copy_tiles();
      } else {
        copy_tiles();
        copy_small();
      }
    }
    outstanding |= 1u << rb;
    outpar = (outpar & ~(1u << rb)) | ((static_cast<uint32_t>(kk / R) & 1u) << rb);
  };
  // lane 0: keep the ring full up to R chunks past `kc` (the next to consume),
  // not past chunk index `limit`, and not after an abort
  auto top_up = [&](int kc, int limit) {
    while (ik < nk && ik < kc + R && !sh[1]) {
      if (c_begin + warp + ik * NW >= limit) break;
      issue(ik);
      ++ik;
    }
  };
  // after an abort, wait (with the full bound, whatever the main-loop bound is)
  // for this warp's copies still in flight before its ring is written or the CTA exits
  auto drain = [&]() {
    if (lane == 0 && outstanding) {
      for (int rb = 0; rb < R; ++rb)
        if (outstanding & (1u << rb)) mbar_wait_bounded(bars + rb, (outpar >> rb) & 1u);
      outstanding = 0;
    }
    __syncwarp();
  };

  // the q row of head h of unit u
  auto q_row = [&](int u, int h) {
    const int bhk = u / a.nhc, hc = u - bhk * a.nhc;
    const int b = bhk / a.Hkv, hk = bhk - b * a.Hkv;
    return a.q + (static_cast<int64_t>(b) * a.Hq + hk * a.G + hc * HC + h) * D;
  };
  // warp w: heads w, w + NW, .. of unit u onto the core's q layout, into q slot `slot`
  auto convert_q = [&](int u, int slot) {
    for (int h = warp; h < HC; h += NW)
      Core::convert_q(smem, Core::load_q_raw(q_row(u, h), lane), a.qscale, slot, h, lane);
  };

  // all threads: combine the warp records of unit u, found at tiles + rec (floats)
  // in every warp's ring, in warp order.  Write the rows, or this CTA's partial
  // when other CTAs share the unit: for the pair merge into the pair buffer of the
  // CTA that merges each half (its own, or the other CTA's through distributed
  // shared memory), else into the workspace.  A thread takes four dims of one head
  // and forms that head's factors 2^(m_w - M) and sums of l and corr itself.
  auto combine = [&](int u, int rec, bool pair) {
    const bool alone = ustart(u) >= c_begin && ustart(u) + ulen(u) <= c_end;  // no other CTA has chunks of u
    const int bhk = u / a.nhc, hc = u - bhk * a.nhc;
    const int b = bhk / a.Hkv, hk = bhk - b * a.Hkv;
    uint16_t *orow = a.out + (static_cast<int64_t>(b) * a.Hq + hk * a.G + hc * HC) * D;
    const int64_t wrec = 2 * static_cast<int64_t>(cta) + (u == u_first ? 0 : 1);
    constexpr int RS = R * C::TILE / 4;  // floats from one warp's ring of tiles to the next
    const float *base = reinterpret_cast<const float *>(smem) + rec;
    for (int e = 4 * tid; e < HC * D; e += 4 * C::THREADS) {  // four dims of one head per step
      const int h = e / D;
      float4 mlc[NW];
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        mlc[w] = *reinterpret_cast<const float4 *>(base + w * RS + HC * D + h * 4);
        M = fmaxf(M, mlc[w].x);
      }
      float Lt = 0.0f, Ct = 0.0f;
      float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = mlc[w].x == -INFINITY ? 0.0f : ex2(mlc[w].x - M);
        Lt = fmaf(f, mlc[w].y, Lt);
        Ct = fmaf(f, mlc[w].z, Ct);
        const float4 x = *reinterpret_cast<const float4 *>(base + w * RS + e);
        O.x = fmaf(f, x.x, O.x);
        O.y = fmaf(f, x.y, O.y);
        O.z = fmaf(f, x.z, O.z);
        O.w = fmaf(f, x.w, O.w);
      }
      O.x = fmaf(O.x, Core::OSCALE, -Ct);
      O.y = fmaf(O.y, Core::OSCALE, -Ct);
      O.z = fmaf(O.z, Core::OSCALE, -Ct);
      O.w = fmaf(O.w, Core::OSCALE, -Ct);
      if (alone) {
        const float inv = Lt > 0.0f ? 1.0f / Lt : 0.0f;
        uint2 pk;
        pk.x = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.x * inv))) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.y * inv))) << 16);
        pk.y = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.z * inv))) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.w * inv))) << 16);
        *reinterpret_cast<uint2 *>(orow + e) = pk;
      } else if (pair) {
        constexpr int Q2 = HC * D / 8;  // float4 items of one half
        const uint32_t me = cluster_rank(), i = static_cast<uint32_t>(e >> 2), owner = i < Q2 ? 0u : 1u;
        const uint32_t buf = smem_u32(smem) + C::PAIR_OFF;
        const uint32_t at = buf + me * (Q2 * 16) + (i - owner * Q2) * 16;
        if (owner == me) st_shared_f4(at, O);
        else st_peer_f4(peer_addr(at, owner), O);
        if (e - h * D == 0) {  // (M, L) of head h to both CTAs
          const uint32_t ml = buf + HC * D * 4 + (me * HC + h) * 8;
          st_shared_f2(ml, make_float2(M, Lt));
          st_peer_f2(peer_addr(ml, me ^ 1u), make_float2(M, Lt));
        }
      } else {
        const int d = e - h * D;
        *reinterpret_cast<float4 *>(a.ws_o + (wrec * HC + h) * D + d) = O;
        if (d == 0) *reinterpret_cast<float2 *>(a.ws_ml + (wrec * HC + h) * 2) = make_float2(M, Lt);
      }
    }
  };

  // owner records of the first (slot 0) and last (slot 1) unit when split:
  // owner o's partial is record 2 c + (u is c's first unit ? 0 : 1), c = its CTA
  int32_t *recs_s = reinterpret_cast<int32_t *>(smem + C::RECS_OFF);
  auto owners_of = [&](int u, int64_t &cf) {
    if (row_aligned) {  // the k_b CTAs of unit u, in order
      const int b = u / UH, k = kb[b];
      cf = Kb[b] + (u - b * UH) * k;
      return k;
    }
    cf = cta_of(ustart(u), W, CT);
    const int64_t cl = cta_of(ustart(u) + ulen(u) - 1, W, CT);
    return cf == cl ? 1 : (W >= CT ? static_cast<int>(cl - cf + 1) : ulen(u));  // W < CT: one chunk per CTA
  };
  // returns the owner count; `first` gets the unit's first owner CTA, which names its merge counter
  auto stage_owners = [&](int u, int slot, int &first) {
    int64_t cf;
    const int owners = owners_of(u, cf);
    first = static_cast<int>(cf);
    for (int o = tid; o < owners && owners > 1; o += C::THREADS) {
      if (row_aligned) {  // every owner's only unit: record 2 c
        recs_s[slot * kMaxCtas + o] = static_cast<int32_t>(2 * (cf + o));
        continue;
      }
      const int64_t c = W >= CT ? cf + o : cta_of(ustart(u) + o, W, CT);
      recs_s[slot * kMaxCtas + o] =
          static_cast<int32_t>(2 * c + (u == unit_of(static_cast<int>(range_start(c, W, CT))) ? 0 : 1));
    }
    return owners;
  };

  // all threads: merge the partials of the split units this CTA completes (slot 0:
  // u_first, slot 1: u_last, when `m0` / `m1`), in owner order.  A thread takes
  // four dims of one head and issues every owner's loads before it uses one.
  auto merge_units = [&](bool m0, bool m1, int own0, int own1) {
    constexpr int Q = HC * D / 4;  // float4 items per unit
    const int n0 = m0 ? Q : 0, n1 = m1 ? Q : 0;
    for (int i = tid; i < n0 + n1; i += C::THREADS) {
      const int slot = i < n0 ? 0 : 1;
      const int e = 4 * (i < n0 ? i : i - n0);
      const int u = slot ? u_last : u_first;
      const int owners = slot ? own1 : own0;
      const int32_t *recs = recs_s + slot * kMaxCtas;
      const int h = e / D, d = e - h * D;
      const int hc = u % a.nhc;
      const int64_t bhk = u / a.nhc;
      const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
      float M = -INFINITY, Lt = 0.0f;
      float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (int o0 = 0; o0 < owners; o0 += 8) {  // eight owners' loads in flight at once
        float2 ml[8];
        float4 v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (o0 + t < owners) {
            const int64_t rr = static_cast<int64_t>(recs[o0 + t]) * HC + h;
            ml[t] = __ldcg(reinterpret_cast<const float2 *>(a.ws_ml + rr * 2));
            v[t] = __ldcg(reinterpret_cast<const float4 *>(a.ws_o + rr * D + d));
          } else {
            ml[t] = make_float2(-INFINITY, 0.0f);
            v[t] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          }
        }
        float Mn = M;
#pragma unroll
        for (int t = 0; t < 8; ++t) Mn = fmaxf(Mn, ml[t].x);
        if (Mn == -INFINITY) continue;
        const float fo = M == -INFINITY ? 0.0f : ex2(M - Mn);
        Lt *= fo;
        O.x *= fo;
        O.y *= fo;
        O.z *= fo;
        O.w *= fo;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float f = ml[t].x == -INFINITY ? 0.0f : ex2(ml[t].x - Mn);
          Lt = fmaf(f, ml[t].y, Lt);
          O.x = fmaf(f, v[t].x, O.x);
          O.y = fmaf(f, v[t].y, O.y);
          O.z = fmaf(f, v[t].z, O.z);
          O.w = fmaf(f, v[t].w, O.w);
        }
        M = Mn;
      }
      const float inv = Lt > 0.0f ? 1.0f / Lt : 0.0f;
      uint2 pk;
      pk.x = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.x * inv))) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.y * inv))) << 16);
      pk.y = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.z * inv))) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(O.w * inv))) << 16);
      *reinterpret_cast<uint2 *>(a.out + (static_cast<int64_t>(b) * a.Hq + hk * a.G + hc * HC) * D + e) = pk;
    }
  };

  // ---- stage q and start the copies.  The heads of the first and the last unit
  // are spread over all warps (at most kQItems per warp); their loads are issued
  // before the warp's burst of bulk copies (loads issued behind it wait for the
  // copy engine), and converted after it.
  constexpr int kQItems = (2 * HC + NW - 1) / NW;
  const int q_items = deferred ? (u_last != u_first ? 2 : 1) * HC : 0;
  typename Core::QRaw qraw[kQItems];
#pragma unroll
  for (int j = 0; j < kQItems; ++j) {
    const int i = warp + j * NW;
    if (i < q_items) qraw[j] = Core::load_q_raw(q_row(i < HC ? u_first : u_last, i % HC), lane);
  }
  if (lane == 0) top_up(0, deferred ? c_end : min(c_end, ustart(u_first) + ulen(u_first)));
#pragma unroll
  for (int j = 0; j < kQItems; ++j) {
    const int i = warp + j * NW;
    if (i < q_items) Core::convert_q(smem, qraw[j], a.qscale, i < HC ? 0 : 1, i % HC, lane);
  }
  __syncthreads();  // q slots written

  // ---- the CTA's units in order
  Core core;
  float *wbuf = reinterpret_cast<float *>(smem + C::WBUF_OFF + warp * C::WBUF_W);  // this warp's scratch
  int k = 0;
  core.reset();
  for (int u = u_first; u <= u_last; ++u) {
    if (ragged && ulen(u) == 0) continue;  // an empty row between the CTA's first and last unit
    const int seg_end = min(c_end, ustart(u) + ulen(u));
    if (!deferred) {
      convert_q(u, 0);
      __syncthreads();  // q slot written (the previous unit's combine is complete)
      if (u != u_first && lane == 0) top_up(k, seg_end);
    } else if (u != u_first) {
      core.save();  // the warp's state so far is the first unit's
      core.reset();
    }
    core.load_q(smem, deferred && u != u_first ? 1 : 0, lane);
    const int kv_u = VARLEN ? row_kv(a, static_cast<int>(u / a.nhc / a.Hkv)) : kv;
    for (; k < nk; ++k) {
      const int idx = c_begin + warp + k * NW;
      if (idx >= seg_end) break;
      const int rb = k % R;
      // every lane of the warp takes the same branch below (it shuffles).  After an
      // abort nothing is waited for: chunks past the abort were never issued, and a
      // parity wait on a buffer still in its earlier phase would succeed at once.
      const bool ok = __all_sync(0xffffffffu, !sh[1] && wait_or_abort(bars + rb, static_cast<uint32_t>(k / R) & 1u,
                                                                      sh + 1, a.wait_ns));
      if (ok) {
        if (lane == 0) outstanding &= ~(1u << rb);
      } else if (lane == 0) {
        report(a.err, KVQ_ERR_TIMEOUT);
        sh[1] = 1;
      }
      const int s0 = (idx - ustart(u)) * CS;
      if (ok && s0 < kv_u)
        core.chunk(smem, tiles + rb * C::TILE, smalls + rb * C::SMALL, wbuf, s0, kv_u, a.mask != nullptr, lane);
      __syncwarp();  // the buffer (and the weights) are free again
      if (lane == 0) top_up(k + 1, deferred ? c_end : seg_end);
    }
    if (!deferred) {
      // the warp's ring is idle (it issues nothing past the unit): publish there
      drain();
      core.publish(reinterpret_cast<float *>(tiles), false, lane);
      __syncthreads();
      combine(u, 0, false);
      fence_proxy_async_smem();  // the rings' generic stores and loads before the next async copies into them
      __syncthreads();           // the rings are free for the next unit's copies
      core.reset();
    }
  }
  // owner records of the split units (needed by the merge only), staged while
  // the slower warps of the CTA still finish their chunks
  int cf0 = 0, cf1 = 0;
  const int own0 = pair_merge ? 2 : stage_owners(u_first, 0, cf0);
  const int own1 = !pair_merge && u_last != u_first ? stage_owners(u_last, 1, cf1) : 1;
  if (deferred) {
    drain();
    // every warp is past its chunks and its ring is idle: records of the first unit at 0, the last at PUB
    float *rw = reinterpret_cast<float *>(tiles);
    if (u_last != u_first) {
      core.publish(rw, true, lane);
      core.publish(rw + C::PUB / 4, false, lane);
    } else {
      core.publish(rw, false, lane);
    }
    __syncthreads();
    combine(u_first, 0, pair_merge);
    if (u_last != u_first) combine(u_last, C::PUB / 4, false);
  }
  if (pair_merge) {
    // Both CTAs' partials of this CTA's half are in its pair buffer once the cluster
    // barrier (release / acquire) is passed; nothing touches this CTA's shared memory
    // after it.  Merge them in rank (= owner) order, as the owner merge below would.
    cluster_sync();
    constexpr int Q2 = HC * D / 8;  // float4 items of one half
    const int me = static_cast<int>(cluster_rank());
    const float *pb = reinterpret_cast<const float *>(smem + C::PAIR_OFF);
    const float2 *pml = reinterpret_cast<const float2 *>(smem + C::PAIR_OFF + HC * D * 4);
    const int bhk = u_first / a.nhc, hc = u_first - bhk * a.nhc;
    const int b = bhk / a.Hkv, hk = bhk - b * a.Hkv;
    uint16_t *orow = a.out + (static_cast<int64_t>(b) * a.Hq + hk * a.G + hc * HC) * D;
    for (int j = tid; j < Q2; j += C::THREADS) {
      const int e = 4 * (me * Q2 + j), h = e / D;
      const float2 ml0 = pml[h], ml1 = pml[HC + h];
      const float4 v0 = *reinterpret_cast<const float4 *>(pb + 4 * j);
      const float4 v1 = *reinterpret_cast<const float4 *>(pb + 4 * (Q2 + j));
      const float M = fmaxf(ml0.x, ml1.x);
      const float f0 = ml0.x == -INFINITY ? 0.0f : ex2(ml0.x - M), f1 = ml1.x == -INFINITY ? 0.0f : ex2(ml1.x - M);
      const float Lt = fmaf(f1, ml1.y, fmaf(f0, ml0.y, 0.0f));
      const float inv = Lt > 0.0f ? 1.0f / Lt : 0.0f;
      const float o0 = fmaf(f1, v1.x, fmaf(f0, v0.x, 0.0f)), o1 = fmaf(f1, v1.y, fmaf(f0, v0.y, 0.0f));
      const float o2 = fmaf(f1, v1.z, fmaf(f0, v0.z, 0.0f)), o3 = fmaf(f1, v1.w, fmaf(f0, v0.w, 0.0f));
      uint2 pk;
      pk.x = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o0 * inv))) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o1 * inv))) << 16);
      pk.y = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o2 * inv))) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o3 * inv))) << 16);
      *reinterpret_cast<uint2 *>(orow + e) = pk;
    }
    return;
  }
  __syncthreads();  // every partial and owner record is written; the scratch is free for the merge

  // Only the first and the last unit of a contiguous range can be shared with
  // other CTAs.  Count this CTA's partials of those (threads 0 and 1); the owner
  // whose count completes a unit merges it, in owner order.  A split unit's
  // counter is the one of its first owner CTA: only the last unit of a CTA's
  // range can run past it, so no two split units share a first owner, and the
  // counters sit at the same place for every problem shape.
  if (tid < 2) {
    const int owners = tid == 0 ? own0 : own1;
    const int cf = tid == 0 ? cf0 : cf1;
    bool mine = false;
    if (owners > 1 && (tid == 0 || u_last != u_first)) {
      if (count_acq_rel(a.ws_cnt + cf) == owners - 1) {
        a.ws_cnt[cf] = 0;  // every owner has counted: ready for the next call
        mine = true;
      }
    }
    sh[2 + tid] = mine ? 1 : 0;
  }
  __syncthreads();
  if (sh[2] || sh[3]) merge_units(sh[2] != 0, sh[3] != 0, own0, own1);
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
// q heads per unit: the tensor-core path takes up to 8 (one MMA row per head),
// the CUDA-core path up to 4 (registers)
int head_chunk_mma(int G) {
  for (int h = G < 8 ? G : 8; h > 1; --h)
    if (G % h == 0) return h;
  return 1;
}
int head_chunk_simt(int G) { return G % 4 == 0 ? 4 : (G % 3 == 0 ? 3 : (G % 2 == 0 ? 2 : 1)); }

// Warps per CTA and ring depth.  Tensor-core path: registers hold q fragments
// (D/8 per lane), O^T accumulators (D/4) and the first unit's saved O^T (D/4).
// A warp's chunk is a chain of dependent steps, so what sets the pace is warps
// per SM sub-partition: eight warps (two per sub-partition) with one buffer each
// beat six with two (two sub-partitions then run one warp alone) at D <= 128.
// CUDA-core path: q (8 words per head), accumulators (2 x D/32 per head) and
// q.k partials (D/16 per head).  The ring takes what shared memory is left.
template <int D, int HC, bool MMA, bool Q4, int MODE = 0>
struct Tune {
  // tensor-core path: 64-slot chunks up to D = 128 (two chunks' worth of independent
  // MMAs and scores per warp step, fixed costs per chunk halved), 32 for D = 256
  static constexpr int CS = MMA && D <= 128 ? 64 : 32;
  static constexpr int NW = MMA ? (D == 256 ? (MODE ? 4 : 6) : 8)  // block caches at D = 256: two buffers a warp
                                : (D == 256 ? 8 : (D == 128 ? (HC <= 2 ? 16 : 12) : 16));
  static constexpr int CB = Q4 || MODE == KVQ_MODE_MXFP4 ? D / 2 : D;
  static constexpr int SBB = MODE == KVQ_MODE_FP8_E4M3 || MODE == KVQ_MODE_FP8_E5M2 || MODE == KVQ_MODE_INT8_SYM ? 4 : 1;
  static constexpr int PER_BUF = 2 * CS * CB + (MODE ? 2 * CS * (D / 32) * SBB + 4 * CS : 14 * CS);
  static constexpr int WB = MODE ? CS * 16 + 2 * (D / 32) * CS * 4 : CS * 20;
  static constexpr int FIXED = (MMA ? 1024 + NW * WB : NW * HC * 128) + NW * 4 * 8 + 64 + 4 * HC * D +
                               16 * HC + 8 * kMaxCtas + 4 * (kMaxRows + 33) + 16 + 4 * HC * D + 16 * HC;
  static constexpr int RMAX = (232448 - FIXED) / (NW * PER_BUF);
  static constexpr int R = RMAX > 4 ? 4 : RMAX;
  static_assert(R >= 1, "ring depth");
};

struct WsLayout {
  size_t cnt, ml, o, total;
};

// The merge counters first, at offset 0 for every shape (one per CTA, kMaxCtas
// of them), then two partial records per CTA (its first and last unit, the only
// ones it can share).  Records of any shape never land on the counters, so a
// workspace can serve calls of different shapes one after another.
WsLayout ws_layout(int D, int HC, int ctas) {
  WsLayout w;
  const size_t recs = 2 * static_cast<size_t>(ctas);
  w.cnt = 0;
  w.ml = kMaxCtas * 4;
  w.o = w.ml + (recs * HC * 2 * 4 + 255) / 256 * 256;
  w.total = w.o + (recs * HC * D * 4 + 255) / 256 * 256;
  return w;
}

// ---- TMA descriptors (tensor-core path): the encoder comes from the driver at
// run time, so the library links only the CUDA runtime
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [rows, D] int8 codes, boxes of box_rows rows x min(D, 128) bytes, swizzled
int make_code_map(CUtensorMap *map, const void *base, int D, int64_t rows, int box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return KVQ_ECUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(D < 128 ? D : 128), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, D < 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? KVQ_OK : KVQ_ECUDA;
}

template <class C, bool VARLEN>
struct KernelTag {};  // names one decode_kernel instantiation for ensure_smem

// Whether a grid of `ctas` CTAs of `kernel` (one per SM) runs in one wave as
// clusters of two: the SMs of a cluster come from one GPC, so an odd GPC could
// leave a pair unplaced.  Queried once per kernel and device.
template <class Tag, class Kernel>
bool pairs_fit(Kernel kernel, int threads, int smem, int ctas) {
  static std::atomic<uint64_t> known{0}, fit{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return false;
  const uint64_t bit = 1ull << dev;
  if (known.load(std::memory_order_acquire) & bit) return (fit.load(std::memory_order_acquire) & bit) != 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  const bool ok = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess && 2 * n >= ctas;
  if (!ok) (void)cudaGetLastError();
  if (ok) fit.fetch_or(bit, std::memory_order_acq_rel);
  known.fetch_or(bit, std::memory_order_acq_rel);
  return ok;
}

template <int D, int HC, bool MMA, bool Q4, int MODE = 0>
int launch_decode(const DecodeArgs &a, const KvMaps &maps, int ctas, cudaStream_t stream) {
  using T = Tune<D, HC, MMA, Q4, MODE>;
  using C = Cfg<D, HC, T::NW, T::R, MMA, Q4, T::CS, MODE>;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t dc = {};
  dc.gridDim = dim3(static_cast<unsigned>(ctas));
  dc.blockDim = dim3(C::THREADS);
  dc.dynamicSmemBytes = C::SMEM;
  dc.stream = stream;
  dc.attrs = attr;
  dc.numAttrs = 1;
  // two CTAs a unit (floor(ctas / units) = 2) may stream as cluster pairs that merge
  // through distributed shared memory
  const int64_t units = static_cast<int64_t>(a.B) * a.Hkv * a.nhc;
  const bool pairs = ctas % 2 == 0 && units > 0 && ctas / units == 2;
  cudaError_t e;
  if (a.kv_per_batch) {
    if (const int st = ensure_smem<KernelTag<C, true>>(decode_kernel<C, true>, C::SMEM)) return st;
    if (pairs && pairs_fit<KernelTag<C, true>>(decode_kernel<C, true>, C::THREADS, C::SMEM, ctas)) dc.numAttrs = 2;
    e = cudaLaunchKernelEx(&dc, decode_kernel<C, true>, a, maps);
  } else {
    if (const int st = ensure_smem<KernelTag<C, false>>(decode_kernel<C, false>, C::SMEM)) return st;
    if (pairs && pairs_fit<KernelTag<C, false>>(decode_kernel<C, false>, C::THREADS, C::SMEM, ctas)) dc.numAttrs = 2;
    e = cudaLaunchKernelEx(&dc, decode_kernel<C, false>, a, maps);
  }
  if (e != cudaSuccess) return KVQ_ECUDA;
  return launch_status();
}

template <int D>
int dispatch_mma(const DecodeArgs &a, const KvMaps &maps, int hc, int ctas, cudaStream_t s) {
  switch (hc) {
    case 1: return launch_decode<D, 1, true, false>(a, maps, ctas, s);
    case 2: return launch_decode<D, 2, true, false>(a, maps, ctas, s);
    case 3: return launch_decode<D, 3, true, false>(a, maps, ctas, s);
    case 4: return launch_decode<D, 4, true, false>(a, maps, ctas, s);
    case 5: return launch_decode<D, 5, true, false>(a, maps, ctas, s);
    case 6: return launch_decode<D, 6, true, false>(a, maps, ctas, s);
    case 7: return launch_decode<D, 7, true, false>(a, maps, ctas, s);
    default: return launch_decode<D, 8, true, false>(a, maps, ctas, s);
  }
}

// block caches of byte codes (kvq_write modes 1, 2, 4, 5, 6)
template <int D, int MODE>
int dispatch_blk(const DecodeArgs &a, const KvMaps &maps, int hc, int ctas, cudaStream_t s) {
  switch (hc) {
    case 1: return launch_decode<D, 1, true, false, MODE>(a, maps, ctas, s);
    case 2: return launch_decode<D, 2, true, false, MODE>(a, maps, ctas, s);
    case 3: return launch_decode<D, 3, true, false, MODE>(a, maps, ctas, s);
    case 4: return launch_decode<D, 4, true, false, MODE>(a, maps, ctas, s);
    case 5: return launch_decode<D, 5, true, false, MODE>(a, maps, ctas, s);
    case 6: return launch_decode<D, 6, true, false, MODE>(a, maps, ctas, s);
    case 7: return launch_decode<D, 7, true, false, MODE>(a, maps, ctas, s);
    default: return launch_decode<D, 8, true, false, MODE>(a, maps, ctas, s);
  }
}
template <int MODE>
int dispatch_blk_mode(const DecodeArgs &a, const KvMaps &maps, int D, int hc, int ctas, cudaStream_t s) {
  switch (D) {
    case 64:
      if constexpr (MODE == KVQ_MODE_MXFP4) return KVQ_EUNSUPPORTED;  // E2M1 codes from D = 128
      else return dispatch_blk<64, MODE>(a, maps, hc, ctas, s);
    case 128: return dispatch_blk<128, MODE>(a, maps, hc, ctas, s);
    default: return dispatch_blk<256, MODE>(a, maps, hc, ctas, s);
  }
}

// TQ4 cache on the tensor cores (D = 128, 256)
template <int D>
int dispatch_q4mma(const DecodeArgs &a, const KvMaps &maps, int hc, int ctas, cudaStream_t s) {
  switch (hc) {
    case 1: return launch_decode<D, 1, true, true>(a, maps, ctas, s);
    case 2: return launch_decode<D, 2, true, true>(a, maps, ctas, s);
    case 3: return launch_decode<D, 3, true, true>(a, maps, ctas, s);
    case 4: return launch_decode<D, 4, true, true>(a, maps, ctas, s);
    case 5: return launch_decode<D, 5, true, true>(a, maps, ctas, s);
    case 6: return launch_decode<D, 6, true, true>(a, maps, ctas, s);
    case 7: return launch_decode<D, 7, true, true>(a, maps, ctas, s);
    default: return launch_decode<D, 8, true, true>(a, maps, ctas, s);
  }
}

template <int D>
int dispatch_q4(const DecodeArgs &a, const KvMaps &maps, int hc, int ctas, cudaStream_t s) {
  switch (hc) {
    case 1: return launch_decode<D, 1, false, true>(a, maps, ctas, s);
    case 2: return launch_decode<D, 2, false, true>(a, maps, ctas, s);
    case 3: return launch_decode<D, 3, false, true>(a, maps, ctas, s);
    default: return launch_decode<D, 4, false, true>(a, maps, ctas, s);
  }
}

// Workspace bytes of either path (the size query does not know which one the
// caller will use, so it returns the larger).
size_t ws_bytes(int G, int D, int ctas) {
  const size_t m = ws_layout(D, head_chunk_mma(G), ctas).total, s = ws_layout(D, head_chunk_simt(G), ctas).total;
  return m > s ? m : s;
}

}  // namespace
}  // namespace kvq
