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
// Design.  One CTA holds 128 query rows of one kv head (HPT q heads x RPH
// positions with GQA, so every K/V tile is dequantized once for all of them)
// and runs four roles, connected by mbarriers:
//   - softmax warpgroup (warps 0-3): thread t owns query row t, i.e. TMEM lane t;
//   - K and V converter warpgroups (warps 4-7, 8-11): turn the int8 codes of
//     128-slot K and V tiles into fp16 in the 128-byte-swizzled shared-memory
//     layout the tensor core reads; each issues the loads of its next tile as
//     soon as it has stored the current one, so the memory latency overlaps
//     the wait for the tensor core to release the buffer;
//   - MMA warp (warp 12): one thread issues every tcgen05.mma.
// Tensor-core work per tile j:  S_j = Q K_j^T (M 128, N 128) into one of two
// TMEM buffers; the softmax writes P_j back over the columns of S_j it came
// from, and O += P_j V_j takes P from TMEM (A operand in tensor memory) and V
// from shared memory.  Issue order QK_0, QK_1, PV_0, QK_2, PV_1, ...: the
// softmax of tile j overlaps QK_{j+1}; the converters rebuild K_{j+1} as soon
// as QK_j has read K_j and V_j as soon as PV_{j-1} has read V_{j-1}, so one
// shared-memory buffer of each suffices.
//
// Numerics: fp16 operands, fp32 accumulation.
//   - K/V codes become the exact fp16 values (c - zp), |c - zp| <= 255, through
//     a byte permute into the mantissa of 1024 and one packed subtract.
//   - Q is multiplied per row by the power of two that brings max|q| into
//     [2^14, 2^15), then rounded to fp16: exact for every element above 2^-14
//     in that scale (bf16 carries 8 significant bits, fp16 11); the power of
//     two is folded back into the row's score scale.
//   - k_scale multiplies the fp32 scores; v_scale is folded into
//     P = p * v_scale * 2^-E, where E is a per-CTA exponent kept between 2 and
//     10 binades above the tile's largest v_scale, so P < 2^7 and P is rounded
//     to fp16 once (relative error <= 2^-11).  When E moves, O is rescaled in
//     TMEM by the exact power of two.
//   - Online softmax in the log2 domain; the running max is raised only when
//     a score exceeds it by more than 8 (O and l then hold values up to 2^8
//     larger, harmless in fp32).
// Per-tile causal bound: with mask_is_causal the tile loop stops at
// min(kv_len, kv_len - Lq + (last row of the CTA) + 1); later tiles would be
// fully masked, so the output is bit-identical with or without the skip.
//
// Every wait is bounded.  A wait that gives up raises a CTA-wide abort flag;
// every role leaves its loop at its next wait, the MMA thread waits (bounded)
// for what it issued, TMEM is freed and KVQ_ERR_TIMEOUT is reported.
#pragma once

#include <atomic>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_common.cuh"

namespace kvq {
namespace tc {

constexpr int kRows = 128;  // query rows per CTA (tcgen05 M)
constexpr int kTile = 128;  // slots per K/V tile (N of Q K^T, K of P V)
constexpr int kSoftmaxThreads = 128;
constexpr int kConvThreads = 128;  // per converter warpgroup (one for K, one for V)
constexpr int kThreads = kSoftmaxThreads + 2 * kConvThreads + 32;
constexpr int kMmaWarp = 12;
constexpr int kScaleBufs = 3;  // k_scale / v_scale tile buffers
constexpr int kMaxSplit = 4;  // CTAs of a KV-split cluster
// registers per thread: 13 warps, one SM sub-partition holds four of them
constexpr int kRegsLaunch = 128;

struct PrefillArgs {
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
  int32_t *err;
  int64_t S;
  int B, Hq, Hkv, G, Lq, nhc;  // nhc: head chunks of HPT heads per kv head
  int is_causal, mask_is_causal;
  float qscale;      // sm_scale * log2(e)
  uint64_t wait_ns;  // bound on each main-loop wait
  int ns;            // KV splits: a cluster of ns CTAs shares one row block, each a share of its KV tiles
  // block caches (kvq_write modes 1-6): codes in k / v, per-32 scales as float
  // (ks / vs) or E8M0 bytes (ks8 / vs8); kz / vz unused
  const uint8_t *ks8, *vs8;
};

// mbarriers.  A parity wait is only meaningful when the barrier has already
// completed every phase before the awaited one and not the one after it; each
// wait below is placed where both hold (the epilogue has its own barrier for
// that reason: O may still be a PV or two behind the softmax).
enum : int {
  kBarQ = 0,   // Q tile written (softmax warpgroup, 128 arrivals)
  kBarKFull,   // K tile written (K converters, 128 arrivals)
  kBarKEmpty,  // QK done with the K tile (commit)
  kBarVFull,   // V tile written (V converters, 128 arrivals)
  kBarVEmpty,  // PV done with the V tile (commit)
  kBarSFull0,  // S buffer 0 / 1 computed (commit)
  kBarSFull1,
  kBarPFull0,  // P in S buffer 0 / 1 written (softmax, 128 arrivals)
  kBarPFull1,
  kBarODone,   // a PV finished (commit)
  kBarOFinal,  // the last PV finished (commit, once)
  kBarDrain,   // abort path: everything issued has finished (commit)
  kBarMask0,   // mask rows of a tile staged in buffer 0 / 1 / 2 (bulk copies, RPH arrivals)
  kBarMask1,
  kBarMask2,
  kNumBars
};

// MODE: the kvq_write mode of the cache (0: int8 affine; 1-6: per-32 block
// formats, whose converters use the factor region FAC_OFF).
template <int D_, int HPT_, bool MASK_, int MODE_ = 0>
struct Cfg {
  static constexpr int D = D_, HPT = HPT_, RPH = kRows / HPT;
  static constexpr bool MASK = MASK_;
  static constexpr int MODE = MODE_;
  static constexpr int NG = D / 32;  // per-32 scale groups of a slot row (block modes)
  static constexpr int PPR = D / 16;                    // 16-code parts per slot row
  static constexpr int NSG = kConvThreads / PPR;        // groups of consecutive slots
  static constexpr int NCH = kTile / NSG;               // slots per group = chunks per converter thread
  static constexpr int Q_OFF = 0;                       // D/64 x [128 rows  x 128 B]
  static constexpr int K_OFF = Q_OFF + kRows * 2 * D;   // D/64 x [128 slots x 128 B]
  static constexpr int V_OFF = K_OFF + kTile * 2 * D;   // D/64 x [128 slots x 128 B]
  static constexpr int KS_OFF = V_OFF + kTile * 2 * D;  // float [kScaleBufs][128]
  static constexpr int VS_OFF = KS_OFF + kScaleBufs * kTile * 4;
  static constexpr int VMX_OFF = VS_OFF + kScaleBufs * kTile * 4;  // float [kScaleBufs][4]
  // block modes: float [K, V][2 tiles][kTile slots][NG] group factors scale_g * 2^-E_slot
  static constexpr int FAC_OFF = VMX_OFF + kScaleBufs * 16;
  static constexpr int FAC_BYTES = MODE == 0 ? 0 : 2 * 2 * kTile * NG * 4;
  static constexpr int BAR_OFF = FAC_OFF + FAC_BYTES;
  static constexpr int MISC_OFF = BAR_OFF + kNumBars * 8;  // TMEM base, abort flag, qs, 4 x max|q|, O valid
  static constexpr int STAT_OFF = (MISC_OFF + 32 + 15) / 16 * 16;  // KV split: float4 [kRows] (m, E, l, -) per row
  // additive mask: with one position per 32 rows of the CTA (4 heads a row block) the
  // mask rows of a tile are staged by bulk copies into a ring of three buffers of
  // [RPH][kTile] floats (rows 16 bytes apart more than their length, which spreads a
  // warp's float4 reads over all banks); else read from global memory
  static constexpr int MROW = kTile * 4 + 16;
  static constexpr int MSK_OFF = STAT_OFF + kRows * 16;
  static constexpr int SMEM_BASE = MSK_OFF + 1024;  // + slack to align the base to 1024
  static constexpr bool MSTAGE = MASK && RPH <= 32 && SMEM_BASE + 3 * RPH * MROW <= 232448;
  static constexpr int SMEM = SMEM_BASE + (MSTAGE ? 3 * RPH * MROW : 0);
  static_assert(STAT_OFF % 16 == 0 && MSK_OFF % 16 == 0 && MROW % 16 == 0, "float4 stores and bulk copies");
  // KV split: the rows' pre-scaled fp32 partial O, [kRows][D], over the Q/K/V tiles
  static constexpr int CONTRIB_OFF = Q_OFF;
  static_assert(kRows * D * 4 <= BAR_OFF, "the partial O fits over the tiles");
  static constexpr int S_COL0 = 0, S_COL1 = kTile, O_COL = 2 * kTile;
  static constexpr int TMEM_COLS = 512;
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(NCH * NSG == kTile && NSG * PPR == kConvThreads && NCH % 4 == 0, "converter mapping");
};

// ---- descriptors -------------------------------------------------------------
// Shared-memory matrix descriptor (tcgen05): start address >> 4 in bits 0-13,
// leading byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45,
// descriptor version 1 in bits 46-47, swizzle mode in 61-63 (2 = 128-byte).
KVQ_DEVINL uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: f32 accumulator (bits 4-5 = 1), f16 A and
// B (bits 7-9, 10-12 = 0), A/B major in bits 15/16 (0 = K-major, 1 = MN-major),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int b_mn_major) {
  return (1u << 4) | (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D (TMEM) (+)= A (shared) x B (shared)
KVQ_DEVINL void mma_ss(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D (TMEM) (+)= A (TMEM) x B (shared)
KVQ_DEVINL void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
KVQ_DEVINL void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
KVQ_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
KVQ_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
KVQ_DEVINL void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's TMEM lane (completes at tmem_ld_wait).
KVQ_DEVINL void tmem_ld32(uint32_t taddr, uint32_t (&u)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]), "=r"(u[8]),
        "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]),
        "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
        "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(taddr));
}
KVQ_DEVINL void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
KVQ_DEVINL void tmem_st32(uint32_t taddr, const uint32_t (&u)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]), "r"(u[9]),
      "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15]), "r"(u[16]), "r"(u[17]), "r"(u[18]),
      "r"(u[19]), "r"(u[20]), "r"(u[21]), "r"(u[22]), "r"(u[23]), "r"(u[24]), "r"(u[25]), "r"(u[26]), "r"(u[27]),
      "r"(u[28]), "r"(u[29]), "r"(u[30]), "r"(u[31])
      : "memory");
}
KVQ_DEVINL void tmem_st16(uint32_t taddr, const uint32_t *u) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]), "r"(u[9]),
      "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
      : "memory");
}
KVQ_DEVINL void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// One probe of a phase, suspending up to 20 us while it is incomplete.
KVQ_DEVINL bool try_wait_short(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
// Bounded wait (limit_ns, the launch's main-loop bound) that also gives up once
// another role has raised the abort flag.  A bound below kNoProbeBelowNs gives
// up at once without probing.
KVQ_DEVINL bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint64_t limit_ns) {
  if (limit_ns < kNoProbeBelowNs) {
    *abort_flag = 1;
    return false;
  }
  if (try_wait_short(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (try_wait_short(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      return false;
    }
  }
}

KVQ_DEVINL float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^e for e in [-126, 127]
KVQ_DEVINL float exp2i(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }
// ceil(log2 v) for v > 0 (v below the normal range counts as 2^-126)
KVQ_DEVINL int ceil_log2(float v) {
  const uint32_t bits = __float_as_uint(v);
  const int e = static_cast<int>(bits >> 23) - 127;
  if (e < -126) return -126;
  return e + ((bits & 0x7FFFFFu) != 0u ? 1 : 0);
}

// Byte offset of the 16-byte chunk `c` (8 halves) of row `r` inside a 128-byte
// swizzled region (rows of 128 B, chunks XOR-permuted by r % 8).
KVQ_DEVINL uint32_t swz(int r, int c) { return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4)); }

// 16 int8 codes -> 16 fp16 values (c - zp), exact: (c + 128) goes into the low
// mantissa bits of 1024 (fp16 0x6400 | byte is 1024 + byte exactly), and one
// packed subtract of (1152 + zp) leaves c - zp.
KVQ_DEVINL void codes16_to_f16(const uint4 &w, uint32_t zc2, uint4 &lo, uint4 &hi) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[8];
  const __half2 z = *reinterpret_cast<const __half2 *>(&zc2);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t u = in[i] ^ 0x80808080u;
    const uint32_t h0 = __byte_perm(u, 0x64646464u, 0x4140);
    const uint32_t h1 = __byte_perm(u, 0x64646464u, 0x4342);
    const __half2 r0 = __hsub2(*reinterpret_cast<const __half2 *>(&h0), z);
    const __half2 r1 = __hsub2(*reinterpret_cast<const __half2 *>(&h1), z);
    o[2 * i] = *reinterpret_cast<const uint32_t *>(&r0);
    o[2 * i + 1] = *reinterpret_cast<const uint32_t *>(&r1);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}
// Global loads that stay in program order with the mbarrier operations (the
// compiler may not hoist them above a wait or an arrive, which would keep two
// tiles of codes in registers).
KVQ_DEVINL uint4 ld_codes(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
KVQ_DEVINL uint32_t ld_u32(const void *p) {
  uint32_t r;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
KVQ_DEVINL float ld_f32(const float *p) {
  float r;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r) : "l"(p));
  return r;
}
// fp16 pair of (1152 + zp): bits 0x6400 | (128 + zp)
KVQ_DEVINL uint32_t zp_const2(int zp) {
  const uint32_t h = 0x6400u | static_cast<uint32_t>((zp + 128) & 0xFF);
  return h | (h << 16);
}

// State shared by the roles (each role runs in its own function, so that the
// register allocation of one does not constrain the others).
struct Ctx {
  uint8_t *smem;  // 1024-byte aligned dynamic shared memory
  uint32_t tmem;  // TMEM base address
  int kv, loop_end;
  int jb, ntiles;  // this CTA's KV tiles: jb .. jb + ntiles - 1 (loops count j from 0)
  int vis_end;     // with is_causal, no row of the CTA sees a slot at or past this
};

// softmax warpgroup: query row t = threadIdx.x, TMEM lane t
template <class C>
__device__ __noinline__ void role_softmax(const PrefillArgs &a, const Ctx x) {
  constexpr int D = C::D, HPT = C::HPT, RPH = C::RPH;
  uint8_t *smem = x.smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF + 4);
  float *qs_s = reinterpret_cast<float *>(smem + C::MISC_OFF + 8);          // sm_scale * log2e * 2^sh
  uint32_t *qmax_s = reinterpret_cast<uint32_t *>(smem + C::MISC_OFF + 12);  // per softmax warp
  const float *ks_s = reinterpret_cast<const float *>(smem + C::KS_OFF);
  const float *vs_s = reinterpret_cast<const float *>(smem + C::VS_OFF);
  const float *vmx_s = reinterpret_cast<const float *>(smem + C::VMX_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int xrow = blockIdx.x / a.ns, hkc = blockIdx.y, b = blockIdx.z;  // a.ns CTAs share a row block
  const int hk = hkc / a.nhc, hc = hkc - hk * a.nhc;
  const uint32_t tmem = x.tmem;
  const int kv = x.kv, loop_end = x.loop_end, ntiles = x.ntiles, jb = x.jb;
  // ======================= softmax warpgroup: query row t
  const int t = tid;
  const int g = t / RPH;
  const int pos = xrow * RPH + (t - g * RPH);
  const int hq = hk * a.G + hc * HPT + g;
  const bool row_ok = pos < a.Lq;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  // last visible slot of this row (the loop bound and the causal rule), -1 if none
  int vis_last = loop_end - 1;
  if (a.is_causal) vis_last = min(vis_last, kv - a.Lq + pos);
  if (!row_ok) vis_last = -1;

  // Q -> fp16 x 2^-sh, swizzled into shared memory; sh is one power of two for
  // the CTA, chosen so that the largest |q| lands in [2^14, 2^15)
  const uint4 *qp =
      reinterpret_cast<const uint4 *>(a.q + ((static_cast<int64_t>(b) * a.Hq + hq) * a.Lq + (row_ok ? pos : 0)) * D);
  // Staged mask (C::MSTAGE): thread t < RPH (the first head of each position) copies
  // its position's mask row of tile j into buffer j % 3.  Tile j + 1's copy is issued
  // once S_j is computed: QK_j needed PV_{j-2}, so every row is past tile j - 2, the
  // last user of that buffer.
  uint8_t *msk = smem + C::MSK_OFF;
  const bool missue = C::MSTAGE && t < RPH;
  uint32_t mpend = 0, mpar = 0;  // buffers with a copy in flight and their phases (issuing threads)
  auto issue_mask = [&](int j) {
    const int mb = j % 3;
    const int t0 = (jb + j) * kTile;
    const int n = row_ok ? max(0, min(kTile, loop_end - t0)) : 0;
    const uint32_t bytes = static_cast<uint32_t>((n + 3) & ~3) * 4;  // loop_end <= S, S % 4 == 0
    mbar_arrive_expect_tx(&bars[kBarMask0 + mb], bytes);
    if (bytes)
      bulk_g2s(msk + (mb * RPH + t) * C::MROW, a.mask + b * a.mask_bstride + static_cast<int64_t>(pos) * a.S + t0,
               bytes, &bars[kBarMask0 + mb]);
    mpend |= 1u << mb;
    mpar = (mpar & ~(1u << mb)) | (static_cast<uint32_t>((j / 3) & 1) << mb);
  };
  if (missue && ntiles > 0) issue_mask(0);
  // Unstaged mask: the row's mask for the first tile into L1 while Q is staged (each
  // tile's is fetched one tile ahead below), so the score pass reads it at L1 latency.
  auto prefetch_mask = [&](int j) {
    if constexpr (C::MASK && !C::MSTAGE) {
      const int t0 = (jb + j) * kTile;
      if (row_ok)
#pragma unroll
        for (int i = 0; i < kTile / 32; ++i)
          if (t0 + 32 * i < loop_end)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(a.mask + b * a.mask_bstride +
                                                          static_cast<int64_t>(pos) * a.S + t0 + 32 * i));
    }
  };
  if (ntiles > 0) prefetch_mask(0);
  // Q row up to D = 128: all its loads in flight at once (one round trip) and kept in
  // registers for the conversion; at D = 256 in groups of four, read twice
  constexpr int QC = D / 8;
  constexpr bool QREG = QC <= 16;
  uint4 qw[QREG ? QC : 1];
  {
    uint32_t mx = 0;
    if (row_ok) {
      if constexpr (QREG) {
#pragma unroll
        for (int i = 0; i < QC; ++i) qw[i] = __ldg(qp + i);
#pragma unroll
        for (int i = 0; i < QC; ++i)
          mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(qw[i].x & 0x7FFF7FFFu, qw[i].y & 0x7FFF7FFFu),
                                     __vmaxu2(qw[i].z & 0x7FFF7FFFu, qw[i].w & 0x7FFF7FFFu)));
      } else {
#pragma unroll 4
        for (int c = 0; c < QC; ++c) {
          const uint4 w = __ldg(qp + c);
          mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                                     __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu)));
        }
      }
    }
    const uint32_t mw = __reduce_max_sync(0xffffffffu, max(mx & 0xFFFFu, mx >> 16));
    if (lane == 0) qmax_s[warp] = mw;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
  const uint32_t mb = max(max(qmax_s[0], qmax_s[1]), max(qmax_s[2], qmax_s[3]));  // largest |q| (bf16 bits)
  int sh = 0;
  if (mb != 0u) sh = max(-100, min(100, static_cast<int>((mb >> 7) & 0xFFu) - 127 - 14));
  const float qs = a.qscale * exp2i(sh);
  {
    const float f = exp2i(-sh);
#pragma unroll QREG ? 16 : 2
    for (int c = 0; c < D / 8; ++c) {
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if constexpr (QREG) {
        if (row_ok) w = qw[c];
      } else {
        if (row_ok) w = __ldg(qp + c);
      }
      const uint32_t in[4] = {w.x, w.y, w.z, w.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 h = __floats2half2_rn(bf16lo(in[i]) * f, bf16hi(in[i]) * f);
        o[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
      *reinterpret_cast<uint4 *>(smem + C::Q_OFF + (c >> 3) * (kRows * 128) + swz(t, c & 7)) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (t == 0) *qs_s = qs;
  proxy_fence();
  mbar_arrive(&bars[kBarQ]);

  // Scores in the log2 domain: x = S_raw * kq (kq = k_scale * qs per slot,
  // prepared by the converters) [+ mask * log2e].  With the running max m and
  // the P exponent E, p' = 2^(x - m - E) = p * 2^-E; P = p' * v_scale, and
  // l and O are both kept in units of 2^-E, so out = O / l.
  float m = -INFINITY, l = 0.0f;
  int E = 0;
  bool have_e = false, ok = true;
  for (int j = 0; j < ntiles; ++j) {
    const int buf = j & 1;
    const int t0 = (jb + j) * kTile;
    const int sb = j % kScaleBufs;
    const uint32_t s_addr = tmem + (buf ? C::S_COL1 : C::S_COL0) + lane_base;
    if (j + 1 < ntiles) prefetch_mask(j + 1);
    const float4 *kq4 = reinterpret_cast<const float4 *>(ks_s + sb * kTile);
    const float4 *vs4 = reinterpret_cast<const float4 *>(vs_s + sb * kTile);
    const bool full = t0 + kTile - 1 <= vis_last;  // every slot of the tile visible to this row
    ok = __all_sync(0xffffffffu, wait_phase(&bars[kBarSFull0 + buf], (j >> 1) & 1, abort_flag, a.wait_ns));
    if (!ok) break;
    tc_fence_after();
    if constexpr (C::MSTAGE) {
      if (missue && j + 1 < ntiles) issue_mask(j + 1);
      ok = __all_sync(0xffffffffu, wait_phase(&bars[kBarMask0 + j % 3], (j / 3) & 1, abort_flag, a.wait_ns));
      if (!ok) break;
      mpend &= ~(1u << (j % 3));
    }
    const float *mrow = reinterpret_cast<const float *>(msk + ((j % 3) * RPH + (t - g * RPH)) * C::MROW);
    // pass 1, per 32 columns: the tile max (masked scores are written back over S)
    float mt = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t u[32];
      tmem_ld32(s_addr + c * 32, u);
      tmem_ld_wait();
      if constexpr (C::MASK) {
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const int j0 = t0 + c * 32 + q4 * 4;
          const float4 kk = kq4[c * 8 + q4];
          float4 mv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          if (row_ok && j0 < loop_end) {  // in bounds: loop_end <= S, S % 4 == 0
            if constexpr (C::MSTAGE)
              mv = *reinterpret_cast<const float4 *>(mrow + c * 32 + q4 * 4);
            else
              mv = *reinterpret_cast<const float4 *>(a.mask + b * a.mask_bstride + static_cast<int64_t>(pos) * a.S + j0);
          }
          const float kf[4] = {kk.x, kk.y, kk.z, kk.w}, mf[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float x = fmaf(__uint_as_float(u[q4 * 4 + e]), kf[e], mf[e] * 1.4426950408889634f);
            if (!full && j0 + e > vis_last) x = -INFINITY;
            u[q4 * 4 + e] = __float_as_uint(x);
            mt = fmaxf(mt, x);
          }
        }
        tmem_st32(s_addr + c * 32, u);
      } else if (full) {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // independent chains
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 kk = kq4[c * 8 + q4];
          m4[0] = fmaxf(m4[0], __uint_as_float(u[q4 * 4]) * kk.x);
          m4[1] = fmaxf(m4[1], __uint_as_float(u[q4 * 4 + 1]) * kk.y);
          m4[2] = fmaxf(m4[2], __uint_as_float(u[q4 * 4 + 2]) * kk.z);
          m4[3] = fmaxf(m4[3], __uint_as_float(u[q4 * 4 + 3]) * kk.w);
        }
        mt = fmaxf(mt, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
      } else {
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const int j0 = t0 + c * 32 + q4 * 4;
          const float4 kk = kq4[c * 8 + q4];
          const float kf[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (j0 + e <= vis_last) mt = fmaxf(mt, __uint_as_float(u[q4 * 4 + e]) * kf[e]);
        }
      }
    }
    if constexpr (C::MASK) tmem_st_wait();
    // running max (raised only by more than 8) and the P exponent E
    const bool raise = mt > m + 8.0f;
    const float mnew = raise ? mt : m;
    const float am = (raise && m != -INFINITY) ? ex2f(m - mnew) : 1.0f;
    const float4 vm4 = *reinterpret_cast<const float4 *>(vmx_s + sb * 4);
    const float vmx = fmaxf(fmaxf(vm4.x, vm4.y), fmaxf(vm4.z, vm4.w));
    int Enew = E;
    if (vmx > 0.0f) {
      const int et = ceil_log2(vmx);  // every v_scale of the tile is <= 2^et
      if (!have_e || et > E - 2 || et < E - 10) Enew = max(-100, min(100, et + 2));
    }
    const float ae = have_e ? exp2i(E - Enew) : 1.0f;
    have_e = have_e || vmx > 0.0f;
    const float ao = am * ae;
    if (j > 0 && __any_sync(0xffffffffu, ao != 1.0f)) {
      // O must hold everything up to PV_{j-1} before it is rescaled
      ok = __all_sync(0xffffffffu, wait_phase(&bars[kBarODone], (j - 1) & 1, abort_flag, a.wait_ns));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + C::O_COL + lane_base + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * ao);
        tmem_st32(tmem + C::O_COL + lane_base + c * 32, o);
      }
      tmem_st_wait();
    }
    l *= ao;
    m = mnew;
    E = Enew;
    // a row that has seen nothing yet has m = -inf: every p' is then 0
    const float me = (m == -INFINITY ? 0.0f : m) + static_cast<float>(E);
    // pass 2: P = p' * v_scale as fp16 pairs; slots 32c..32c+31 become the
    // packed columns 16c..16c+15, below every column not yet read back
    float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // independent chains for the row sum
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t u[32];
      tmem_ld32(s_addr + c * 32, u);
      tmem_ld_wait();
      uint32_t pw[16];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const int j0 = t0 + c * 32 + q4 * 4;
        const float4 kk = kq4[c * 8 + q4];
        const float4 vv = vs4[c * 8 + q4];
        const float kf[4] = {kk.x, kk.y, kk.z, kk.w}, vf[4] = {vv.x, vv.y, vv.z, vv.w};
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float r = __uint_as_float(u[q4 * 4 + e]);
          float x = C::MASK ? r - me : fmaf(r, kf[e], -me);
          if (!C::MASK && !full && j0 + e > vis_last) x = -INFINITY;
          p[e] = ex2f(x);  // -inf -> 0
          l4[e] += p[e];
          p[e] *= vf[e];
        }
        const __half2 h0 = __floats2half2_rn(p[0], p[1]);
        const __half2 h1 = __floats2half2_rn(p[2], p[3]);
        pw[q4 * 2] = *reinterpret_cast<const uint32_t *>(&h0);
        pw[q4 * 2 + 1] = *reinterpret_cast<const uint32_t *>(&h1);
      }
      tmem_st16(s_addr + c * 16, pw);
    }
    l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(&bars[kBarPFull0 + buf]);
  }
  // after an abort: this thread's mask copies still in flight land before the CTA exits
  if (missue && mpend)
    for (int mb = 0; mb < 3; ++mb)
      if (mpend & (1u << mb)) mbar_wait_bounded(&bars[kBarMask0 + mb], (mpar >> mb) & 1u);
  // ---- epilogue: O / l -> bf16 (the TMEM loads are warp-collective: every lane runs them)
  if (ok && ntiles > 0) ok = __all_sync(0xffffffffu, wait_phase(&bars[kBarOFinal], 0, abort_flag, a.wait_ns));
  if (a.ns > 1) {
    // KV split: publish this row's running max, P exponent and sum; the cluster
    // merge reads O from TMEM
    const bool have = ok && ntiles > 0 && m != -INFINITY;
    reinterpret_cast<float4 *>(smem + C::STAT_OFF)[t] =
        make_float4(have ? m : -INFINITY, static_cast<float>(E), have ? l : 0.0f, 0.0f);
    return;
  }
  if (ok) {
    tc_fence_after();
    uint16_t *op = a.out + ((static_cast<int64_t>(b) * a.Hq + hq) * a.Lq + (row_ok ? pos : 0)) * D;
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tmem + C::O_COL + lane_base + c * 32, o);
      tmem_ld_wait();
      if (row_ok) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __nv_bfloat162 v2 =
              __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          w[i] = *reinterpret_cast<const uint32_t *>(&v2);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(op + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
  }
}

// converter warpgroups: K (warps 4-7), V (warps 8-11)
template <class C>
__device__ __noinline__ void role_convert(const PrefillArgs &a, const Ctx x) {
  constexpr int D = C::D;
  uint8_t *smem = x.smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF + 4);
  const float *qs_s = reinterpret_cast<const float *>(smem + C::MISC_OFF + 8);  // sm_scale * log2e * 2^sh
  float *ks_s = reinterpret_cast<float *>(smem + C::KS_OFF);
  float *vs_s = reinterpret_cast<float *>(smem + C::VS_OFF);
  float *vmx_s = reinterpret_cast<float *>(smem + C::VMX_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * a.Hkv + blockIdx.y / a.nhc;
  const int loop_end = x.loop_end, ntiles = x.ntiles, jb = x.jb;
  // ======================= converter warpgroups: K (warps 4-7), V (warps 8-11)
  const bool is_k = warp < 8;
  const int c = tid - kSoftmaxThreads - (is_k ? 0 : kConvThreads);  // 0..127
  const int part = c % C::PPR;  // which 16 codes of a slot row
  const int sg = c / C::PPR;    // this thread's slots: sg*NCH .. sg*NCH + NCH-1
  // placement: 64-element block and 16-byte chunk of the two halves; lanes
  // with bit 2 set store their halves in the other order, which puts the 8
  // lanes of every quarter-warp on 8 different 16-byte bank groups
  const int blk = part >> 2;
  const int ch = (part & 3) * 2;
  const bool swap = (c & 4) != 0;
  const int8_t *base = (is_k ? a.k : a.v) + bh * a.S * D + part * 16;
  const int8_t *zb = (is_k ? a.kz : a.vz) + bh * a.S + sg * C::NCH;
  const int off = is_k ? C::K_OFF : C::V_OFF;

  // Each thread streams its chunks through a window of W registers: right
  // after chunk r of tile j is converted and stored, the load of the chunk W
  // places later (in this tile or the next) is issued into the same
  // registers, so loads are in flight while earlier chunks are converted and
  // while the tensor core still holds the buffer.
  constexpr int W = C::NCH < 8 ? C::NCH : 8;
  static_assert(C::NCH % W == 0, "window");
  uint4 w[W];
  uint32_t zw[C::NCH / 4], zn[C::NCH / 4];  // zero points of this / the next tile, 4 per word
  auto load_chunk = [&](int r, int t0, int n) {
    const int s = sg * C::NCH + r;
    w[r % W] = s < n ? ld_codes(base + static_cast<int64_t>(t0 + s) * D)
                     : make_uint4(0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u);
  };
  auto load_zp = [&](uint32_t (&z)[C::NCH / 4], int t0, int n) {
    const bool any = sg * C::NCH < n;  // the group starts inside the tile (and inside the cache)
#pragma unroll
    for (int i = 0; i < C::NCH / 4; ++i) z[i] = any ? ld_u32(zb + t0 + 4 * i) : 0u;
    // past the tile's end: code -128 with zero point -128 gives exactly 0
#pragma unroll
    for (int r = 0; r < C::NCH; ++r)
      if (sg * C::NCH + r >= n) z[r >> 2] = (z[r >> 2] & ~(0xFFu << (8 * (r & 3)))) | (0x80u << (8 * (r & 3)));
  };
  auto tile_n = [&](int j) { return min(kTile, loop_end - (jb + j) * kTile); };
  // convert + store this tile's chunks, loading W chunks ahead behind them
  auto convert_tile = [&](int j) {
    const bool next = j + 1 < ntiles;
    const int t0 = (jb + j) * kTile, n0 = tile_n(j);
    const int t1 = (jb + j + 1) * kTile, n1 = next ? tile_n(j + 1) : 0;
#pragma unroll
    for (int r = 0; r < C::NCH; ++r) {
      const int s = sg * C::NCH + r;
      const int zp = static_cast<int8_t>((zw[r >> 2] >> (8 * (r & 3))) & 0xFFu);
      uint4 lo, hi;
      codes16_to_f16(w[r % W], zp_const2(zp), lo, hi);
      const uint32_t o = static_cast<uint32_t>(off + blk * (kTile * 128));
      const uint32_t a_lo = o + swz(s, ch), a_hi = o + swz(s, ch + 1);
      *reinterpret_cast<uint4 *>(smem + (swap ? a_hi : a_lo)) = swap ? hi : lo;
      *reinterpret_cast<uint4 *>(smem + (swap ? a_lo : a_hi)) = swap ? lo : hi;
      if (r + W < C::NCH)
        load_chunk(r + W, t0, n0);
      else if (next)
        load_chunk(r + W - C::NCH, t1, n1);
    }
#pragma unroll
    for (int i = 0; i < C::NCH / 4; ++i) zw[i] = zn[i];
  };
  bool ok = true;
  {
    const int n0 = tile_n(0);
#pragma unroll
    for (int r = 0; r < W; ++r) load_chunk(r, jb * kTile, n0);
    load_zp(zw, jb * kTile, n0);
  }
  if (is_k) {
    // K tiles, and with each the per-slot k_scale * qs, v_scale and max v_scale
    float qs = 0.0f;
    float ksv = c < tile_n(0) ? ld_f32(a.ks + bh * a.S + jb * kTile + c) : 0.0f;
    float vsv = c < tile_n(0) ? ld_f32(a.vs + bh * a.S + jb * kTile + c) : 0.0f;
    for (int j = 0; j < ntiles; ++j) {
      float ksn = 0.0f, vsn = 0.0f;
      if (j + 1 < ntiles) {
        const int t1 = (jb + j + 1) * kTile, n1 = tile_n(j + 1);
        load_zp(zn, t1, n1);
        ksn = c < n1 ? ld_f32(a.ks + bh * a.S + t1 + c) : 0.0f;
        vsn = c < n1 ? ld_f32(a.vs + bh * a.S + t1 + c) : 0.0f;
      }
      // the buffer is free once QK_{j-1} has run; qs is published with Q
      ok = __all_sync(0xffffffffu, j == 0 ? wait_phase(&bars[kBarQ], 0, abort_flag, a.wait_ns)
                                          : wait_phase(&bars[kBarKEmpty], (j - 1) & 1, abort_flag, a.wait_ns));
      if (!ok) break;
      if (j == 0) qs = *qs_s;
      convert_tile(j);
      const int sb = j % kScaleBufs;
      ks_s[sb * kTile + c] = ksv * qs;
      vs_s[sb * kTile + c] = vsv;
      float vm = (jb + j) * kTile + c < x.vis_end ? vsv : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
      if (lane == 0) vmx_s[sb * 4 + (warp - 4)] = vm;
      proxy_fence();
      mbar_arrive(&bars[kBarKFull]);
      ksv = ksn;
      vsv = vsn;
    }
  } else {
    for (int j = 0; j < ntiles; ++j) {
      if (j + 1 < ntiles) load_zp(zn, (jb + j + 1) * kTile, tile_n(j + 1));
      if (j > 0) {  // the buffer is free once PV_{j-1} has run
        ok = __all_sync(0xffffffffu, wait_phase(&bars[kBarVEmpty], (j - 1) & 1, abort_flag, a.wait_ns));
        if (!ok) break;
      }
      convert_tile(j);
      proxy_fence();
      mbar_arrive(&bars[kBarVFull]);
    }
  }
}

// ---- block caches (kvq_write modes 1-6) ---------------------------------------
// IndexerQuantCache, 计算公式: x ~ code * scale_g with one scale per 32
// elements along the head dim.  The scales vary along the contraction of
// Q K^T (and along the output dim of P V), so they cannot be applied to the
// fp32 scores as the int8 k_scale is; the converters apply them instead, per
// element, after factoring out one power of two per slot:
//   K'[s][d] = code * scale_g(d) * 2^-E_s  (fp16),  k factor of slot s = 2^E_s,
// with 2^E_s the smallest power of two >= the slot's largest group scale, so
// |K'| <= |code| (at most 57344 for E5M2, inside fp16).  V likewise with its
// own exponent F_s, and 2^F_s takes the place of v_scale in P.  With E8M0
// scales the group factor is a power of two and K', V' are exact unless they
// fall below fp16's smallest subnormal (2^-24 of the slot's largest group
// factor); with float scales (modes 1, 4, 6) each element is rounded to fp16
// once (relative error <= 2^-11).
template <int MODE>
struct BlockFmt {
  static constexpr bool FP4 = MODE == KVQ_MODE_MXFP4;
  static constexpr bool E5 = MODE == KVQ_MODE_FP8_E5M2 || MODE == KVQ_MODE_MXFP8_E5M2;
  static constexpr bool I8 = MODE == KVQ_MODE_INT8_SYM;
  static constexpr bool F32S = MODE == KVQ_MODE_FP8_E4M3 || MODE == KVQ_MODE_FP8_E5M2 || I8;
  static constexpr int PART_BYTES = FP4 ? 8 : 16;  // bytes holding 16 codes
};

// Four byte codes of a word -> two f16x2 words (code 0 in the low half), exact.
template <int MODE>
KVQ_DEVINL void codes4_to_f16(uint32_t w, uint32_t &h01, uint32_t &h23) {
  using F = BlockFmt<MODE>;
  if constexpr (F::E5) {  // an E5M2 code is the high byte of the equal fp16
    h01 = __byte_perm(w, 0u, 0x1404);
    h23 = __byte_perm(w, 0u, 0x3424);
  } else if constexpr (F::I8) {  // (c + 128) in the mantissa of 1024, minus 1152
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t a = __byte_perm(u, 0x64646464u, 0x4140), b = __byte_perm(u, 0x64646464u, 0x4342);
    const __half2 k1152 = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
    const __half2 ra = __hsub2(*reinterpret_cast<const __half2 *>(&a), k1152);
    const __half2 rb = __hsub2(*reinterpret_cast<const __half2 *>(&b), k1152);
    h01 = *reinterpret_cast<const uint32_t *>(&ra);
    h23 = *reinterpret_cast<const uint32_t *>(&rb);
  } else {  // E4M3
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"(static_cast<uint16_t>(w & 0xFFFFu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"(static_cast<uint16_t>(w >> 16)));
  }
}

// 16 codes of one part (16 bytes; E2M1: 8 bytes, element 2i in the low nibble
// of byte i) -> 16 fp16 values code * f, in element order.
template <int MODE>
KVQ_DEVINL void block16_to_f16(const uint4 &w, float f, uint4 &lo, uint4 &hi) {
  using F = BlockFmt<MODE>;
  uint32_t h[8];
  if constexpr (F::FP4) {
    const uint32_t in[2] = {w.x, w.y};
#pragma unroll
    for (int i = 0; i < 8; ++i)
      asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
          : "=r"(h[i])
          : "r"((in[i >> 2] >> (8 * (i & 3))) & 0xFFu));
  } else {
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) codes4_to_f16<MODE>(in[i], h[2 * i], h[2 * i + 1]);
  }
  if constexpr (F::F32S) {  // one rounding: code * f in fp32, then to fp16
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&h[i]));
      const __half2 r = __floats2half2_rn(v.x * f, v.y * f);
      h[i] = *reinterpret_cast<const uint32_t *>(&r);
    }
  } else {  // f is a power of two (or 0): exact unless the result is below 2^-24
    const __half2 ff = __float2half2_rn(f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&h[i]), ff);
      h[i] = *reinterpret_cast<const uint32_t *>(&r);
    }
  }
  lo = make_uint4(h[0], h[1], h[2], h[3]);
  hi = make_uint4(h[4], h[5], h[6], h[7]);
}

KVQ_DEVINL uint2 ld_codes8(const void *p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

// The NG per-32 scales of one slot as raw 32-bit words (floats, or E8M0 bytes
// packed four per word).
template <int MODE, int NG>
struct ScaleRow {
  static constexpr int W = BlockFmt<MODE>::F32S ? NG : (NG + 3) / 4;
  uint32_t w[W];
  KVQ_DEVINL void clear() {
#pragma unroll
    for (int i = 0; i < W; ++i) w[i] = 0u;
  }
  KVQ_DEVINL void load(const void *row) {
    if constexpr (BlockFmt<MODE>::F32S) {
#pragma unroll
      for (int i = 0; i < NG; i += 2) {
        const uint2 v = ld_codes8(static_cast<const uint32_t *>(row) + i);
        w[i] = v.x;
        w[i + 1] = v.y;
      }
    } else if constexpr (NG == 2) {
      uint16_t h;
      asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(h) : "l"(row));
      w[0] = h;
    } else if constexpr (NG == 4) {
      w[0] = ld_u32(row);
    } else {
      const uint2 v = ld_codes8(row);
      w[0] = v.x;
      w[1] = v.y;
    }
  }
  // The slot's exponent E (2^E >= every group scale, E in [-126, 126]) and the
  // group factors scale_g * 2^-E.
  KVQ_DEVINL int factors(float (&f)[NG]) const {
    if constexpr (BlockFmt<MODE>::F32S) {
      uint32_t mx = 0u;
#pragma unroll
      for (int g = 0; g < NG; ++g) mx = max(mx, w[g] & 0x7FFFFFFFu);
      const int E = mx == 0u ? 0 : max(-126, min(126, ceil_log2(__uint_as_float(mx))));
      const float inv = exp2i(-E);
#pragma unroll
      for (int g = 0; g < NG; ++g) f[g] = __uint_as_float(w[g]) * inv;
      return E;
    } else {
      int e[NG], mx = 0;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        e[g] = static_cast<int>((w[g >> 2] >> (8 * (g & 3))) & 0xFFu);
        mx = max(mx, e[g]);
      }
      const int E = max(-126, mx - 127);
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const int k = e[g] - 127 - E;  // <= 0
        f[g] = k >= -126 ? exp2i(k) : 0.0f;
      }
      return E;
    }
  }
};

// AND of `v` over the 128 threads of one converter warpgroup (named barrier
// `id`); also orders their shared-memory accesses like a barrier.
KVQ_DEVINL bool group_and(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(id)
      : "memory");
  return r != 0;
}

// converter warpgroups over a block cache: K (warps 4-7), V (warps 8-11).
// Thread c first turns the scale row of slot c into the slot's exponent and
// group factors (shared memory, double-buffered by tile), then converts its
// 16-code parts as the int8 converters do.
template <class C>
__device__ __noinline__ void role_convert_block(const PrefillArgs &a, const Ctx x) {
  constexpr int D = C::D, MODE = C::MODE, NG = C::NG;
  using F = BlockFmt<MODE>;
  using Row = ScaleRow<MODE, NG>;
  constexpr int CBS = F::FP4 ? D / 2 : D;  // code bytes per slot
  constexpr int SRB = F::F32S ? NG * 4 : NG;  // scale bytes per slot
  uint8_t *smem = x.smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF + 4);
  const float *qs_s = reinterpret_cast<const float *>(smem + C::MISC_OFF + 8);
  float *ks_s = reinterpret_cast<float *>(smem + C::KS_OFF);
  float *vs_s = reinterpret_cast<float *>(smem + C::VS_OFF);
  float *vmx_s = reinterpret_cast<float *>(smem + C::VMX_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = static_cast<int64_t>(blockIdx.z) * a.Hkv + blockIdx.y / a.nhc;
  const int loop_end = x.loop_end, ntiles = x.ntiles, jb = x.jb;
  const bool is_k = warp < 8;
  const int c = tid - kSoftmaxThreads - (is_k ? 0 : kConvThreads);  // 0..127
  const int part = c % C::PPR, sg = c / C::PPR, grp = part >> 1;
  const int blk = part >> 2, ch = (part & 3) * 2;
  const bool swap = (c & 4) != 0;  // bank spreading of the stores, as in role_convert
  const uint8_t *base = reinterpret_cast<const uint8_t *>(is_k ? a.k : a.v) + bh * a.S * CBS + part * F::PART_BYTES;
  const uint8_t *own_sc =
      F::F32S ? reinterpret_cast<const uint8_t *>(is_k ? a.ks : a.vs) : (is_k ? a.ks8 : a.vs8);
  const uint8_t *v_sc = F::F32S ? reinterpret_cast<const uint8_t *>(a.vs) : a.vs8;
  own_sc += bh * a.S * SRB;
  v_sc += bh * a.S * SRB;
  float *fac = reinterpret_cast<float *>(smem + C::FAC_OFF) + (is_k ? 0 : 2 * kTile * NG);
  const int off = is_k ? C::K_OFF : C::V_OFF;
  const int bar_id = is_k ? 2 : 3;

  constexpr int W = C::NCH < 8 ? C::NCH : 8;
  static_assert(C::NCH % W == 0, "window");
  uint4 w[W];
  auto load_chunk = [&](int r, int t0, int n) {
    const int s = sg * C::NCH + r;
    if (s < n) {
      const uint8_t *p = base + static_cast<int64_t>(t0 + s) * CBS;
      if constexpr (F::FP4) {
        const uint2 v = ld_codes8(p);
        w[r % W] = make_uint4(v.x, v.y, 0u, 0u);
      } else {
        w[r % W] = ld_codes(p);
      }
    } else {
      w[r % W] = make_uint4(0u, 0u, 0u, 0u);  // code 0 is +0 in every format
    }
  };
  auto tile_n = [&](int j) { return min(kTile, loop_end - (jb + j) * kTile); };
  auto convert_tile = [&](int j) {
    const bool next = j + 1 < ntiles;
    const int t0 = (jb + j) * kTile, n0 = tile_n(j);
    const int t1 = (jb + j + 1) * kTile, n1 = next ? tile_n(j + 1) : 0;
    const float *fb = fac + (j & 1) * kTile * NG;
#pragma unroll
    for (int r = 0; r < C::NCH; ++r) {
      const int s = sg * C::NCH + r;
      uint4 lo, hi;
      block16_to_f16<MODE>(w[r % W], fb[s * NG + grp], lo, hi);
      const uint32_t o = static_cast<uint32_t>(off + blk * (kTile * 128));
      const uint32_t a_lo = o + swz(s, ch), a_hi = o + swz(s, ch + 1);
      *reinterpret_cast<uint4 *>(smem + (swap ? a_hi : a_lo)) = swap ? hi : lo;
      *reinterpret_cast<uint4 *>(smem + (swap ? a_lo : a_hi)) = swap ? lo : hi;
      if (r + W < C::NCH)
        load_chunk(r + W, t0, n0);
      else if (next)
        load_chunk(r + W - C::NCH, t1, n1);
    }
  };

  // scale rows of slot c: this tile's (cur) and the next tile's (nxt); the K
  // converters also read the V rows, for the per-slot V factor 2^F
  Row cur, nxt, vcur, vnxt;
  {
    const int n0 = tile_n(0);
#pragma unroll
    for (int r = 0; r < W; ++r) load_chunk(r, jb * kTile, n0);
    cur.clear();
    vcur.clear();
    if (c < n0) {
      cur.load(own_sc + static_cast<int64_t>(jb * kTile + c) * SRB);
      if (is_k) vcur.load(v_sc + static_cast<int64_t>(jb * kTile + c) * SRB);
    }
  }
  float qs = 0.0f;
  bool ok = true;
  for (int j = 0; j < ntiles; ++j) {
    const int n = tile_n(j);
    nxt.clear();
    vnxt.clear();
    if (j + 1 < ntiles && c < tile_n(j + 1)) {
      const int64_t t = static_cast<int64_t>(jb + j + 1) * kTile + c;
      nxt.load(own_sc + t * SRB);
      if (is_k) vnxt.load(v_sc + t * SRB);
    }
    // K: the buffer is free once QK_{j-1} has run (qs is published with Q);
    // V: once PV_{j-1} has run
    if (is_k)
      ok = __all_sync(0xffffffffu, j == 0 ? wait_phase(&bars[kBarQ], 0, abort_flag, a.wait_ns)
                                          : wait_phase(&bars[kBarKEmpty], (j - 1) & 1, abort_flag, a.wait_ns));
    else if (j > 0)
      ok = __all_sync(0xffffffffu, wait_phase(&bars[kBarVEmpty], (j - 1) & 1, abort_flag, a.wait_ns));
    if (ok) {
      float f[NG];
      const int E = cur.factors(f);
      const bool valid = c < n;
      float *fr = fac + ((j & 1) * kTile + c) * NG;
#pragma unroll
      for (int g = 0; g < NG; ++g) fr[g] = valid ? f[g] : 0.0f;
      if (is_k) {
        if (j == 0) qs = *qs_s;
        float fv[NG];
        const int Ev = vcur.factors(fv);
        const int sb = j % kScaleBufs;
        const float vsv = valid ? exp2i(Ev) : 0.0f;
        ks_s[sb * kTile + c] = valid ? exp2i(E) * qs : 0.0f;
        vs_s[sb * kTile + c] = vsv;
        float vm = (jb + j) * kTile + c < x.vis_end ? vsv : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
        if (lane == 0) vmx_s[sb * 4 + (warp - 4)] = vm;
      }
    }
    // one decision for the warpgroup (a warp that gave up must not leave the
    // others at the barrier), which also publishes the factors
    ok = group_and(bar_id, ok);
    if (!ok) break;
    convert_tile(j);
    proxy_fence();
    mbar_arrive(&bars[is_k ? kBarKFull : kBarVFull]);
    cur = nxt;
    vcur = vnxt;
  }
}

// MMA warp: lane 0 issues
template <class C>
__device__ __noinline__ void role_mma(const PrefillArgs &a, const Ctx x) {
  constexpr int D = C::D;
  uint8_t *smem = x.smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF + 4);
  const int lane = threadIdx.x & 31;
  const uint32_t tmem = x.tmem;
  const int ntiles = x.ntiles;
  // ======================= MMA warp: lane 0 issues
  if (lane == 0) {
    constexpr uint32_t ID_QK = idesc_f16(kRows, kTile, 0);
    constexpr uint32_t ID_PV = idesc_f16(kRows, D, 1);
    const uint32_t q_base = smem_u32(smem + C::Q_OFF), k_base = smem_u32(smem + C::K_OFF);
    const uint32_t v_base = smem_u32(smem + C::V_OFF);
    // Q and K regions share the [128 rows x 128 B] block shape (kRows == kTile)
    static_assert(kRows == kTile, "Q and K block strides");
    auto issue_qk = [&](int j) {
      const uint32_t d = tmem + ((j & 1) ? C::S_COL1 : C::S_COL0);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = static_cast<uint32_t>(k >> 2) * (kRows * 128) + (k & 3) * 32;
        mma_ss(d, sdesc(q_base + off, 16, 1024), sdesc(k_base + off, 16, 1024), ID_QK, k > 0 ? 1u : 0u);
      }
      mma_commit(&bars[kBarSFull0 + (j & 1)]);
      mma_commit(&bars[kBarKEmpty]);
    };
    bool ok = ntiles > 0;  // a KV split can be left without tiles
    if (ok) ok = wait_phase(&bars[kBarQ], 0, abort_flag, a.wait_ns);
    if (ok) ok = wait_phase(&bars[kBarKFull], 0, abort_flag, a.wait_ns);
    if (ok) {
      tc_fence_after();
      issue_qk(0);
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      if (j + 1 < ntiles) {
        ok = wait_phase(&bars[kBarKFull], (j + 1) & 1, abort_flag, a.wait_ns);
        // S buffer (j+1)&1 holds P_{j-1} until PV_{j-1} has run
        if (ok && j >= 1) ok = wait_phase(&bars[kBarODone], (j - 1) & 1, abort_flag, a.wait_ns);
        if (!ok) break;
        tc_fence_after();
        issue_qk(j + 1);
      }
      ok = wait_phase(&bars[kBarVFull], j & 1, abort_flag, a.wait_ns);
      if (ok) ok = wait_phase(&bars[kBarPFull0 + (j & 1)], (j >> 1) & 1, abort_flag, a.wait_ns);
      if (!ok) break;
      tc_fence_after();
      const uint32_t p_tmem = tmem + ((j & 1) ? C::S_COL1 : C::S_COL0);
#pragma unroll
      for (int k = 0; k < kTile / 16; ++k)  // 16 slots = 8 packed TMEM columns of P
        mma_ts(tmem + C::O_COL, p_tmem + k * 8, sdesc(v_base + k * 2048, kTile * 128, 1024), ID_PV,
               (j > 0 || k > 0) ? 1u : 0u);
      mma_commit(&bars[kBarODone]);
      mma_commit(&bars[kBarVEmpty]);
      if (j + 1 == ntiles) mma_commit(&bars[kBarOFinal]);
    }
    // everything issued finishes before TMEM is released, on every path (after
    // an abort the softmax may have stopped waiting for the last PV)
    mma_commit(&bars[kBarDrain]);
    mbar_wait_bounded(&bars[kBarDrain], 0);
  }
  __syncwarp();
}

// ---- KV split across a thread-block cluster --------------------------------
// The cluster's CTAs each hold (m, E, l, O) of one share of the KV tiles for
// the same 128 query rows (O and l in units of 2^-(m+E)).  Against the share r
// with the largest m (the first such), share c weighs f_c = 2^(m_c - m_r) 2^(E_c - E_r),
// the power of two applied exactly, and contributes O_c f_c / L with
// L = sum_c l_c f_c.  A share whose E moved by k over tiles that no row sees
// has O and l scaled by exactly 2^-k and f_c by 2^k, so the output does not
// depend on whether such tiles were visited.  Each CTA writes its contribution
// to its own shared memory, then sums one slice of the rows over the cluster
// (distributed shared memory) and stores it.  All threads take part.
template <class C>
__device__ __noinline__ void cluster_merge(const PrefillArgs &a, const Ctx x, bool o_valid) {
  constexpr int D = C::D, HPT = C::HPT, RPH = C::RPH;
  uint8_t *smem = x.smem;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int ns = a.ns;
  const uint32_t rank = cluster_rank();
  const uint32_t stat_l = smem_u32(smem + C::STAT_OFF), contrib_l = smem_u32(smem + C::CONTRIB_OFF);
  // 16-byte chunk k of row r sits at chunk k ^ (r & 7) (rows are D * 4 bytes apart)
  auto cidx = [](int r, int k) { return r * (D / 4) + (k ^ (r & 7)); };
  cluster_sync();  // every share's row statistics are published
  if (tid < kRows) {  // the softmax warps own TMEM lanes 0..127: row t
    const int t = tid;
    float4 st[kMaxSplit];  // (m, E, l, -) of every share, all loads in flight at once
#pragma unroll
    for (int c = 0; c < kMaxSplit; ++c)
      st[c] = c < ns ? ld_peer_f4(peer_addr(stat_l + 16 * t, c)) : make_float4(-INFINITY, 0.0f, 0.0f, 0.0f);
    float mr = -INFINITY, er = 0.0f;
#pragma unroll
    for (int c = 0; c < kMaxSplit; ++c) {
      if (c < ns && st[c].x > mr) {
        mr = st[c].x;
        er = st[c].y;
      }
    }
    auto weight = [&](const float4 &sc) {
      return sc.x == -INFINITY ? 0.0f : ldexpf(ex2f(sc.x - mr), static_cast<int>(sc.y - er));
    };
    float L = 0.0f, w_self = 0.0f;
#pragma unroll
    for (int c = 0; c < kMaxSplit; ++c) {
      if (c < ns) {
        const float w = weight(st[c]);
        L = fmaf(st[c].z, w, L);
        if (c == static_cast<int>(rank)) w_self = w;
      }
    }
    const float f = L > 0.0f ? w_self / L : 0.0f;
    float4 *dst = reinterpret_cast<float4 *>(smem + C::CONTRIB_OFF);
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    if (o_valid) tc_fence_after();
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      if (o_valid) {  // warp-uniform
        tmem_ld32(x.tmem + C::O_COL + lane_base + cc * 32, o);
        tmem_ld_wait();
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 v = o_valid && f != 0.0f
                             ? make_float4(__uint_as_float(o[4 * i]) * f, __uint_as_float(o[4 * i + 1]) * f,
                                           __uint_as_float(o[4 * i + 2]) * f, __uint_as_float(o[4 * i + 3]) * f)
                             : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        dst[cidx(t, cc * 8 + i)] = v;
      }
    }
  }
  cluster_sync();  // every contribution is written
  {
    const int xrow = blockIdx.x / ns, hkc = blockIdx.y, b = blockIdx.z;
    const int hk = hkc / a.nhc, hc = hkc - hk * a.nhc;
    const int r0 = static_cast<int>(rank) * kRows / ns, r1 = (static_cast<int>(rank) + 1) * kRows / ns;
    // kBatch items a thread at a time, every share's loads of all of them in flight
    // before the first add (a load from another CTA's shared memory is a long trip)
    constexpr int kBatch = 4;
    const int items = (r1 - r0) * (D / 4);
    for (int i0 = tid; i0 < items; i0 += kBatch * kThreads) {
      float4 v[kBatch][kMaxSplit];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kThreads;
        const int r = r0 + i / (D / 4), k = i % (D / 4);
#pragma unroll
        for (int c = 0; c < kMaxSplit; ++c)
          v[u][c] = i < items && c < ns ? ld_peer_f4(peer_addr(contrib_l + 16 * cidx(r, k), c))
                                        : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kThreads;
        if (i >= items) break;
        const int r = r0 + i / (D / 4), k = i % (D / 4);
        const int g = r / RPH, pos = xrow * RPH + (r - g * RPH);
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int c = 0; c < kMaxSplit; ++c) {
          if (c < ns) {
            acc.x += v[u][c].x;
            acc.y += v[u][c].y;
            acc.z += v[u][c].z;
            acc.w += v[u][c].w;
          }
        }
        if (pos < a.Lq) {
          const int hq = hk * a.G + hc * HPT + g;
          const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t *>(&lo);
          pk.y = *reinterpret_cast<const uint32_t *>(&hi);
          *reinterpret_cast<uint2 *>(a.out + ((static_cast<int64_t>(b) * a.Hq + hq) * a.Lq + pos) * D + 4 * k) = pk;
        }
      }
    }
  }
  cluster_sync();  // no CTA leaves while others still read its shared memory
}

template <class C>
__global__ void __maxnreg__(kRegsLaunch) prefill_tc_kernel(const __grid_constant__ PrefillArgs a) {
  constexpr int RPH = C::RPH;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (the 128-byte swizzle is a function of address bits 4-9)
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::MISC_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF + 4);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int xrow = blockIdx.x / a.ns, hkc = blockIdx.y, b = blockIdx.z;

  // ---- set-up
  if (tid == 0) {
    mbar_init(&bars[kBarQ], kSoftmaxThreads);
    mbar_init(&bars[kBarKFull], kConvThreads);
    mbar_init(&bars[kBarKEmpty], 1);
    mbar_init(&bars[kBarVFull], kConvThreads);
    mbar_init(&bars[kBarVEmpty], 1);
    mbar_init(&bars[kBarSFull0], 1);
    mbar_init(&bars[kBarSFull1], 1);
    mbar_init(&bars[kBarPFull0], kSoftmaxThreads);
    mbar_init(&bars[kBarPFull1], kSoftmaxThreads);
    mbar_init(&bars[kBarODone], 1);
    mbar_init(&bars[kBarOFinal], 1);
    mbar_init(&bars[kBarDrain], 1);
    for (int i = 0; i < 3; ++i) mbar_init(&bars[kBarMask0 + i], RPH);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  int kv = a.kv_per_batch ? a.kv_len[b] : *a.kv_len;
  if (kv < a.Lq || kv > a.S) {
    if (tid == 0 && xrow == 0 && hkc == 0 && (a.kv_per_batch || b == 0)) report(a.err, KVQ_ERR_KV_LEN_RANGE);
    kv = kv < a.Lq ? a.Lq : static_cast<int>(a.S);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // per-tile causal bound (the same in every role)
  const int last_pos = min(xrow * RPH + RPH, a.Lq) - 1;
  const int loop_end = a.mask_is_causal ? min(kv, kv - a.Lq + last_pos + 1) : kv;
  // With a KV split, share r of the cluster takes tiles [r T / ns, (r + 1) T / ns) of
  // the T tiles of the whole kv_len, clipped to the causal bound: the shares do not
  // depend on the bound, so the output is the same bit for bit with or without it.
  int jb = 0, ntiles = (loop_end + kTile - 1) / kTile;
  if (a.ns > 1) {
    const int T = (kv + kTile - 1) / kTile, r = static_cast<int>(cluster_rank());
    jb = r * T / a.ns;
    ntiles = max(0, min((r + 1) * T / a.ns, ntiles) - jb);
  }

  // The P exponent follows the largest v_scale of the slots some row of the CTA
  // can see; slots past the causal bound are left out, so visiting them (no
  // per-tile bound) changes nothing
  const int vis_end = a.is_causal ? min(kv, kv - a.Lq + last_pos + 1) : kv;
  const Ctx x{smem, tmem, kv, loop_end, jb, ntiles, vis_end};
  if (warp < 4)
    role_softmax<C>(a, x);
  else if (warp < 12)
    if constexpr (C::MODE == 0)
      role_convert<C>(a, x);
    else
      role_convert_block<C>(a, x);
  else
    role_mma<C>(a, x);

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (a.ns > 1) cluster_merge<C>(a, x, ntiles > 0 && !*abort_flag);
  if (tid == 0 && *abort_flag) report(a.err, KVQ_ERR_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

inline int hpt_for(int G) { return G % 4 == 0 ? 4 : (G % 2 == 0 ? 2 : 1); }

// Clusters of ns CTAs of kernel C that can be resident at once (0 if the query
// fails), queried once per kernel and cluster size.
template <class C>
int clusters_fit(int ns, dim3 grid) {
  static std::atomic<int> known[kMaxSplit + 1];
  const int k = known[ns].load(std::memory_order_relaxed);
  if (k != 0) return k > 0 ? k : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(ns);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, prefill_tc_kernel<C>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = -1;
  }
  known[ns].store(n, std::memory_order_relaxed);
  return n > 0 ? n : 0;
}

template <int D, int HPT, bool MASK, int MODE>
int launch_prefill_tc(PrefillArgs a, cudaStream_t stream) {
  using C = Cfg<D, HPT, MASK, MODE>;
  if (const int st = ensure_smem<C>(prefill_tc_kernel<C>, C::SMEM)) return st;
  a.nhc = a.G / HPT;
  const int rowblocks = (a.Lq + C::RPH - 1) / C::RPH;
  // KV split: when the row blocks leave most SMs idle, a cluster of ns CTAs
  // shares each one (up to 4, while the grid still fits one wave and every
  // share can hold a tile of the cache)
  const int64_t base = static_cast<int64_t>(rowblocks) * a.Hkv * a.nhc * a.B;
  const int64_t tiles = (a.S + kTile - 1) / kTile;
  const int sms = sm_count();
  a.ns = 1;
  if (base * 2 <= sms) {
    while (a.ns < kMaxSplit && base * a.ns * 2 <= sms && a.ns * 2 <= tiles) a.ns *= 2;
  } else {
    // Several waves of one CTA an SM: a launch takes about ceil(row blocks / clusters
    // resident at once) waves of 1/ns of a row block's tiles each; split when that is
    // shorter by more than the merge costs (a few percent), e.g. 512 row blocks on 148
    // SMs: 4 waves unsplit, 7 half-waves in pairs.
    double best = static_cast<double>((base + sms - 1) / sms);
    for (int ns = 2; ns <= kMaxSplit && ns * 2 <= tiles; ns *= 2) {
      const int fit = clusters_fit<C>(ns, dim3(rowblocks * ns, a.Hkv * a.nhc, a.B));
      if (fit <= 0) continue;
      const double t = static_cast<double>((base + fit - 1) / fit) / ns;
      if (t < 0.97 * best) {
        best = t;
        a.ns = ns;
      }
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rowblocks * a.ns, a.Hkv * a.nhc, a.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.ns;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.ns > 1 ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, prefill_tc_kernel<C>, a) != cudaSuccess) return KVQ_ECUDA;
  return launch_status();
}

template <int D, bool MASK, int MODE>
int dispatch_hpt(const PrefillArgs &a, cudaStream_t s) {
  switch (hpt_for(a.G)) {
    case 4: return launch_prefill_tc<D, 4, MASK, MODE>(a, s);
    case 2: return launch_prefill_tc<D, 2, MASK, MODE>(a, s);
    default: return launch_prefill_tc<D, 1, MASK, MODE>(a, s);
  }
}

// Every (D, mask, GQA head chunk) variant of one cache mode; D is 64, 128 or 256.
template <int MODE>
int dispatch_prefill_mode(const PrefillArgs &a, int D, cudaStream_t s) {
  switch (D) {
    case 64: return a.mask ? dispatch_hpt<64, true, MODE>(a, s) : dispatch_hpt<64, false, MODE>(a, s);
    case 128: return a.mask ? dispatch_hpt<128, true, MODE>(a, s) : dispatch_hpt<128, false, MODE>(a, s);
    default: return a.mask ? dispatch_hpt<256, true, MODE>(a, s) : dispatch_hpt<256, false, MODE>(a, s);
  }
}

}  // namespace tc
}  // namespace kvq
