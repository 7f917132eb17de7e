// kvq_decode.cu -- one-query (decode) attention over the int8 KV cache.
//
// What it computes (abaddon src/attention_cache/mod.rs, trait KvCache,
// forward_attention; ExecuTorch PR 20351 commit notes on the kv_len bound;
// ExecuTorch PR 24473, Summary, on the additive mask):
//   out[b,h] = softmax_j(sm_scale * q[b,h] . K[b,hk,j] + mask[j]) . V[b,hk,j],
//   j in [0, kv_len), hk = h / G, K = (k - k_zp) * k_scale, V likewise.
//
// Design (B200, sm_100a).  Decode is HBM-bound in bytes but, with GQA, heavy in
// CUDA-core instructions per byte, so the kernel is built to keep both the
// memory pipe and the issue slots busy:
//  - Persistent grid: one CTA per SM.  The work -- units (b, kv head, head
//    chunk) x chunks of 32 slots, with the chunk count derived on the device
//    from *kv_len -- is flattened and cut into equal contiguous ranges, one per
//    CTA, so every SM streams the same number of bytes (to one chunk) whatever
//    B, Hkv and kv_len are.  With one kv_len per batch row the flattening uses
//    each row's own length (a prefix of the rows' chunk counts in shared
//    memory), so long rows do not pile onto a few CTAs.  A CTA closes a segment
//    whenever its range moves to the next unit.
//  - Inside a CTA, chunk i of the range belongs to pipeline i mod NP.  A
//    pipeline is P warps (two when the head chunk is even: each takes half the
//    heads, which halves its registers and lets 16 warps share an SM) around an
//    R-deep ring of chunk buffers: the 1-D bulk async copies (TMA) of a chunk's
//    K/V codes, scales, zero points and mask land in a free buffer, completion
//    is counted on that buffer's mbarrier, and the warp of the pipeline that
//    finishes a buffer last refills it with the pipeline's chunk R ahead.  No
//    producer warp and no cross-pipeline hand-off.  Every wait is bounded.
//  - A lane owns 16 dims of L = D/16 slots of its pipeline's chunk in turn.
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
//      p.v: one byte permute turns a V code into the exact subnormal float
//      (c + 128) * 2^-149; the weights p * v_scale, scaled by 2^96, are
//      broadcast per slot through shared memory and accumulated with packed
//      fp32 FMA (the accumulators hold 2^-53 of the sums).  The zero point
//      and the +128 bias leave as one per-head correction,
//      sum_j p_j v_scale_j (128 + zp_j), subtracted when the warps merge; the
//      cancellation costs at most a few bits of fp32 (the sums are < 2^16).
//  - Segment close: groups merge by shuffles, warps through shared memory, in
//    a fixed order.  A unit that a CTA covers alone is written directly; a
//    unit split across CTAs leaves one partial per CTA in the workspace, and
//    the owner that completes the unit (a per-unit counter in the workspace,
//    reset to zero by that owner) merges the partials in owner order, so the
//    result does not depend on which CTA finishes last.
//  - The decode kernel itself is launched as a programmatic dependent of the
//    kernel before it (typically the cache write of the new token): its launch
//    and barrier set-up overlap that kernel's tail, and it reads nothing before
//    griddepcontrol.wait has seen that kernel complete.
#include <cuda_bf16.h>

#include <mutex>

#include "kvq_common.cuh"

namespace kvq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest p kept without rescaling
// p.v runs on V codes held as subnormal floats b * 2^-149 (b = code + 128, exact)
// and weights scaled by 2^96, so the accumulators hold 2^-53 of the true sums.
constexpr float kWScale = 79228162514264337593543950336.0f;  // 2^96
constexpr float kOScale = 9007199254740992.0f;                // 2^53
constexpr int kMaxCtas = 256;  // grid size limit (owner records staged per unit)
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
  const int32_t *kv_len;  // one device scalar, or [B] with kv_per_batch
  int kv_per_batch;
  uint16_t *out;
  int32_t *ws_cnt;    // [kMaxCtas] merge counters, one per CTA: the split unit whose first owner it is
  float *ws_ml;       // [C][2][HC][2]: (m, l) of the CTA's first and last unit, when split
  float *ws_o;        // [C][2][HC][D]
  int32_t *err;
  int64_t S;
  int B, Hq, Hkv, G, nhc;
  float qscale;  // sm_scale * log2(e)
};

// NP chunk pipelines of P warps each; a pipeline's warps share its chunk ring
// and split the HC heads of the unit, HW each.
template <int D_, int HC_, int NP_, int P_, int R_, bool Q4_ = false>
struct Cfg {
  static constexpr int D = D_, HC = HC_, NP = NP_, P = P_, R = R_;
  static constexpr int HW = HC / P, NW = NP * P;
  static_assert(HW * P == HC, "heads split evenly over a pipeline's warps");
  static constexpr bool Q4 = Q4_;            // TQ4 cache: 4-bit codes, two per byte
  static constexpr int CB = Q4 ? D / 2 : D;  // code bytes per slot
  static constexpr int L = D / 16;           // lanes per slot group (16 dims per lane)
  static constexpr int NG = 32 / L;          // slot groups per warp
  static constexpr int CS = 32;              // slots per chunk (one warp step)
  // one chunk buffer
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = CS * CB;
  static constexpr int KS_OFF = 2 * CS * CB;
  static constexpr int VS_OFF = KS_OFF + 4 * CS;
  static constexpr int M_OFF = VS_OFF + 4 * CS;
  static constexpr int KZ_OFF = M_OFF + 4 * CS;
  static constexpr int VZ_OFF = KZ_OFF + CS;
  static constexpr int CHUNK = VZ_OFF + CS;
  static_assert(CHUNK % 16 == 0, "chunk alignment");
  // NP rings of R chunk buffers, then the per-warp scratch
  static constexpr int WBUF_OFF = NP * R * CHUNK;              // [NW][32][4] float
  // a warp's published state: O [HW][D] float, then (m, l, corr, -) [HW][4] float
  static constexpr int PUBW = HW * D * 4 + HW * 16;
  static constexpr int OSCR_OFF = WBUF_OFF + NW * 32 * 16;     // [NW] published states (first unit)
  static constexpr int BAR_OFF = OSCR_OFF + NW * PUBW;         // [NP][R] mbarrier
  static constexpr int CNT_OFF = BAR_OFF + NP * R * 8;         // [NP][R] int: warps done with the buffer
  static constexpr int SH_OFF = (CNT_OFF + NP * R * 4 + 15) / 16 * 16;  // 8 ints
  static_assert(P * PUBW <= R * CHUNK, "the last unit's states fit a pipeline's (then idle) ring");
  static constexpr int Q_OFF = (SH_OFF + 32 + 15) / 16 * 16;     // [2][HC] q rows: D/4 high, D/4 low words
  static constexpr int QMETA_OFF = Q_OFF + 2 * HC * 2 * D;       // [2][HC] (sum n, 2^E)
  static constexpr int RECS_OFF = QMETA_OFF + 2 * HC * 8;        // [2][kMaxCtas] owner records
  static constexpr int PFX_OFF = RECS_OFF + 2 * kMaxCtas * 4;    // [kMaxRows + 1] chunk prefix, [32] scratch
  static constexpr int SMEM = PFX_OFF + (kMaxRows + 1 + 32) * 4;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr int THREADS = NW * 32;
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
// Add 1 to a merge counter, releasing this CTA's partial (written before the
// barrier that precedes the call) and acquiring the other owners'.
KVQ_DEVINL int count_acq_rel(int32_t *p) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// Count a warp as done with a ring buffer (the count orders its reads before
// the refill that the last warp of the pipeline issues).
KVQ_DEVINL int done_count(int32_t *p) {
  int old;
  asm volatile("atom.add.acq_rel.cta.shared::cta.s32 %0, [%1], 1;" : "=r"(old) : "r"(smem_u32(p)) : "memory");
  return old;
}

// Work split: CTA c owns flattened chunks [c*W/C, (c+1)*W/C); cta_of is its inverse.
KVQ_DEVINL int64_t range_start(int64_t c, int64_t W, int64_t C) { return c * W / C; }
KVQ_DEVINL int64_t cta_of(int64_t idx, int64_t W, int64_t C) { return ((idx + 1) * C - 1) / W; }

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
  constexpr int D = C::D, HC = C::HC, NW = C::NW, R = C::R, L = C::L, NG = C::NG, CS = C::CS, CB = C::CB;
  constexpr int NP = C::NP, P = C::P, HW = C::HW;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  volatile int32_t *sh = reinterpret_cast<volatile int32_t *>(smem + C::SH_OFF);  // scratch int, abort

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t *cnt = reinterpret_cast<int32_t *>(smem + C::CNT_OFF);
  if (tid == 0) {
    for (int i = 0; i < NP * R; ++i) {
      mbar_init(&full[i], 1);
      cnt[i] = 0;
    }
    fence_mbar_init();
    sh[1] = 0;
    sh[2] = 0;  // length of the merge list
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
  const int64_t CT = gridDim.x, cta = blockIdx.x;

  if (nch == 0) {  // nothing to attend to: every row is zero
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
  // chunk indices fit in 32 bits (the host checks U * ceil(S / 32) < 2^31)
  const bool ragged = VARLEN && a.B <= kMaxRows;
  const int UH = a.Hkv * a.nhc;  // units per batch row
  int32_t *pfx = reinterpret_cast<int32_t *>(smem + C::PFX_OFF);  // pfx[b]: first chunk of row b
  if (ragged) {  // block scan of the rows' chunk counts, rows [b0, b1) per thread
    const int per = (a.B + C::THREADS - 1) / C::THREADS;
    const int b0 = min(a.B, tid * per), b1 = min(a.B, b0 + per);
    int sum = 0;
    for (int b = b0; b < b1; ++b) sum += UH * ((row_kv(a, b) + CS - 1) / CS);
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    int32_t *wsum = pfx + kMaxRows + 1;
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
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
    for (int64_t u = cta; u < U; u += CT) {
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
  const int c_begin = static_cast<int>(range_start(cta, W, CT)), c_end = static_cast<int>(range_start(cta + 1, W, CT));
  if (c_begin >= c_end) return;  // more CTAs than chunks

  // ---- this warp's pipeline pi and its chunks: c_begin + pi + k * NP for k in [0, nk),
  // chunk k in buffer k % R of the pipeline; member pm takes heads [pm * HW, pm * HW + HW)
  const int pi = warp / P, pm = warp % P;
  const int nk = c_begin + pi < c_end ? (c_end - 1 - c_begin - pi) / NP + 1 : 0;
  // lane 0 only: start the copies of the warp's chunk k (flattened index idx)
  auto issue = [&](int idx, int k) {
    const int uu = unit_of(idx);
    const int s0 = (idx - ustart(uu)) * CS;
    const int64_t bhk = uu / a.nhc;  // = b * Hkv + hk
    const int kvu = VARLEN ? row_kv(a, static_cast<int>(bhk / a.Hkv)) : kv;
    const int n = max(0, min(CS, kvu - s0));
    const int n16 = (n + 15) & ~15;  // S % 16 == 0 keeps this inside the slab
    uint8_t *buf = smem + (pi * R + k % R) * C::CHUNK;
    uint64_t *bar = full + pi * R + k % R;
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(n16) * (2 * CB + 10) + (a.mask ? 4u * n16 : 0u));
    if (n16 > 0) {  // 0 bytes: the expect_tx above is a plain arrival
      const uint64_t pol = policy_evict_first();
      const int64_t row = bhk * a.S + s0;
      bulk_g2s_hint(buf + C::K_OFF, a.k + row * CB, n16 * CB, bar, pol);
      bulk_g2s_hint(buf + C::V_OFF, a.v + row * CB, n16 * CB, bar, pol);
      bulk_g2s(buf + C::KS_OFF, a.ks + row, n16 * 4, bar);
      bulk_g2s(buf + C::VS_OFF, a.vs + row, n16 * 4, bar);
      bulk_g2s(buf + C::KZ_OFF, a.kz + row, n16, bar);
      bulk_g2s(buf + C::VZ_OFF, a.vz + row, n16, bar);
      if (a.mask) bulk_g2s(buf + C::M_OFF, a.mask + s0, n16 * 4, bar);
    }
  };
  if (lane == 0 && pm == 0)
    for (int k = 0; k < min(R, nk); ++k) issue(c_begin + pi + k * NP, k);

  const int u_first = unit_of(c_begin), u_last = unit_of(c_end - 1);  // the CTA's units
  const int g = lane / L, sub = lane % L;
  const int own = g + NG * sub;  // this lane's slot within the chunk after the reduce-scatter
  float *wbuf = reinterpret_cast<float *>(smem + C::WBUF_OFF) + warp * 32 * 4;

  uint32_t qhi[HW][4], qlo[HW][4];
  int nsum[HW];
  float escale[HW];
  float m[HW], lsum[HW], corr[HW];  // corr: sum of p * v_scale * (128 + v_zp), see kWScale
  float2 o2[HW][8];

  // warps 0 .. HC-1: head `warp` of unit u onto the fixed-point grid, into q slot `slot`
  //   n = rne(q * sm_scale * log2e / 2^E), |n| <= 32767, E per head; stored as the
  //   high and low bytes of n, four dims per word in the order the dp4a lanes read
  auto convert_q = [&](int u, int slot) {
    if (warp >= HC) return;
    const int h = warp;
    const int hc = u % a.nhc;
    const int64_t bhk = u / a.nhc;
    const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
    const uint16_t *qg = a.q + (static_cast<int64_t>(b) * a.Hq + hk * a.G + hc * HC + h) * D;
    constexpr int NWD = D / 4;                 // words of one head
    constexpr int PER = (NWD + 31) / 32;       // words per lane
    float x[PER][4];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int wd = lane + 32 * i, sb = wd >> 2, kk = wd & 3;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // byte j of word kk of lane sb pairs with the code of dim 16 sb + (4 kk + j); unpacked
        // TQ4 nibbles come as (0,2,4,6), (1,3,5,7), (8,10,12,14), (9,11,13,15)
        const int dim = sb * 16 + (C::Q4 ? (kk >> 1) * 8 + (kk & 1) + 2 * j : 4 * kk + j);
        x[i][j] = wd < NWD ? __uint_as_float(static_cast<uint32_t>(qg[dim]) << 16) * a.qscale : 0.0f;
        amax = fmaxf(amax, fabsf(x[i][j]));
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // step 2^E with amax / 2^E < 2^15: E = floor(log2 amax) + 1 - 15
    int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127 + 1 - 15;
    E = E < -126 ? -126 : E;
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - E) << 23);  // 2^-E (E in [-126, 113])
    uint32_t *qs = reinterpret_cast<uint32_t *>(smem + C::Q_OFF) + (slot * HC + h) * 2 * NWD;
    int s = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int wd = lane + 32 * i;
      uint32_t hw = 0, lw = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int n = __float2int_rn(x[i][j] * inv);
        n = n > 32767 ? 32767 : (n < -32767 ? -32767 : n);
        s += n;
        hw |= (static_cast<uint32_t>(n >> 8) & 0xFFu) << (8 * j);
        lw |= (static_cast<uint32_t>(n) & 0xFFu) << (8 * j);
      }
      if (wd < NWD) {
        qs[wd] = hw;
        qs[NWD + wd] = lw;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      int32_t *meta = reinterpret_cast<int32_t *>(smem + C::QMETA_OFF) + (slot * HC + h) * 2;
      meta[0] = s;
      meta[1] = static_cast<int32_t>(static_cast<uint32_t>(127 + E) << 23);  // 2^E as float bits
    }
  };
  // every lane: its slices of q slot `slot`, fresh softmax state
  auto load_q = [&](int slot) {
#pragma unroll
    for (int h = 0; h < HW; ++h) {
      const uint32_t *qs = reinterpret_cast<const uint32_t *>(smem + C::Q_OFF) + (slot * HC + pm * HW + h) * (D / 2);
      const uint4 hw = *reinterpret_cast<const uint4 *>(qs + sub * 4);
      const uint4 lw = *reinterpret_cast<const uint4 *>(qs + D / 4 + sub * 4);
      qhi[h][0] = hw.x; qhi[h][1] = hw.y; qhi[h][2] = hw.z; qhi[h][3] = hw.w;
      qlo[h][0] = lw.x; qlo[h][1] = lw.y; qlo[h][2] = lw.z; qlo[h][3] = lw.w;
      const int2 meta = *reinterpret_cast<const int2 *>(smem + C::QMETA_OFF + (slot * HC + pm * HW + h) * 8);
      nsum[h] = meta.x;
      escale[h] = __int_as_float(meta.y);
      m[h] = -INFINITY;
      lsum[h] = 0.0f;
      corr[h] = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) o2[h][j] = make_float2(0.0f, 0.0f);
    }
  };

  // this warp's state: merge the NG lane groups (shuffles), then lane group 0
  // writes (O, m, l, corr) for the warp: O at o_dst[h * D + d], the rest at ml_dst[h * 4]
  auto publish = [&](float *o_dst, float *ml_dst) {
#pragma unroll
    for (int h = 0; h < HW; ++h) {
#pragma unroll
      for (int o = L / 2; o >= 1; o >>= 1) {
        lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
        corr[h] += __shfl_xor_sync(0xffffffffu, corr[h], o);
      }
#pragma unroll
      for (int o = L; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[h], o);
        const float lo = __shfl_xor_sync(0xffffffffu, lsum[h], o);
        const float co = __shfl_xor_sync(0xffffffffu, corr[h], o);
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
        corr[h] = corr[h] * fs + co * fo;
        m[h] = M;
      }
    }
    if (g == 0) {
#pragma unroll
      for (int h = 0; h < HW; ++h) {
        float4 *dst = reinterpret_cast<float4 *>(o_dst + h * D + sub * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dst[k] = make_float4(o2[h][2 * k].x, o2[h][2 * k].y, o2[h][2 * k + 1].x, o2[h][2 * k + 1].y);
        if (sub == 0) *reinterpret_cast<float4 *>(ml_dst + h * 4) = make_float4(m[h], lsum[h], corr[h], 0.0f);
      }
    }
  };

  // all threads: combine the warp states of unit u in pipeline order; the state of
  // head h is held by member h / HW of every pipeline: warp (pi, pm)'s O at
  // o_base + pi * p_stride + pm * m_stride (+ hh * D + d), its (m, l, corr) at
  // ml_base + the same offsets (+ hh * 4).  Write the rows, or this CTA's partial
  // when other CTAs share the unit.
  auto combine = [&](int u, const float *o_base, const float *ml_base, int p_stride, int m_stride) {
    const int64_t CTn = gridDim.x;
    const bool alone = cta_of(ustart(u), W, CTn) == cta_of(ustart(u) + ulen(u) - 1, W, CTn);
    const int hc = u % a.nhc;
    const int64_t bhk = u / a.nhc;
    const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
    uint16_t *orow = a.out + (static_cast<int64_t>(b) * a.Hq + hk * a.G + hc * HC) * D;
    const int64_t rec = 2 * static_cast<int64_t>(blockIdx.x) + (u == u_first ? 0 : 1);
    for (int e = tid; e < HC * D; e += C::THREADS) {
      const int h = e / D, d = e - h * D;
      const int off = (h / HW) * m_stride;
      const int hh = h % HW;
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < NP; ++q) M = fmaxf(M, ml_base[q * p_stride + off + hh * 4]);
      float Lt = 0.0f, O = 0.0f;
      if (M != -INFINITY) {
#pragma unroll
        for (int q = 0; q < NP; ++q) {
          const float4 mlc = *reinterpret_cast<const float4 *>(ml_base + q * p_stride + off + hh * 4);
          const float f = mlc.x == -INFINITY ? 0.0f : ex2(mlc.x - M);
          Lt = fmaf(f, mlc.y, Lt);
          O = fmaf(f, fmaf(o_base[q * p_stride + off + hh * D + d], kOScale, -mlc.z), O);
        }
      }
      if (alone) {
        const float r = Lt > 0.0f ? O / Lt : 0.0f;
        orow[e] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
      } else {
        a.ws_o[(rec * HC + h) * D + d] = O;
        if (d == 0) *reinterpret_cast<float2 *>(a.ws_ml + (rec * HC + h) * 2) = make_float2(M, Lt);
      }
    }
  };

  // owner records of the first (slot 0) and last (slot 1) unit when split:
  // owner o's partial is record 2 c + (u is c's first unit ? 0 : 1), c = its CTA
  int32_t *recs_s = reinterpret_cast<int32_t *>(smem + C::RECS_OFF);
  auto owners_of = [&](int u, int64_t &cf) {
    const int64_t CTn = gridDim.x;
    cf = cta_of(ustart(u), W, CTn);
    const int64_t cl = cta_of(ustart(u) + ulen(u) - 1, W, CTn);
    return cf == cl ? 1 : (W >= CTn ? static_cast<int>(cl - cf + 1) : ulen(u));  // W < CTn: one chunk per CTA
  };
  // returns the owner count; `first` gets the unit's first owner CTA, which names its merge counter
  auto stage_owners = [&](int u, int slot, int &first) {
    int64_t cf;
    const int owners = owners_of(u, cf);
    first = static_cast<int>(cf);
    const int64_t CTn = gridDim.x;
    for (int o = tid; o < owners && owners > 1; o += C::THREADS) {
      const int64_t c = W >= CTn ? cf + o : cta_of(ustart(u) + o, W, CTn);
      recs_s[slot * kMaxCtas + o] =
          static_cast<int32_t>(2 * c + (u == unit_of(static_cast<int>(range_start(c, W, CTn))) ? 0 : 1));
    }
    return owners;
  };

  // all threads: merge the partials of split unit u (records in slot `slot`) in owner order
  auto merge_unit = [&](int u, int slot, int owners) {
    const int32_t *recs = recs_s + slot * kMaxCtas;
    const int hc = u % a.nhc;
    const int64_t bhk = u / a.nhc;
    const int hk = static_cast<int>(bhk % a.Hkv), b = static_cast<int>(bhk / a.Hkv);
    uint16_t *orow = a.out + (static_cast<int64_t>(b) * a.Hq + hk * a.G + hc * HC) * D;
    for (int e = tid; e < HC * D; e += C::THREADS) {
      const int h = e / D, d = e - h * D;
      float M = -INFINITY, Lt = 0.0f, O = 0.0f;
      for (int o0 = 0; o0 < owners; o0 += 8) {  // eight owners' loads in flight at once
        float2 ml[8];
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (o0 + t < owners) {
            const int64_t r = static_cast<int64_t>(recs[o0 + t]) * HC + h;
            ml[t] = __ldcg(reinterpret_cast<const float2 *>(a.ws_ml + r * 2));
            v[t] = __ldcg(a.ws_o + r * D + d);
          } else {
            ml[t] = make_float2(-INFINITY, 0.0f);
            v[t] = 0.0f;
          }
        }
        float Mn = M;
#pragma unroll
        for (int t = 0; t < 8; ++t) Mn = fmaxf(Mn, ml[t].x);
        if (Mn == -INFINITY) continue;
        const float fo = M == -INFINITY ? 0.0f : ex2(M - Mn);
        Lt *= fo;
        O *= fo;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float f = ml[t].x == -INFINITY ? 0.0f : ex2(ml[t].x - Mn);
          Lt = fmaf(f, ml[t].y, Lt);
          O = fmaf(f, v[t], O);
        }
        M = Mn;
      }
      const float r = Lt > 0.0f ? O / Lt : 0.0f;
      orow[e] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    }
  };

  // ---- the CTA's units in order.  With at most two (a unit spans more chunks than
  // a CTA range) no warp waits for another until the end: the first unit's warp
  // states go to the scratch, the last unit's to each warp's own (then idle) ring.
  // With more, every unit closes with two CTA barriers.
  const bool deferred = u_last - u_first <= 1;
  float *oscr = reinterpret_cast<float *>(smem + C::OSCR_OFF);
  constexpr int kRingStride = R * C::CHUNK / 4;  // floats from one pipeline's ring to the next
  int cf0 = 0, cf1 = 0;
  const int own0 = stage_owners(u_first, 0, cf0);
  const int own1 = u_last != u_first ? stage_owners(u_last, 1, cf1) : 1;
  if (deferred) {
    convert_q(u_first, 0);
    if (u_last != u_first) convert_q(u_last, 1);
  }
  __syncthreads();  // q slots and owner records written
  int k = 0;
  for (int u = u_first; u <= u_last; ++u) {
    if (ragged && ulen(u) == 0) continue;  // an empty row between the CTA's first and last unit
    if (!deferred) {
      convert_q(u, 0);
      __syncthreads();  // q slot written; the previous unit's combine has read the scratch
    }
    load_q(deferred && u != u_first ? 1 : 0);
    const int kv_u = VARLEN ? row_kv(a, static_cast<int>(u / a.nhc / a.Hkv)) : kv;
    const int seg_end = min(c_end, ustart(u) + ulen(u));
    for (; k < nk; ++k) {
      const int idx = c_begin + pi + k * NP;
      if (idx >= seg_end) break;
      const uint8_t *stage = smem + (pi * R + k % R) * C::CHUNK;
      const bool ok = wait_or_abort(full + pi * R + k % R, static_cast<uint32_t>(k / R) & 1u, sh + 1);
      if (!ok && lane == 0) {
        report(a.err, KVQ_ERR_TIMEOUT);
        sh[1] = 1;
      }
      const int s0 = (idx - ustart(u)) * CS;
      if (ok && s0 < kv_u) {
        // ---- q . k on dp4a for the L slots of this lane group (slot = g + NG*jj)
        int part[L][HW];
#pragma unroll
        for (int jj = 0; jj < L; ++jj) {
          const int sl = g + NG * jj;
          if constexpr (C::Q4) {
            const uint2 cw = *reinterpret_cast<const uint2 *>(stage + C::K_OFF + sl * CB + sub * 8);
            uint4 c;
            unpack_nibbles(cw.x, c.x, c.y);
            unpack_nibbles(cw.y, c.z, c.w);
#pragma unroll
            for (int h = 0; h < HW; ++h) {
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
            for (int h = 0; h < HW; ++h) {
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
            for (int h = 0; h < HW; ++h) {
              const int keep = upper ? part[j + o][h] : part[j][h];
              const int send = upper ? part[j][h] : part[j + o][h];
              part[j][h] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        // ---- scores (log2 domain) for this lane's slot
        const bool valid = s0 + own < kv_u;
        const int kzp = static_cast<int8_t>(stage[C::KZ_OFF + own]);
        const float ksc = reinterpret_cast<const float *>(stage + C::KS_OFF)[own];
        const float vsc = reinterpret_cast<const float *>(stage + C::VS_OFF)[own];
        const float zc = static_cast<float>(128 + static_cast<int8_t>(stage[C::VZ_OFF + own]));
        const float madd = a.mask ? reinterpret_cast<const float *>(stage + C::M_OFF)[own] * kLog2e : 0.0f;
        float sc[HW];
        bool need = false;
#pragma unroll
        for (int h = 0; h < HW; ++h) {
          // exact: |sum n (c - zp)| < 2^31 for D <= 256 (computed modulo 2^32)
          const int dz = static_cast<int>(static_cast<uint32_t>(part[0][h]) -
                                          static_cast<uint32_t>(kzp) * static_cast<uint32_t>(nsum[h]));
          sc[h] = valid ? fmaf(static_cast<float>(dz), escale[h] * ksc, madd) : -INFINITY;
          need |= sc[h] > m[h] + kRescaleThreshold;
        }
        // the group maximum is only needed when some score would overflow the lazy bound
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            float mt = sc[h];
#pragma unroll
            for (int o = L / 2; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
            const float mnew = fmaxf(m[h], mt);
            if (mnew > m[h] + kRescaleThreshold) {
              const float alpha = m[h] == -INFINITY ? 0.0f : ex2(m[h] - mnew);
              lsum[h] *= alpha;
              corr[h] *= alpha;
              const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
              for (int j = 0; j < 8; ++j) o2[h][j] = __fmul2_rn(o2[h][j], al2);
              m[h] = mnew;
            }
          }
        }
        float wv[4];
#pragma unroll
        for (int h = 0; h < HW; ++h) {
          const float p = sc[h] == -INFINITY ? 0.0f : ex2(sc[h] - m[h]);
          lsum[h] += p;
          const float wt = p > 0.0f ? p * vsc : 0.0f;
          corr[h] = fmaf(wt, zc, corr[h]);
          wv[h] = wt * kWScale;
        }
#pragma unroll
        for (int h = HW; h < 4; ++h) wv[h] = 0.0f;
        *reinterpret_cast<float4 *>(wbuf + own * 4) = make_float4(wv[0], wv[1], wv[2], wv[3]);
        __syncwarp();
        // ---- p . v over the same L slots: code + 128 as the subnormal float (code + 128) * 2^-149
#pragma unroll
        for (int jj = 0; jj < L; ++jj) {
          const int sl = g + NG * jj;
          const float4 w4 = *reinterpret_cast<const float4 *>(wbuf + sl * 4);
          const float wj[4] = {w4.x, w4.y, w4.z, w4.w};
          uint32_t x[4], y[4];  // dims (4i .. 4i+3) of the lane's 16: bytes of x[i] (low dims) or x/y pairs
          if constexpr (C::Q4) {  // element 2i in the low nibble of byte i
            const uint2 cw = *reinterpret_cast<const uint2 *>(stage + C::V_OFF + sl * CB + sub * 8);
            x[0] = (cw.x & 0x0F0F0F0Fu) | 0x80808080u;         // dims 0, 2, 4, 6
            y[0] = ((cw.x >> 4) & 0x0F0F0F0Fu) | 0x80808080u;  // dims 1, 3, 5, 7
            x[1] = (cw.y & 0x0F0F0F0Fu) | 0x80808080u;         // dims 8, 10, 12, 14
            y[1] = ((cw.y >> 4) & 0x0F0F0F0Fu) | 0x80808080u;  // dims 9, 11, 13, 15
          } else {
            const uint4 c = *reinterpret_cast<const uint4 *>(stage + C::V_OFF + sl * D + sub * 16);
            x[0] = c.x ^ 0x80808080u;
            x[1] = c.y ^ 0x80808080u;
            x[2] = c.z ^ 0x80808080u;
            x[3] = c.w ^ 0x80808080u;
          }
          float2 vv2[8];
#pragma unroll
          for (int k2 = 0; k2 < 8; ++k2) {
            uint32_t lo, hi;
            if constexpr (C::Q4) {  // vv2[k2] = dims (2 k2, 2 k2 + 1): byte k2 % 4 of the even / odd word
              const uint32_t ev = x[k2 >> 2], od = y[k2 >> 2];
              lo = __byte_perm(ev, 0u, 0x4440u + (k2 & 3));
              hi = __byte_perm(od, 0u, 0x4440u + (k2 & 3));
            } else {  // vv2[k2] = bytes 2 (k2 % 2), 2 (k2 % 2) + 1 of word k2 / 2
              const uint32_t wd = x[k2 >> 1];
              lo = __byte_perm(wd, 0u, 0x4440u + 2 * (k2 & 1));
              hi = __byte_perm(wd, 0u, 0x4441u + 2 * (k2 & 1));
            }
            vv2[k2] = make_float2(__uint_as_float(lo), __uint_as_float(hi));
          }
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            const float2 w2 = make_float2(wj[h], wj[h]);
#pragma unroll
            for (int j = 0; j < 8; ++j) o2[h][j] = __ffma2_rn(w2, vv2[j], o2[h][j]);
          }
        }
      }
      __syncwarp();  // the buffer and wbuf are free again (for this warp)
      if (lane == 0 && (P == 1 || done_count(cnt + pi * R + k % R) == P - 1)) {
        if (P > 1) cnt[pi * R + k % R] = 0;  // the pipeline's last warp refills the buffer
        if (k + R < nk && !sh[1]) issue(idx + R * NP, k + R);
      }
    }
    if (deferred && u == u_last && u_last != u_first) {
      // the rings hold the last unit's state once every warp is past its chunks
      __syncthreads();
      float *rw = reinterpret_cast<float *>(smem + pi * R * C::CHUNK + pm * C::PUBW);
      publish(rw, rw + HW * D);
    } else {
      float *ow = oscr + warp * (C::PUBW / 4);
      publish(ow, ow + HW * D);
      if (!deferred) {
        __syncthreads();
        combine(u, oscr, oscr + HW * D, P * C::PUBW / 4, C::PUBW / 4);
      }
    }
  }
  if (deferred) {
    __syncthreads();
    combine(u_first, oscr, oscr + HW * D, P * C::PUBW / 4, C::PUBW / 4);
    if (u_last != u_first)
      combine(u_last, reinterpret_cast<const float *>(smem), reinterpret_cast<const float *>(smem) + HW * D,
              kRingStride, C::PUBW / 4);
  }
  __syncthreads();  // every partial is written; the scratch is free for the merge

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
  if (sh[2]) merge_unit(u_first, 0, own0);
  if (sh[3]) merge_unit(u_last, 1, own1);
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
int head_chunk(int G) { return G % 4 == 0 ? 4 : (G % 3 == 0 ? 3 : (G % 2 == 0 ? 2 : 1)); }

// Pipelines and warps per pipeline: with an even head chunk two warps share a
// pipeline and take half the heads each (fewer registers per warp, so more
// warps per SM to hide latency); D = 256 chunks are 16.5 KB, so fewer
// pipelines.  The ring takes what shared memory is left (at most 4 deep).
template <int D, int HC, bool Q4>
struct Tune {
  static constexpr int P = HC % 2 == 0 ? 2 : 1;
  static constexpr int HW = HC / P;
  static constexpr int NP = D == 256 ? (P == 2 ? (HC == 4 ? 5 : 6) : 5) : (P == 2 ? 8 : 11);
  static constexpr int NW = NP * P;
  static constexpr int CHUNK = 64 * (Q4 ? D / 2 : D) + 448;
  static constexpr int PUBW = HW * D * 4 + HW * 16;
  static constexpr int FIXED =
      NW * 512 + NW * PUBW + NP * 8 * 12 + 64 + 4 * HC * D + 16 * HC + 8 * kMaxCtas + 4 * (kMaxRows + 33);
  static constexpr int RMAX = (232448 - FIXED) / (NP * CHUNK);
  static constexpr int R = RMAX > 4 ? 4 : RMAX;
  static_assert(R >= 2, "ring depth");
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

template <class C, bool VARLEN>
struct KernelTag {};  // names one decode_kernel instantiation for ensure_smem

template <int D, int HC, bool Q4>
int launch_decode(DecodeArgs a, int ctas, cudaStream_t stream) {
  using T = Tune<D, HC, Q4>;
  using C = Cfg<D, HC, T::NP, T::P, T::R, Q4>;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  {
    cudaLaunchConfig_t dc = {};
    dc.gridDim = dim3(static_cast<unsigned>(ctas));
    dc.blockDim = dim3(C::THREADS);
    dc.dynamicSmemBytes = C::SMEM;
    dc.stream = stream;
    dc.attrs = attr;
    dc.numAttrs = 1;
    cudaError_t e;
    if (a.kv_per_batch) {
      if (const int st = ensure_smem<KernelTag<C, true>>(decode_kernel<C, true>, C::SMEM)) return st;
      e = cudaLaunchKernelEx(&dc, decode_kernel<C, true>, a);
    } else {
      if (const int st = ensure_smem<KernelTag<C, false>>(decode_kernel<C, false>, C::SMEM)) return st;
      e = cudaLaunchKernelEx(&dc, decode_kernel<C, false>, a);
    }
    if (e != cudaSuccess) return KVQ_ECUDA;
  }
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
  return ws_layout(D, hc, sm_count()).total;
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
  if (static_cast<int64_t>(B) * Hkv * nhc * ((S + 31) / 32) >= INT32_MAX) return KVQ_EUNSUPPORTED;
  const int ctas = sm_count();
  const WsLayout w = ws_layout(D, hc, ctas);
  if (ctas > kMaxCtas) return KVQ_EUNSUPPORTED;  // owner records staged per unit
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
  a.ws_cnt = reinterpret_cast<int32_t *>(ws + w.cnt);
  a.err = err_word;
  a.S = S;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = G;
  a.nhc = nhc;
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

extern "C" int kvq_decode_static_reset(void *stream) {
  void *scratch = nullptr;
  const int st = kvq::static_scratch_address(&scratch);
  if (st != KVQ_OK) return st;
  if (cudaMemsetAsync(scratch, 0, KVQ_STATIC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVQ_ECUDA;
  return KVQ_OK;
}
