// kvq_prefill_simt.cuh -- CUDA-core chunked-prefill attention over the int8
// cache.  Straightforward and exact in structure: used for shapes the tensor
// core path does not take, and as its in-library cross-check.
//
// Grid (ceil(Lq / 16), Hq, B); 4 warps, 4 query rows per warp.  K/V code tiles
// of 64 slots are staged in shared memory; each lane scores two slots of a
// tile for one row (full dot over D), the warp keeps that row's online softmax,
// and PV gives each lane D/32 output dims.  The per-tile causal upper bound
// (ExecuTorch PR 20351 commit notes: loop_end = min(kv_len, (kv_len - Lq) +
// max(seq_pos) + 1)) limits the tile loop when mask_is_causal is set; tiles
// past it would be fully masked, so the result is identical either way.
#pragma once

#include <cuda_bf16.h>

#include "kvq_common.cuh"

namespace kvq {
namespace simt {

constexpr int kRowsPerCta = 16;
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
  int B, Hq, Hkv, Lq;
  int is_causal, mask_is_causal;
  float qscale;  // sm_scale * log2(e)
};

template <int D>
__global__ void __launch_bounds__(kThreads) prefill_simt_kernel(const PrefillArgs a) {
  constexpr int DPT = D / 32;             // output dims per lane
  constexpr int kTile = D == 256 ? 32 : 64;
  constexpr int SPL = kTile / 32;         // slots scored per lane
  constexpr int KW = D / 4 + 1;           // padded row length in 32-bit words (bank-conflict free)
  __shared__ uint32_t kt[kTile][KW];
  __shared__ __align__(16) int8_t vt[kTile][D];
  __shared__ float ksc[kTile], vsc[kTile];
  __shared__ int kzs[kTile], vzs[kTile];
  __shared__ float qs[kRowsPerCta][D];
  __shared__ int kv_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = blockIdx.x * kRowsPerCta;
  const int hq = blockIdx.y, b = blockIdx.z;
  const int hk = hq / (a.Hq / a.Hkv);
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + hk;

  if (tid == 0) {
    int kv = *a.kv_len;
    if (kv < a.Lq || kv > a.S) {
      if (blockIdx.x == 0 && hq == 0 && b == 0) report(a.err, KVQ_ERR_KV_LEN_RANGE);
      kv = kv < a.Lq ? a.Lq : static_cast<int>(a.S);
    }
    kv_sh = kv;
  }
  for (int e = tid; e < kRowsPerCta * D; e += kThreads) {
    const int r = e / D, d = e - r * D;
    const int row = r0 + r;
    float qv = 0.0f;
    if (row < a.Lq) {
      const uint16_t bits = a.q[((static_cast<int64_t>(b) * a.Hq + hq) * a.Lq + row) * D + d];
      qv = __uint_as_float(static_cast<uint32_t>(bits) << 16) * a.qscale;
    }
    qs[r][d] = qv;
  }
  __syncthreads();
  const int kv = kv_sh;
  const int last_row = min(r0 + kRowsPerCta, a.Lq) - 1;
  // per-tile causal upper bound over this CTA's rows
  int loop_end = kv;
  if (a.mask_is_causal) loop_end = min(kv, kv - a.Lq + last_row + 1);

  float m[4], l[4], o[4][DPT];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.0f;
#pragma unroll
    for (int i = 0; i < DPT; ++i) o[rr][i] = 0.0f;
  }

  for (int t0 = 0; t0 < loop_end; t0 += kTile) {
    const int n = min(kTile, loop_end - t0);
    __syncthreads();
    for (int e = tid; e < kTile * D / 16; e += kThreads) {
      const int j = e / (D / 16), c = e - j * (D / 16);
      uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (j < n) {
        kk = *reinterpret_cast<const uint4 *>(a.k + (bh * a.S + t0 + j) * D + c * 16);
        vv = *reinterpret_cast<const uint4 *>(a.v + (bh * a.S + t0 + j) * D + c * 16);
      }
      kt[j][c * 4 + 0] = kk.x;
      kt[j][c * 4 + 1] = kk.y;
      kt[j][c * 4 + 2] = kk.z;
      kt[j][c * 4 + 3] = kk.w;
      *reinterpret_cast<uint4 *>(&vt[j][c * 16]) = vv;
    }
    for (int j = tid; j < kTile; j += kThreads) {
      const bool in = j < n;
      ksc[j] = in ? a.ks[bh * a.S + t0 + j] : 0.0f;
      vsc[j] = in ? a.vs[bh * a.S + t0 + j] : 0.0f;
      kzs[j] = in ? a.kz[bh * a.S + t0 + j] : 0;
      vzs[j] = in ? a.vz[bh * a.S + t0 + j] : 0;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr;
      const int row = r0 + r;
      if (row >= a.Lq) continue;  // warp-uniform
      float s[SPL], w[SPL];
      float mt = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < SPL; ++hh) {
        const int j = lane + 32 * hh;
        const int slot = t0 + j;
        bool vis = j < n;
        if (a.is_causal && slot > kv - a.Lq + row) vis = false;
        float dot = 0.0f;
        const float zp = static_cast<float>(kzs[j]);
#pragma unroll 8
        for (int d4 = 0; d4 < D / 4; ++d4) {
          const uint32_t wd = kt[j][d4];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            dot = fmaf(qs[r][4 * d4 + c], static_cast<float>(static_cast<int8_t>(wd >> (8 * c))) - zp, dot);
        }
        float sc = dot * ksc[j];
        if (a.mask && vis) sc += a.mask[static_cast<int64_t>(row) * a.S + slot] * 1.4426950408889634f;
        s[hh] = vis ? sc : -INFINITY;
        mt = fmaxf(mt, s[hh]);
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float mnew = fmaxf(m[rr], mt);
      const float muse = mnew == -INFINITY ? 0.0f : mnew;
      const float alpha = exp2f(m[rr] - muse);
      float ps = 0.0f;
#pragma unroll
      for (int hh = 0; hh < SPL; ++hh) {
        const float p = exp2f(s[hh] - muse);
        ps += p;
        w[hh] = p > 0.0f ? p * vsc[lane + 32 * hh] : 0.0f;
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[rr] = l[rr] * alpha + ps;
      m[rr] = mnew;
#pragma unroll
      for (int i = 0; i < DPT; ++i) o[rr][i] *= alpha;
      for (int j = 0; j < n; ++j) {
        const float wj = __shfl_sync(0xffffffffu, SPL == 1 || j < 32 ? w[0] : w[SPL - 1], j & 31);
        if (wj == 0.0f) continue;  // warp-uniform
        const float zp = static_cast<float>(vzs[j]);
#pragma unroll
        for (int i = 0; i < DPT; ++i) o[rr][i] = fmaf(wj, static_cast<float>(vt[j][lane + 32 * i]) - zp, o[rr][i]);
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int row = r0 + warp * 4 + rr;
    if (row >= a.Lq) continue;
    uint16_t *op = a.out + ((static_cast<int64_t>(b) * a.Hq + hq) * a.Lq + row) * D;
    const float inv = l[rr] > 0.0f ? 1.0f / l[rr] : 0.0f;
#pragma unroll
    for (int i = 0; i < DPT; ++i)
      op[lane + 32 * i] = __bfloat16_as_ushort(__float2bfloat16_rn(l[rr] > 0.0f ? o[rr][i] * inv : 0.0f));
  }
}

template <int D>
int launch_prefill_simt(const PrefillArgs &a, cudaStream_t stream) {
  dim3 grid((a.Lq + kRowsPerCta - 1) / kRowsPerCta, a.Hq, a.B);
  prefill_simt_kernel<D><<<grid, kThreads, 0, stream>>>(a);
  return launch_status();
}

}  // namespace simt
}  // namespace kvq
