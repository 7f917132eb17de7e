// kvq_decode_blk.cuh -- the launch of the tensor-core decode over a block cache,
// shared by the per-mode translation units.
#pragma once

#include <cstring>

#include "kvq_decode_blk.h"
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace {

template <int MODE>
int decode_blk_run_impl(const BlkCall &c) {
  const int G = c.Hq / c.Hkv;
  const int hc = head_chunk_mma(G);
  const int nhc = G / hc;
  if (static_cast<int64_t>(c.B) * c.Hkv * nhc * ((c.S + 31) / 32) >= INT32_MAX) return KVQ_EUNSUPPORTED;
  if (static_cast<int64_t>(c.B) * c.Hkv * c.S >= INT32_MAX) return KVQ_EUNSUPPORTED;  // TMA row coordinates
  const int ctas = sm_count();
  if (ctas > kMaxCtas) return KVQ_EUNSUPPORTED;
  const WsLayout w = ws_layout(c.D, hc, ctas);
  if (!c.workspace || c.workspace_bytes < w.total || !aligned16(c.workspace)) return KVQ_EINVAL;
  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = static_cast<const uint16_t *>(c.q);
  a.k = reinterpret_cast<const int8_t *>(c.k_codes);
  a.v = reinterpret_cast<const int8_t *>(c.v_codes);
  a.kscl = c.k_scales;
  a.vscl = c.v_scales;
  a.mask = c.mask;
  a.mask_bstride = 0;
  a.kv_len = c.kv_len;
  a.kv_per_batch = 0;
  a.out = static_cast<uint16_t *>(c.out);
  uint8_t *ws = static_cast<uint8_t *>(c.workspace);
  a.ws_cnt = reinterpret_cast<int32_t *>(ws + w.cnt);
  a.ws_ml = reinterpret_cast<float *>(ws + w.ml);
  a.ws_o = reinterpret_cast<float *>(ws + w.o);
  a.err = c.err_word;
  a.S = c.S;
  a.B = c.B;
  a.Hq = c.Hq;
  a.Hkv = c.Hkv;
  a.G = G;
  a.nhc = nhc;
  a.qscale = c.sm_scale * kLog2e;
  a.wait_ns = wait_limit_ns();
  KvMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int64_t rows = static_cast<int64_t>(c.B) * c.Hkv * c.S;
  const int box_rows = c.D <= 128 ? 64 : 32;  // the tensor-core path's chunk (Tune::CS)
  const int row_bytes = MODE == KVQ_MODE_MXFP4 ? c.D / 2 : c.D;  // E2M1: two codes a byte
  if (const int st = make_code_map(&maps.k, c.k_codes, row_bytes, rows, box_rows)) return st;
  if (const int st = make_code_map(&maps.v, c.v_codes, row_bytes, rows, box_rows)) return st;
  return dispatch_blk_mode<MODE>(a, maps, c.D, hc, ctas, c.stream);
}

}  // namespace
}  // namespace kvq
