// kvq_decode.cu -- entry points of the one-query (decode) attention over the int8
// and TQ4 caches: argument checks, the workspace, the static scratch.  The kernel
// is in kvq_decode_kernel.cuh.
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "kvq_decode_kernel.cuh"

extern "C" size_t kvq_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t S) {
  using namespace kvq;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S % 16 != 0) return 0;
  if (D != 64 && D != 128 && D != 256) return 0;
  return ws_bytes(Hq / Hkv, D, sm_count());
}

namespace kvq {
namespace {
int decode_impl(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k, const float *k_scale,
                const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp, int64_t S,
                const int32_t *kv_len, int kv_per_batch, bool q4, const float *mask, int64_t mask_bstride,
                float sm_scale, void *out, void *workspace, size_t workspace_bytes, int32_t *err_word,
                void *stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S > INT32_MAX) return KVQ_EINVAL;
  if (D != 64 && D != 128 && D != 256) return KVQ_EUNSUPPORTED;
  if (S % 16 != 0) return KVQ_EUNSUPPORTED;
  if (B == 0) return KVQ_OK;
  if (!q || !k || !k_scale || !k_zp || !v || !v_scale || !v_zp || !kv_len || !out) return KVQ_EINVAL;
  const void *ptrs[] = {q, k, k_scale, k_zp, v, v_scale, v_zp, out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return KVQ_EINVAL;
  if (mask && !aligned16(mask)) return KVQ_EINVAL;
  if (mask_bstride < 0 || mask_bstride % 4 != 0) return KVQ_EINVAL;  // keeps every row's mask 16-byte aligned
  if (!(sm_scale == sm_scale)) return KVQ_EINVAL;
  const int G = Hq / Hkv;
  const bool q4_mma = q4 && D >= 128;  // TQ4 on the tensor cores; at D = 64 on the CUDA cores
  const int hc = q4 && !q4_mma ? head_chunk_simt(G) : head_chunk_mma(G);
  const int nhc = G / hc;
  if (static_cast<int64_t>(B) * Hkv * nhc * ((S + 31) / 32) >= INT32_MAX) return KVQ_EUNSUPPORTED;
  // TMA row coordinates are 32-bit
  if ((!q4 || q4_mma) && static_cast<int64_t>(B) * Hkv * S >= INT32_MAX) return KVQ_EUNSUPPORTED;
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
  a.mask_bstride = mask_bstride;
  a.kv_len = kv_len;
  a.kv_per_batch = kv_per_batch;
  a.out = static_cast<uint16_t *>(out);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  a.ws_cnt = reinterpret_cast<int32_t *>(ws + w.cnt);
  a.ws_ml = reinterpret_cast<float *>(ws + w.ml);
  a.ws_o = reinterpret_cast<float *>(ws + w.o);
  a.err = err_word;
  a.S = S;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = G;
  a.nhc = nhc;
  a.qscale = sm_scale * kLog2e;
  a.wait_ns = wait_limit_ns();
  KvMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q4 && !q4_mma) return dispatch_q4<64>(a, maps, hc, ctas, s);
  const int64_t rows = static_cast<int64_t>(B) * Hkv * S;
  const int box_rows = D <= 128 ? 64 : 32;  // the tensor-core path's chunk (Tune::CS)
  const int row_bytes = q4 ? D / 2 : D;     // TQ4: two codes a byte
  if (const int st = make_code_map(&maps.k, k, row_bytes, rows, box_rows)) return st;
  if (const int st = make_code_map(&maps.v, v, row_bytes, rows, box_rows)) return st;
  if (q4) return D == 128 ? dispatch_q4mma<128>(a, maps, hc, ctas, s) : dispatch_q4mma<256>(a, maps, hc, ctas, s);
  switch (D) {
    case 64: return dispatch_mma<64>(a, maps, hc, ctas, s);
    case 128: return dispatch_mma<128>(a, maps, hc, ctas, s);
    default: return dispatch_mma<256>(a, maps, hc, ctas, s);
  }
}
}  // namespace
}  // namespace kvq

extern "C" int kvq_decode_attn(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k, const float *k_scale,
                               const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp,
                               int64_t S, const int32_t *kv_len, const float *mask, float sm_scale, void *out,
                               void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream) {
  return kvq::decode_impl(q, B, Hq, Hkv, D, k, k_scale, k_zp, v, v_scale, v_zp, S, kv_len, 0, false, mask, 0,
                          sm_scale, out, workspace, workspace_bytes, err_word, stream);
}

extern "C" int kvq_decode_attn_tq4(const void *q, int B, int Hq, int Hkv, int D, const uint8_t *k,
                                   const float *k_scale, const uint8_t *k_zp, const uint8_t *v, const float *v_scale,
                                   const uint8_t *v_zp, int64_t S, const int32_t *kv_len, const float *mask,
                                   float sm_scale, void *out, void *workspace, size_t workspace_bytes,
                                   int32_t *err_word, void *stream) {
  return kvq::decode_impl(q, B, Hq, Hkv, D, reinterpret_cast<const int8_t *>(k), k_scale,
                          reinterpret_cast<const int8_t *>(k_zp), reinterpret_cast<const int8_t *>(v), v_scale,
                          reinterpret_cast<const int8_t *>(v_zp), S, kv_len, 0, true, mask, 0, sm_scale, out,
                          workspace, workspace_bytes, err_word, stream);
}

extern "C" int kvq_decode_attn_varlen(const void *q, int B, int Hq, int Hkv, int D, const int8_t *k,
                                      const float *k_scale, const int8_t *k_zp, const int8_t *v,
                                      const float *v_scale, const int8_t *v_zp, int64_t S, const int32_t *kv_lens,
                                      const float *mask, int64_t mask_batch_stride, float sm_scale, void *out,
                                      void *workspace, size_t workspace_bytes, int32_t *err_word, void *stream) {
  return kvq::decode_impl(q, B, Hq, Hkv, D, k, k_scale, k_zp, v, v_scale, v_zp, S, kv_lens, 1, false, mask,
                          mask_batch_stride, sm_scale, out, workspace, workspace_bytes, err_word, stream);
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
