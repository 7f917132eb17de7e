// kvq_prefill.cu -- chunked-prefill attention entry points over the int8 cache.
#include "kvq_common.cuh"
#include "kvq_prefill_tc.cuh"

namespace {
int prefill_impl(const void *q, int B, int Hq, int Hkv, int Lq, int D, const int8_t *k, const float *k_scale,
                 const int8_t *k_zp, const int8_t *v, const float *v_scale, const int8_t *v_zp, int64_t S,
                 const int32_t *kv_len, int kv_per_batch, const float *mask, int64_t mask_bstride, int is_causal,
                 int mask_is_causal, float sm_scale, void *out, int32_t *err_word, void *stream) {
  using namespace kvq;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S > INT32_MAX || Lq <= 0 || Lq > S)
    return KVQ_EINVAL;
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
  if (Hq > 65535 || B > 65535) return KVQ_EUNSUPPORTED;
  tc::PrefillArgs a;
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
  a.err = err_word;
  a.S = S;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.Lq = Lq;
  a.nhc = 1;
  a.is_causal = is_causal ? 1 : 0;
  a.mask_is_causal = mask_is_causal ? 1 : 0;
  a.qscale = sm_scale * 1.4426950408889634f;
  a.wait_ns = wait_limit_ns();
  a.ks8 = nullptr;
  a.vs8 = nullptr;
  return tc::dispatch_prefill_mode<0>(a, D, static_cast<cudaStream_t>(stream));
}
}  // namespace

extern "C" int kvq_prefill_attn(const void *q, int B, int Hq, int Hkv, int Lq, int D, const int8_t *k,
                                const float *k_scale, const int8_t *k_zp, const int8_t *v, const float *v_scale,
                                const int8_t *v_zp, int64_t S, const int32_t *kv_len, const float *mask,
                                int is_causal, int mask_is_causal, float sm_scale, void *out, int32_t *err_word,
                                void *stream) {
  return prefill_impl(q, B, Hq, Hkv, Lq, D, k, k_scale, k_zp, v, v_scale, v_zp, S, kv_len, 0, mask, 0, is_causal,
                      mask_is_causal, sm_scale, out, err_word, stream);
}

extern "C" int kvq_prefill_attn_varlen(const void *q, int B, int Hq, int Hkv, int Lq, int D, const int8_t *k,
                                       const float *k_scale, const int8_t *k_zp, const int8_t *v,
                                       const float *v_scale, const int8_t *v_zp, int64_t S, const int32_t *kv_lens,
                                       const float *mask, int64_t mask_batch_stride, int is_causal,
                                       int mask_is_causal, float sm_scale, void *out, int32_t *err_word,
                                       void *stream) {
  return prefill_impl(q, B, Hq, Hkv, Lq, D, k, k_scale, k_zp, v, v_scale, v_zp, S, kv_lens, 1, mask,
                      mask_batch_stride, is_causal, mask_is_causal, sm_scale, out, err_word, stream);
}
