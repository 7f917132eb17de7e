// kvq_prefill_block.cu -- chunked-prefill attention over the per-32 block caches
// (kvq_write modes 1-6), on the tcgen05 prefill kernel with block-format
// converters.  The kernel variants of each cache mode are compiled in
// kvq_prefill_e4m3.cu (modes 1, 2), kvq_prefill_e5m2.cu (4, 5) and
// kvq_prefill_fp4_int8.cu (3, 6).
#include "kvq_common.cuh"
#include "kvq_prefill_tc.cuh"

namespace kvq {
namespace tc {
extern template int dispatch_prefill_mode<KVQ_MODE_FP8_E4M3>(const PrefillArgs &, int, cudaStream_t);
extern template int dispatch_prefill_mode<KVQ_MODE_MXFP8>(const PrefillArgs &, int, cudaStream_t);
extern template int dispatch_prefill_mode<KVQ_MODE_MXFP4>(const PrefillArgs &, int, cudaStream_t);
extern template int dispatch_prefill_mode<KVQ_MODE_FP8_E5M2>(const PrefillArgs &, int, cudaStream_t);
extern template int dispatch_prefill_mode<KVQ_MODE_MXFP8_E5M2>(const PrefillArgs &, int, cudaStream_t);
extern template int dispatch_prefill_mode<KVQ_MODE_INT8_SYM>(const PrefillArgs &, int, cudaStream_t);
}  // namespace tc
}  // namespace kvq

extern "C" int kvq_prefill_attn_block(int mode, const void *q, int B, int Hq, int Hkv, int Lq, int D,
                                      const uint8_t *k_codes, const void *k_scales, const uint8_t *v_codes,
                                      const void *v_scales, int64_t S, const int32_t *kv_len, const float *mask,
                                      int is_causal, int mask_is_causal, float sm_scale, void *out,
                                      int32_t *err_word, void *stream) {
  using namespace kvq;
  if (mode < KVQ_MODE_FP8_E4M3 || mode > KVQ_MODE_INT8_SYM) return KVQ_EINVAL;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || S > INT32_MAX || Lq <= 0 || Lq > S)
    return KVQ_EINVAL;
  if (D != 64 && D != 128 && D != 256) return KVQ_EUNSUPPORTED;
  if (S % 16 != 0) return KVQ_EUNSUPPORTED;
  if (B == 0) return KVQ_OK;
  if (!q || !k_codes || !k_scales || !v_codes || !v_scales || !kv_len || !out) return KVQ_EINVAL;
  const void *ptrs[] = {q, k_codes, k_scales, v_codes, v_scales, out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return KVQ_EINVAL;
  if (mask && !aligned16(mask)) return KVQ_EINVAL;
  if (!(sm_scale == sm_scale)) return KVQ_EINVAL;
  if (Hq > 65535 || B > 65535) return KVQ_EUNSUPPORTED;
  const bool f32 = mode == KVQ_MODE_FP8_E4M3 || mode == KVQ_MODE_FP8_E5M2 || mode == KVQ_MODE_INT8_SYM;
  tc::PrefillArgs a{};
  a.q = static_cast<const uint16_t *>(q);
  a.k = reinterpret_cast<const int8_t *>(k_codes);
  a.v = reinterpret_cast<const int8_t *>(v_codes);
  a.ks = f32 ? static_cast<const float *>(k_scales) : nullptr;
  a.vs = f32 ? static_cast<const float *>(v_scales) : nullptr;
  a.ks8 = f32 ? nullptr : static_cast<const uint8_t *>(k_scales);
  a.vs8 = f32 ? nullptr : static_cast<const uint8_t *>(v_scales);
  a.kz = nullptr;
  a.vz = nullptr;
  a.mask = mask;
  a.mask_bstride = 0;
  a.kv_len = kv_len;
  a.kv_per_batch = 0;
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
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (mode) {
    case KVQ_MODE_FP8_E4M3: return tc::dispatch_prefill_mode<KVQ_MODE_FP8_E4M3>(a, D, s);
    case KVQ_MODE_MXFP8: return tc::dispatch_prefill_mode<KVQ_MODE_MXFP8>(a, D, s);
    case KVQ_MODE_MXFP4: return tc::dispatch_prefill_mode<KVQ_MODE_MXFP4>(a, D, s);
    case KVQ_MODE_FP8_E5M2: return tc::dispatch_prefill_mode<KVQ_MODE_FP8_E5M2>(a, D, s);
    case KVQ_MODE_MXFP8_E5M2: return tc::dispatch_prefill_mode<KVQ_MODE_MXFP8_E5M2>(a, D, s);
    default: return tc::dispatch_prefill_mode<KVQ_MODE_INT8_SYM>(a, D, s);
  }
}
