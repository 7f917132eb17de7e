// kvq_sink.cu -- attention-sink / ring slot assignment and additive mask.
//
// ExecuTorch PR 24473, Summary: CachePositionsManagerWithSink hands out the
// write slots of a cache with a pinned sink prefix followed by a ring (the
// ring cache is sink_size = 0), and _create_causal_mask_for_attention_sink
// builds the additive float mask that the quantized SDPA then uses.  Both read
// the position from device memory, so a decode step stays capturable.
#include "kvq_common.cuh"

namespace kvq {
namespace {

__global__ void sink_plan_kernel(const int32_t *__restrict__ input_pos, int B, int T, int sink, int64_t S,
                                 int32_t *__restrict__ slot_mapping, int32_t *__restrict__ slot_pos,
                                 int32_t *__restrict__ kv_len, int32_t *err) {
  const int64_t p0 = *input_pos;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (p0 < 0) {
    if (t < T)
      for (int b = 0; b < B; ++b) slot_mapping[static_cast<int64_t>(b) * T + t] = -1;
    if (t == 0) {
      *kv_len = 0;
      report(err, KVQ_ERR_INPUT_POS);
    }
    return;
  }
  if (t < T) {
    const int64_t p = p0 + t;
    const int64_t slot = p < sink ? p : sink + (p - sink) % (S - sink);
    for (int b = 0; b < B; ++b) slot_mapping[static_cast<int64_t>(b) * T + t] = static_cast<int32_t>(slot);
    slot_pos[slot] = static_cast<int32_t>(p);
  }
  if (t == 0) {
    const int64_t end = p0 + T;
    *kv_len = static_cast<int32_t>(end < S ? end : S);
  }
}

// One thread per 4 consecutive slots of one row; float4 stores.
__global__ void sink_mask_kernel(const int32_t *__restrict__ input_pos, int Lq,
                                 const int32_t *__restrict__ slot_pos, int64_t S, float *__restrict__ mask) {
  const int64_t quads = S >> 2;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= quads * Lq) return;
  const int r = static_cast<int>(i / quads);
  const int64_t s = (i - static_cast<int64_t>(r) * quads) * 4;
  const int64_t qpos = static_cast<int64_t>(*input_pos) + r;
  const int4 sp = *reinterpret_cast<const int4 *>(slot_pos + s);
  const float ninf = __int_as_float(0xff800000);
  float4 m;
  m.x = (sp.x >= 0 && sp.x <= qpos) ? 0.0f : ninf;
  m.y = (sp.y >= 0 && sp.y <= qpos) ? 0.0f : ninf;
  m.z = (sp.z >= 0 && sp.z <= qpos) ? 0.0f : ninf;
  m.w = (sp.w >= 0 && sp.w <= qpos) ? 0.0f : ninf;
  *reinterpret_cast<float4 *>(mask + static_cast<int64_t>(r) * S + s) = m;
}

// Per-row positions: batch row b is its own sequence, at positions
// input_pos[b] .. input_pos[b] + T - 1, with its own slot table slot_pos[b, :].
// grid (ceil(T / 128), B).
__global__ void sink_plan_rows_kernel(const int32_t *__restrict__ input_pos, int T, int sink, int64_t S,
                                      int32_t *__restrict__ slot_mapping, int32_t *__restrict__ slot_pos,
                                      int32_t *__restrict__ kv_lens, int32_t *err) {
  const int b = blockIdx.y;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t p0 = input_pos[b];
  int32_t *sm = slot_mapping + static_cast<int64_t>(b) * T;
  if (p0 < 0) {
    if (t < T) sm[t] = -1;
    if (t == 0) {
      kv_lens[b] = 0;
      report(err, KVQ_ERR_INPUT_POS);
    }
    return;
  }
  if (t < T) {
    const int64_t p = p0 + t;
    const int64_t slot = p < sink ? p : sink + (p - sink) % (S - sink);
    sm[t] = static_cast<int32_t>(slot);
    slot_pos[static_cast<int64_t>(b) * S + slot] = static_cast<int32_t>(p);
  }
  if (t == 0) {
    const int64_t end = p0 + T;
    kv_lens[b] = static_cast<int32_t>(end < S ? end : S);
  }
}

// mask [B, Lq, S]: row r of batch row b sits at input_pos[b] + r and reads
// slot_pos[b, :].  One thread per 4 consecutive slots; float4 stores.
__global__ void sink_mask_rows_kernel(const int32_t *__restrict__ input_pos, int B, int Lq,
                                      const int32_t *__restrict__ slot_pos, int64_t S, float *__restrict__ mask) {
  const int64_t quads = S >> 2;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= quads * Lq * B) return;
  const int64_t row = i / quads;  // b * Lq + r
  const int b = static_cast<int>(row / Lq), r = static_cast<int>(row - static_cast<int64_t>(b) * Lq);
  const int64_t s = (i - row * quads) * 4;
  const int64_t qpos = static_cast<int64_t>(input_pos[b]) + r;
  const int4 sp = *reinterpret_cast<const int4 *>(slot_pos + static_cast<int64_t>(b) * S + s);
  const float ninf = __int_as_float(0xff800000);
  float4 m;
  m.x = (sp.x >= 0 && sp.x <= qpos) ? 0.0f : ninf;
  m.y = (sp.y >= 0 && sp.y <= qpos) ? 0.0f : ninf;
  m.z = (sp.z >= 0 && sp.z <= qpos) ? 0.0f : ninf;
  m.w = (sp.w >= 0 && sp.w <= qpos) ? 0.0f : ninf;
  *reinterpret_cast<float4 *>(mask + row * S + s) = m;
}

}  // namespace
}  // namespace kvq

extern "C" int kvq_sink_plan(const int32_t *input_pos, int B, int T, int sink_size, int64_t S,
                             int32_t *slot_mapping, int32_t *slot_pos, int32_t *kv_len, int32_t *err_word,
                             void *stream) {
  using namespace kvq;
  if (!input_pos || !slot_mapping || !slot_pos || !kv_len) return KVQ_EINVAL;
  if (B <= 0 || T <= 0 || S <= 0 || S > INT32_MAX || sink_size < 0 || sink_size >= S) return KVQ_EINVAL;
  if (T > S - sink_size) return KVQ_EUNSUPPORTED;
  const int threads = 128;
  const int blocks = (T + threads - 1) / threads;
  sink_plan_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(input_pos, B, T, sink_size, S,
                                                                             slot_mapping, slot_pos, kv_len,
                                                                             err_word);
  return launch_status();
}

extern "C" int kvq_sink_mask(const int32_t *input_pos, int Lq, const int32_t *slot_pos, int64_t S, float *mask,
                             void *stream) {
  using namespace kvq;
  if (!input_pos || !slot_pos || !mask) return KVQ_EINVAL;
  if (Lq <= 0 || S <= 0 || S > INT32_MAX) return KVQ_EINVAL;
  if (S % 4 != 0 || !aligned16(slot_pos) || !aligned16(mask)) return KVQ_EINVAL;
  const int64_t work = (S / 4) * Lq;
  const int threads = 256;
  const int64_t blocks = (work + threads - 1) / threads;
  if (blocks > INT32_MAX) return KVQ_EUNSUPPORTED;
  sink_mask_kernel<<<static_cast<int>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      input_pos, Lq, slot_pos, S, mask);
  return launch_status();
}

extern "C" int kvq_sink_plan_rows(const int32_t *input_pos, int B, int T, int sink_size, int64_t S,
                                  int32_t *slot_mapping, int32_t *slot_pos, int32_t *kv_lens, int32_t *err_word,
                                  void *stream) {
  using namespace kvq;
  if (!input_pos || !slot_mapping || !slot_pos || !kv_lens) return KVQ_EINVAL;
  if (B <= 0 || T <= 0 || S <= 0 || S > INT32_MAX || sink_size < 0 || sink_size >= S) return KVQ_EINVAL;
  if (B > 65535) return KVQ_EUNSUPPORTED;
  if (T > S - sink_size) return KVQ_EUNSUPPORTED;
  const int threads = 128;
  const dim3 grid((T + threads - 1) / threads, B);
  sink_plan_rows_kernel<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(input_pos, T, sink_size, S,
                                                                                  slot_mapping, slot_pos, kv_lens,
                                                                                  err_word);
  return launch_status();
}

extern "C" int kvq_sink_mask_rows(const int32_t *input_pos, int B, int Lq, const int32_t *slot_pos, int64_t S,
                                  float *mask, void *stream) {
  using namespace kvq;
  if (!input_pos || !slot_pos || !mask) return KVQ_EINVAL;
  if (B <= 0 || Lq <= 0 || S <= 0 || S > INT32_MAX) return KVQ_EINVAL;
  if (S % 4 != 0 || !aligned16(slot_pos) || !aligned16(mask)) return KVQ_EINVAL;
  const int64_t work = (S / 4) * Lq * B;
  const int threads = 256;
  const int64_t blocks = (work + threads - 1) / threads;
  if (blocks > INT32_MAX) return KVQ_EUNSUPPORTED;
  sink_mask_rows_kernel<<<static_cast<int>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      input_pos, B, Lq, slot_pos, S, mask);
  return launch_status();
}
