// kvq_decode_blk.h -- the tensor-core decode over a byte-coded block cache (kvq_write
// modes 1, 2, 4, 5, 6), as seen from the kvq_decode_attn_block entry point.  The
// kernel variants of each mode are compiled in kvq_decode_blk_*.cu.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kvq {

// One call, arguments already checked by the entry point.
struct BlkCall {
  const void *q;
  int B, Hq, Hkv, D;
  const uint8_t *k_codes, *v_codes;
  const void *k_scales, *v_scales;  // [B, Hkv, S, D/32] float or E8M0 bytes
  int64_t S;
  const int32_t *kv_len;
  const float *mask;
  float sm_scale;
  void *out, *workspace;
  size_t workspace_bytes;
  int32_t *err_word;
  cudaStream_t stream;
};

// Workspace bytes of the tensor-core path for G = Hq / Hkv and D (0 if unsupported).
size_t decode_blk_ws_bytes(int G, int D);

// Runs the call on the tensor-core path for cache mode MODE.
template <int MODE>
int decode_blk_run(const BlkCall &c);

}  // namespace kvq
