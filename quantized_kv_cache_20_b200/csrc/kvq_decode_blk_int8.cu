// kvq_decode_blk_int8.cu -- the tensor-core decode variants over block caches of
// mode 6 (int8 codes, float scales per 32), and the path's workspace size.
#include "kvq_decode_blk.cuh"

namespace kvq {
template <>
int decode_blk_run<KVQ_MODE_INT8_SYM>(const BlkCall &c) {
  return decode_blk_run_impl<KVQ_MODE_INT8_SYM>(c);
}

size_t decode_blk_ws_bytes(int G, int D) {
  if (G < 1 || (D != 64 && D != 128 && D != 256)) return 0;
  return ws_layout(D, head_chunk_mma(G), sm_count()).total;
}
}  // namespace kvq
