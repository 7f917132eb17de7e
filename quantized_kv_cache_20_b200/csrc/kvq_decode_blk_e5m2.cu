// kvq_decode_blk_e5m2.cu -- the tensor-core decode variants over block caches of
// modes 4 (E5M2, float scales) and 5 (E5M2, E8M0 scales); one file per mode pair so the variants compile in parallel.
#include "kvq_decode_blk.cuh"

namespace kvq {
template <>
int decode_blk_run<KVQ_MODE_FP8_E5M2>(const BlkCall &c) {
  return decode_blk_run_impl<KVQ_MODE_FP8_E5M2>(c);
}
template <>
int decode_blk_run<KVQ_MODE_MXFP8_E5M2>(const BlkCall &c) {
  return decode_blk_run_impl<KVQ_MODE_MXFP8_E5M2>(c);
}
}  // namespace kvq
