// kvq_decode_blk_e4m3.cu -- the tensor-core decode variants over block caches of
// modes 1 (E4M3, float scales) and 2 (MX-FP8); one file per mode pair so the variants compile in parallel.
#include "kvq_decode_blk.cuh"

namespace kvq {
template <>
int decode_blk_run<KVQ_MODE_FP8_E4M3>(const BlkCall &c) {
  return decode_blk_run_impl<KVQ_MODE_FP8_E4M3>(c);
}
template <>
int decode_blk_run<KVQ_MODE_MXFP8>(const BlkCall &c) {
  return decode_blk_run_impl<KVQ_MODE_MXFP8>(c);
}
}  // namespace kvq
