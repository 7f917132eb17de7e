// kvq_decode_blk_fp4.cu -- the tensor-core decode variants over MX-FP4 block caches
// (kvq_write mode 3: E2M1 codes two per byte, E8M0 scales), D = 128 and 256.
#include "kvq_decode_blk.cuh"

namespace kvq {
template <>
int decode_blk_run<KVQ_MODE_MXFP4>(const BlkCall &c) {
  return decode_blk_run_impl<KVQ_MODE_MXFP4>(c);
}
}  // namespace kvq
