// kvq_prefill_fp4_int8.cu -- the tcgen05 prefill kernel variants over block caches of
// modes 3 (MX-FP4) and 6 (int8 codes, float scales); one file per mode pair so the variants compile in parallel.
#include "kvq_common.cuh"
#include "kvq_prefill_tc.cuh"

namespace kvq {
namespace tc {
template int dispatch_prefill_mode<KVQ_MODE_MXFP4>(const PrefillArgs &, int, cudaStream_t);
template int dispatch_prefill_mode<KVQ_MODE_INT8_SYM>(const PrefillArgs &, int, cudaStream_t);
}  // namespace tc
}  // namespace kvq
