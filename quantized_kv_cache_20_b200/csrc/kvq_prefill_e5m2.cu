// kvq_prefill_e5m2.cu -- the tcgen05 prefill kernel variants over block caches of
// modes 4 (E5M2, float scales) and 5 (E5M2, E8M0 scales); one file per mode pair so the variants compile in parallel.
#include "kvq_common.cuh"
#include "kvq_prefill_tc.cuh"

namespace kvq {
namespace tc {
template int dispatch_prefill_mode<KVQ_MODE_FP8_E5M2>(const PrefillArgs &, int, cudaStream_t);
template int dispatch_prefill_mode<KVQ_MODE_MXFP8_E5M2>(const PrefillArgs &, int, cudaStream_t);
}  // namespace tc
}  // namespace kvq
