// kvq_api.cu -- status strings, version and the process-wide wait bound of the kvq C ABI.
#include <atomic>

#include "kvq_common.cuh"

namespace kvq {
namespace {
std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};
}  // namespace
uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
}  // namespace kvq

extern "C" int kvq_set_wait_limit_ns(uint64_t ns) {
  kvq::g_wait_limit_ns.store(ns == 0 ? kvq::kWaitLimitNs : ns, std::memory_order_relaxed);
  return KVQ_OK;
}

extern "C" const char *kvq_strerror(int status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_EINVAL: return "invalid argument (null or misaligned pointer, bad size or stride)";
    case KVQ_EUNSUPPORTED: return "unsupported configuration";
    case KVQ_ECUDA: return "CUDA launch failed";
    case KVQ_ESCRATCH: return "the problem needs more scratch than the library's static buffer holds";
    default: return "unknown kvq status";
  }
}

extern "C" int kvq_version(void) { return 100; }
