// kvq_api.cu -- status strings and version of the kvq C ABI.
#include "kvq.h"

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
