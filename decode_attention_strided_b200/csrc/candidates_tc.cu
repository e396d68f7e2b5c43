// candidates_tc.cu -- tensor-core (tcgen05) nearest-reference search.
#include "internal.h"

namespace dkv {

bool candidates_tc_supported(const Plan& p) { (void)p; return false; }

cudaError_t launch_candidates_tc(const Plan& p, int T, const KVView& kv, const void* cache,
                                 void* ws, cudaStream_t st) {
  (void)p; (void)T; (void)kv; (void)cache; (void)ws; (void)st;
  return cudaErrorNotSupported;
}

}  // namespace dkv
