// Prefill-regime grouped expert FFN on the tcgen05 tensor cores.
#include "common.cuh"

namespace moeq {

bool tc_supported(const FfnArgs& a) {
  (void)a;
  return false;
}

moe_status_t launch_ffn_tc(const FfnArgs& a, cudaStream_t s) {
  (void)a;
  (void)s;
  set_error("tensor-core FFN path not available for this shape");
  return MOE_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace moeq
