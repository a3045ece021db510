// Static per-expert bit widths (EdgeMoE-style expert-wise bit-width
// adaptation; the fixed-width special case of D2MoE's nested weights): every
// assignment of expert e runs at width_of[e], so bits[t][j] =
// width_of[topk_idx[t][j]].  The nested-plane FFN then reads, per expert,
// only the planes up to that width.
#include "common.cuh"

namespace moeq {
namespace {

__global__ void __launch_bounds__(256) k_static_bits(const int32_t* __restrict__ idx,
                                                      const uint8_t* __restrict__ width_of, int n, int E,
                                                      uint8_t* __restrict__ bits, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  bool bad = false;
  for (int a = blockIdx.x * blockDim.x + threadIdx.x; a < n; a += gridDim.x * blockDim.x) {
    int e = idx[a];
    if (e < 0 || e >= E) {
      bad = true;
      e = e < 0 ? 0 : E - 1;
    }
    int b = width_of[e];
    if (b < 2 || b > 4) {
      bad = true;
      b = b < 2 ? 2 : 4;
    }
    bits[a] = static_cast<uint8_t>(b);
  }
  if (bad) flag_status(status, MOE_DEV_BAD_INDEX);
}

}  // namespace

moe_status_t launch_static_bits(const int32_t* idx, const uint8_t* width_of, int n, int E, uint8_t* bits,
                                int32_t* status, cudaStream_t s) {
  const int blocks = std::max(1, std::min((n + 255) / 256, 1184));
  return cuda_check(launch_pdl(pdl_for(n), k_static_bits, dim3(blocks), dim3(256), 0, s, idx, width_of, n, E,
                               bits, status),
                    "moe_static_bits launch");
}

}  // namespace moeq
