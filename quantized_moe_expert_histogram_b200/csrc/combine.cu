// Weighted unpermute-combine: y[t] = bf16(res[t] + sum_j g[t][j] * y_perm[inv_perm[t*k+j]]).
// One thread produces 4 consecutive outputs of one token (float4 loads of
// the k permuted rows), summing in fp32 in ascending j.
#include <algorithm>

#include "common.cuh"

namespace moeq {
namespace {

__global__ void __launch_bounds__(256) k_combine(const float* __restrict__ y_perm,
                                                  const int32_t* __restrict__ inv_perm,
                                                  const float* __restrict__ gw,
                                                  const __nv_bfloat16* __restrict__ residual, int T,
                                                  int k, int d, __nv_bfloat16* __restrict__ y) {
  const int vec = d / 4;
  const long total = static_cast<long>(T) * vec;
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / vec);
    const int c = static_cast<int>(i % vec) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (residual) {
      const __nv_bfloat162* r = reinterpret_cast<const __nv_bfloat162*>(residual + static_cast<size_t>(t) * d + c);
      const float2 a = __bfloat1622float2(r[0]);
      const float2 b = __bfloat1622float2(r[1]);
      acc = make_float4(a.x, a.y, b.x, b.y);
    }
    for (int j = 0; j < k; ++j) {
      const float g = gw[static_cast<size_t>(t) * k + j];
      const int p = inv_perm[static_cast<size_t>(t) * k + j];
      const float4 v = *reinterpret_cast<const float4*>(y_perm + static_cast<size_t>(p) * d + c);
      acc.x = fmaf(g, v.x, acc.x);
      acc.y = fmaf(g, v.y, acc.y);
      acc.z = fmaf(g, v.z, acc.z);
      acc.w = fmaf(g, v.w, acc.w);
    }
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(y + static_cast<size_t>(t) * d + c);
    o[0] = __floats2bfloat162_rn(acc.x, acc.y);
    o[1] = __floats2bfloat162_rn(acc.z, acc.w);
  }
}

}  // namespace

moe_status_t launch_combine(const float* y_perm, const int32_t* inv_perm, const float* w,
                            const void* residual, int T, int k, int d, void* y, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const long vecs = static_cast<long>(T) * (d / 4);
  const int blocks = static_cast<int>(std::min<long>((vecs + 255) / 256, 148L * 16));
  k_combine<<<blocks, 256, 0, s>>>(y_perm, inv_perm, w, static_cast<const __nv_bfloat16*>(residual),
                                   T, k, d, static_cast<__nv_bfloat16*>(y));
  return cuda_check(cudaGetLastError(), "moe_unpermute_combine launch");
}

}  // namespace moeq
