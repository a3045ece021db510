// Weighted unpermute-combine: y[t] = bf16(res[t] + sum_j g[t][j] * y_perm[inv_perm[t*k+j]]).
// One thread produces 8 consecutive outputs of one token (one 16-byte load
// per permuted fp16 row), summing in fp32 in ascending j.
#include <algorithm>

#include "common.cuh"

namespace moeq {
namespace {

__global__ void __launch_bounds__(256) k_combine(const __half* __restrict__ y_perm,
                                                  const int32_t* __restrict__ inv_perm,
                                                  const float* __restrict__ gw,
                                                  const __nv_bfloat16* __restrict__ residual, int T,
                                                  int k, int d, __nv_bfloat16* __restrict__ y, int early) {
  const int vec = d / 8;
  const long total = static_cast<long>(T) * vec;
  const long first = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x;
  // early (the caller's previous launch writes only y_perm, e.g. the FFN's
  // second GEMM, and gates, inv_perm and residual were written at least two
  // launches back, complete once this kernel has started): the gates and
  // rows of this thread's first token and its residual are read before the
  // wait
  float g0[8];
  int p0[8];
  uint4 r0 = make_uint4(0, 0, 0, 0);
  if (early && first < total) {
    const int t = static_cast<int>(first / vec);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      g0[u] = 0.0f;
      p0[u] = 0;
      if (u < k) {
        g0[u] = gw[static_cast<size_t>(t) * k + u];
        p0[u] = min(max(inv_perm[static_cast<size_t>(t) * k + u], 0), T * k - 1);
      }
    }
    if (residual) r0 = *reinterpret_cast<const uint4*>(residual + static_cast<size_t>(t) * d + (first % vec) * 8);
  }
  pdl_wait();
  pdl_trigger();
  for (long i = first; i < total; i += static_cast<long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / vec);
    const int c = static_cast<int>(i % vec) * 8;
    const bool pre = early && i == first;
    float acc[8];
    if (residual) {
      const uint4 r = pre ? r0 : *reinterpret_cast<const uint4*>(residual + static_cast<size_t>(t) * d + c);
      const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(r2[u]);
        acc[2 * u] = f.x;
        acc[2 * u + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
    }
    // up to 8 choices at a time: their gates and rows are loaded before any
    // is summed (independent loads in flight), the sum stays in ascending j
    for (int j0 = 0; j0 < k; j0 += 8) {
      float g[8];
      int p[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        g[u] = 0.0f;
        p[u] = 0;
        if (pre && j0 == 0) {
          g[u] = g0[u];
          p[u] = p0[u];
        } else if (j0 + u < k) {
          g[u] = gw[static_cast<size_t>(t) * k + j0 + u];
          // clamped: an inconsistent inv_perm gives wrong rows, never an out-of-range read
          p[u] = min(max(inv_perm[static_cast<size_t>(t) * k + j0 + u], 0), T * k - 1);
        }
      }
      uint4 raw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (j0 + u < k) raw[u] = *reinterpret_cast<const uint4*>(y_perm + static_cast<size_t>(p[u]) * d + c);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (j0 + u >= k) break;
        const __half2* v2 = reinterpret_cast<const __half2*>(&raw[u]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __half22float2(v2[q]);
          acc[2 * q] = fmaf(g[u], f.x, acc[2 * q]);
          acc[2 * q + 1] = fmaf(g[u], f.y, acc[2 * q + 1]);
        }
      }
    }
    uint4 o;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int u = 0; u < 4; ++u) o2[u] = __floats2bfloat162_rn(acc[2 * u], acc[2 * u + 1]);
    *reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * d + c) = o;
  }
}

}  // namespace

moe_status_t launch_combine(const void* y_perm, const int32_t* inv_perm, const float* w,
                            const void* residual, int T, int k, int d, void* y, cudaStream_t s, bool early) {
  if (T == 0) return MOE_OK;
  const long vecs = static_cast<long>(T) * (d / 8);
  const int blocks = static_cast<int>(std::min<long>((vecs + 255) / 256, 148L * 16));
  const cudaError_t e = launch_pdl(pdl_for(static_cast<long>(T) * k), k_combine, dim3(blocks), dim3(256), 0, s, static_cast<const __half*>(y_perm), inv_perm, w,
                                   static_cast<const __nv_bfloat16*>(residual), T, k, d,
                                   static_cast<__nv_bfloat16*>(y), early ? 1 : 0);
  return cuda_check(e, "moe_unpermute_combine launch");
}

}  // namespace moeq
