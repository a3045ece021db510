// Bit-width router: the "bit gate" that D2MoE places beside the expert gate
// (Design, Dual Routing; Token-Adaptive Bit-Width Selection).  For the j-th
// selected expert e of token t it scores the three widths
//   l[c] = x[t] . W_bit[e][c] + b_bit[e][c],   c = 0, 1, 2  (b = 2, 3, 4)
// and picks the first maximum (equal scores -> the narrower width).
//
// The decision must equal the one the exact scores give.  As in the expert
// router, the scores are evaluated in fp32 with a proven error bound and
// only undecided assignments are re-evaluated in fp64 (every bf16 x fp32
// product is exact there):
//   a lane sums its d/32 products with an FMA chain, the warp adds the 32
//   lane sums in a shuffle tree (5 levels), so |S - s| <= g(m) sum |x_i W_i|
//   with m = (products per lane) + 5 and g(m) = m u / (1 - m u), u = 2^-24.
//   The sum of magnitudes A is accumulated alongside (it errs by the same
//   relative g(m), covered by the factor 1 + 2^-8), and adding the bias
//   rounds once more:
//     |L[c] - l[c]| <= D[c] = 2 (g(m) A[c] (1 + 2^-8) + u (|L[c]| + |b[c]|))
//   (factor 2: margin).  The fp32 winner c* is certain when it beats every
//   other width by more than both bounds, L[c*] - D[c*] > L[c] + D[c].
//
// A warp per (token, selected expert): x[t] comes through L1, the expert's
// three W_bit rows (3 x d fp32) through L2, two 8-element steps of loads in
// flight per lane.
//
// Up to 32 assignments (k_bit_gate_tiny): the 3 T k scores over a
// thread-block cluster (each CTA one slice of d, fp32 partials with
// magnitude sums into CTA 0's shared memory, a tighter per-score bound,
// fp64 only for the assignments it leaves open; tiny_bit_gate).
#include <cmath>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32) k_bit_gate(const __nv_bfloat16* __restrict__ x,
                                                         const float* __restrict__ wb,
                                                         const float* __restrict__ bb,
                                                         const int32_t* __restrict__ idx, int T, int d, int E,
                                                         int k, float gamma, uint8_t* __restrict__ bits,
                                                         int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a = blockIdx.x * kWarps + warp;  // assignment t * k + j
  if (a >= T * k) return;                    // warp-uniform
  const int t = a / k;
  const __nv_bfloat16* xr = x + static_cast<size_t>(t) * d;
  int e = idx[a];
  if (e < 0 || e >= E) {
    if (lane == 0) flag_status(status, MOE_DEV_BAD_INDEX);
    e = e < 0 ? 0 : E - 1;
  }
  const float* w0 = wb + static_cast<size_t>(e) * 3 * d;
  float s[3] = {0.f, 0.f, 0.f}, am[3] = {0.f, 0.f, 0.f};
  // one 8-element piece of x and of the three rows per step, the loads of
  // two steps in flight together
  auto piece = [&](int i, uint4& xv, float4 (&wv)[3][2]) {
    xv = *reinterpret_cast<const uint4*>(xr + i);
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      wv[c][0] = *reinterpret_cast<const float4*>(w0 + static_cast<size_t>(c) * d + i);
      wv[c][1] = *reinterpret_cast<const float4*>(w0 + static_cast<size_t>(c) * d + i + 4);
    }
  };
  auto fold = [&](const uint4& xv, const float4 (&wv)[3][2]) {
    const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      const float w[8] = {wv[c][0].x, wv[c][0].y, wv[c][0].z, wv[c][0].w,
                          wv[c][1].x, wv[c][1].y, wv[c][1].z, wv[c][1].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(x2[q]);
        s[c] = fmaf(f.x, w[2 * q], s[c]);
        am[c] = fmaf(fabsf(f.x), fabsf(w[2 * q]), am[c]);
        s[c] = fmaf(f.y, w[2 * q + 1], s[c]);
        am[c] = fmaf(fabsf(f.y), fabsf(w[2 * q + 1]), am[c]);
      }
    }
  };
  int i = lane * 8;
  for (; i + 256 < d; i += 512) {
    uint4 xa, xb;
    float4 wa[3][2], wbv[3][2];
    piece(i, xa, wa);
    piece(i + 256, xb, wbv);
    fold(xa, wa);
    fold(xb, wbv);
  }
  if (i < d) {
    uint4 xa;
    float4 wa[3][2];
    piece(i, xa, wa);
    fold(xa, wa);
  }
#pragma unroll
  for (int c = 0; c < 3; ++c)
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      s[c] += __shfl_xor_sync(0xffffffffu, s[c], o);
      am[c] += __shfl_xor_sync(0xffffffffu, am[c], o);
    }
  float L[3], D[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const float b = bb ? bb[static_cast<size_t>(e) * 3 + c] : 0.f;
    L[c] = s[c] + b;
    D[c] = 2.0f * (gamma * am[c] * (1.0f + 0.00390625f) + 5.9604645e-8f * (fabsf(L[c]) + fabsf(b))) + 1e-30f;
  }
  int best = 0;
  if (L[1] > L[best]) best = 1;
  if (L[2] > L[best]) best = 2;
  // certain when the winner's lower bound clears every other upper bound
  // (comparisons with NaN are false: non-finite scores go to fp64)
  bool sure = true;
#pragma unroll
  for (int c = 0; c < 3; ++c)
    if (c != best) sure = sure && (L[best] - D[best] > L[c] + D[c]);
  if (!sure) {  // warp-uniform: every lane holds the reduced sums
    double v[3];
#pragma unroll
    for (int c = 0; c < 3; ++c)
      v[c] = dot_bf16_f32_fp64(xr, w0 + static_cast<size_t>(c) * d, d, lane) +
             (bb ? static_cast<double>(bb[static_cast<size_t>(e) * 3 + c]) : 0.0);
    best = 0;
    if (v[1] > v[best]) best = 1;
    if (v[2] > v[best]) best = 2;
  }
  if (lane == 0) bits[a] = static_cast<uint8_t>(2 + best);
}

__global__ void __launch_bounds__(kWarps * 32) k_bit_gate_tiny(const __nv_bfloat16* __restrict__ x,
                                                              const float* __restrict__ wb,
                                                              const float* __restrict__ bb,
                                                              const int32_t* __restrict__ idx, int T, int d,
                                                              int E, int k, float gamma, uint8_t* __restrict__ bits,
                                                              int32_t* status) {
  __shared__ TinyGateSmem S;
  __shared__ int32_t ids[kTinyGateAssign];
  pdl_wait();
  pdl_trigger();
  cluster_sync_start();
  const int na = T * k;
  for (int a = threadIdx.x; a < na; a += blockDim.x) {
    const int e = idx[a];
    if ((e < 0 || e >= E) && blockIdx.x == 0) flag_status(status, MOE_DEV_BAD_INDEX);
    ids[a] = e < 0 ? 0 : (e >= E ? E - 1 : e);
  }
  __syncthreads();
  tiny_bit_gate(x, wb, bb, ids, T, d, k, gamma, bits, nullptr, S);
}

}  // namespace

moe_status_t launch_bit_gate(const void* x, const float* w_bit, const float* bias_bit, const int32_t* idx,
                             int T, int d, int E, int k, uint8_t* bits, int32_t* status, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  // up to kTinyGateAssign assignments (at most two rounds of scores per
  // warp of the cluster): measured 46.9 -> 36.2 us for the one-token step of
  // the nested layer with its gate, 82.1 -> 77.1 us at four tokens
  if (g_route_fused == 1 && T * k <= kTinyGateAssign && d % (8 * kClusterSlices) == 0)
    return cuda_check(launch_cluster_pdl(k_bit_gate_tiny, kClusterSlices, dim3(kWarps * 32), 0, s,
                                         static_cast<const __nv_bfloat16*>(x), w_bit, bias_bit, idx, T, d, E, k,
                                         cluster_gamma(d), bits, status),
                      "moe_bit_gate cluster launch");
  const double u = std::ldexp(1.0, -24);
  const double m = ceil_div(d, 256) * 8 + 5;
  const float gamma = static_cast<float>(m * u / (1.0 - m * u));
  return cuda_check(launch_pdl(pdl_for(static_cast<long>(T) * k), k_bit_gate, dim3(ceil_div(T * k, kWarps)),
                               dim3(kWarps * 32), 0, s, static_cast<const __nv_bfloat16*>(x), w_bit, bias_bit,
                               idx, T, d, E, k, gamma, bits, status),
                    "moe_bit_gate launch");
}

}  // namespace moeq
