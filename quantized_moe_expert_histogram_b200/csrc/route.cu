// Softmax top-k router.
//
// Logits l[t][e] = x[t] . W_r[e] (+ bias[e]) are accumulated in fp64: a
// bf16 x fp32 product is exact in fp64, and fp64 leaves no practical room
// for a summation-order difference to flip a top-k decision, so the expert
// choice equals a plain fp64 evaluation of the definition.  A block owns
// TT tokens and walks the expert dimension in chunks of EC; each thread
// keeps an MT x ME register tile of logits.  Selection is a warp argmax
// repeated k times (ties -> lower index), then a softmax over the k picks.
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kThreads = 128;
constexpr int kDC = 32;  // d-chunk staged in shared memory

template <int EC, int ME, int MT>
struct RouteCfg {
  static constexpr int TX = EC / ME;
  static constexpr int TY = kThreads / TX;
  static constexpr int TT = TY * MT;
};

template <int EC, int ME, int MT>
__global__ void __launch_bounds__(kThreads) k_route(const __nv_bfloat16* __restrict__ x,
                                                     const float* __restrict__ wr,
                                                     const float* __restrict__ bias,
                                                     const int32_t* __restrict__ forced, int T,
                                                     int d, int E, int k,
                                                     int32_t* __restrict__ out_idx,
                                                     float* __restrict__ out_w) {
  using C = RouteCfg<EC, ME, MT>;
  extern __shared__ double smem_d[];
  double* xs = smem_d;                          // [kDC][TT]
  double* ws = xs + C::TT * kDC;                // [kDC][EC]
  double* logits = ws + EC * kDC;               // [TT][E]

  const int tid = threadIdx.x;
  const int tx = tid % C::TX, ty = tid / C::TX;
  const int t0 = blockIdx.x * C::TT;

  for (int e0 = 0; e0 < E; e0 += EC) {
    double acc[MT][ME];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
      for (int j = 0; j < ME; ++j) acc[i][j] = 0.0;

    for (int k0 = 0; k0 < d; k0 += kDC) {
      __syncthreads();
      for (int i = tid; i < C::TT * kDC; i += kThreads) {
        const int r = i / kDC, c = i % kDC;
        const int t = t0 + r;
        xs[c * C::TT + r] =
            (t < T) ? static_cast<double>(__bfloat162float(x[static_cast<size_t>(t) * d + k0 + c])) : 0.0;
      }
      for (int i = tid; i < EC * kDC; i += kThreads) {
        const int r = i / kDC, c = i % kDC;
        const int e = e0 + r;
        ws[c * EC + r] = (e < E) ? static_cast<double>(wr[static_cast<size_t>(e) * d + k0 + c]) : 0.0;
      }
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < kDC; ++c) {
        double xv[MT], wv[ME];
#pragma unroll
        for (int i = 0; i < MT; ++i) xv[i] = xs[c * C::TT + i * C::TY + ty];
#pragma unroll
        for (int j = 0; j < ME; ++j) wv[j] = ws[c * EC + j * C::TX + tx];
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
          for (int j = 0; j < ME; ++j) acc[i][j] = fma(xv[i], wv[j], acc[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
      for (int j = 0; j < ME; ++j) {
        const int e = e0 + j * C::TX + tx;
        if (e < E) {
          double v = acc[i][j];
          if (bias) v += static_cast<double>(bias[e]);
          logits[(i * C::TY + ty) * E + e] = v;
        }
      }
  }
  __syncthreads();

  // Selection: one warp per token.
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < C::TT; r += kThreads / 32) {
    const int t = t0 + r;
    if (t >= T) break;
    double* lr = logits + r * E;
    int sel_e[16];
    double sel_l[16];
    if (forced) {
      for (int j = 0; j < k; ++j) {
        int e = forced[static_cast<size_t>(t) * k + j];
        e = e < 0 ? 0 : (e >= E ? E - 1 : e);
        sel_e[j] = e;
        sel_l[j] = lr[e];
      }
    } else {
      // mark picked experts with a flag array in registers: lane owns e = lane + 32 m
      uint32_t taken = 0;  // bit m -> expert lane + 32 m taken (E <= 256 -> m < 8)
      for (int j = 0; j < k; ++j) {
        double best = -INFINITY;
        int best_e = 0x7fffffff;
        for (int m = 0; lane + 32 * m < E; ++m) {
          const int e = lane + 32 * m;
          if (taken & (1u << m)) continue;
          const double v = lr[e];
          if (v > best || (v == best && e < best_e)) {
            best = v;
            best_e = e;
          }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const double ov = __shfl_xor_sync(0xffffffffu, best, o);
          const int oe = __shfl_xor_sync(0xffffffffu, best_e, o);
          if (ov > best || (ov == best && oe < best_e)) {
            best = ov;
            best_e = oe;
          }
        }
        sel_e[j] = best_e;
        sel_l[j] = best;
        if ((best_e & 31) == lane) taken |= 1u << (best_e >> 5);
      }
    }
    double m = sel_l[0];
    for (int j = 1; j < k; ++j) m = fmax(m, sel_l[j]);
    double sum = 0.0;
    double ex[16];
    for (int j = 0; j < k; ++j) {
      ex[j] = exp(sel_l[j] - m);
      sum += ex[j];
    }
    if (lane < k) {
      // lane j writes output j (registers indexed by a runtime lane: use a loop)
      for (int j = 0; j < k; ++j)
        if (j == lane) {
          out_idx[static_cast<size_t>(t) * k + j] = sel_e[j];
          out_w[static_cast<size_t>(t) * k + j] = static_cast<float>(ex[j] / sum);
        }
    }
  }
}

template <int EC, int ME, int MT>
moe_status_t run(const void* x, const float* wr, const float* bias, const int32_t* forced, int T,
                 int d, int E, int k, int32_t* idx, float* w, cudaStream_t s) {
  using C = RouteCfg<EC, ME, MT>;
  const size_t smem = sizeof(double) * (static_cast<size_t>(C::TT) * kDC + EC * kDC +
                                        static_cast<size_t>(C::TT) * E);
  auto kern = k_route<EC, ME, MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_check(e, "moe_route_topk smem attribute");
  const int blocks = ceil_div(T, C::TT);
  kern<<<blocks, kThreads, smem, s>>>(static_cast<const __nv_bfloat16*>(x), wr, bias, forced, T, d,
                                      E, k, idx, w);
  return cuda_check(cudaGetLastError(), "moe_route_topk launch");
}

}  // namespace

moe_status_t launch_route(const void* x, const float* w_router, const float* bias,
                          const int32_t* forced, int T, int d, int E, int k, int32_t* idx,
                          float* w, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (d % kDC != 0) {
    set_error("moe_route_topk: d=%d must be a multiple of %d", d, kDC);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (E <= 8) return run<8, 2, 4>(x, w_router, bias, forced, T, d, E, k, idx, w, s);
  if (E <= 16) return run<16, 4, 4>(x, w_router, bias, forced, T, d, E, k, idx, w, s);
  if (E <= 32) return run<32, 4, 4>(x, w_router, bias, forced, T, d, E, k, idx, w, s);
  return run<64, 4, 4>(x, w_router, bias, forced, T, d, E, k, idx, w, s);
}

}  // namespace moeq
