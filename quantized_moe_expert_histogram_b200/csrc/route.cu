// Softmax top-k router.
//
// Logits l[t][e] = x[t] . W_r[e] (+ bias[e]) are accumulated in fp64: a
// bf16 x fp32 product is exact in fp64, and fp64 leaves no practical room
// for a summation-order difference to flip a top-k decision, so the expert
// choice equals a plain fp64 evaluation of the definition.
//
// Two kernels:
//   k_route_partial  grid (token tiles, expert tiles, K splits): a 64 x 64
//                    (token x expert) tile over one slice of d, 4 x 4 fp64
//                    register tile per thread, 32-wide d chunks staged in
//                    shared memory as fp64; writes partial[split][t][e].
//   k_route_select   one warp per token: sums the splits in split order
//                    (the same order for every expert, so identical router
//                    rows give identical logits), adds the bias, takes the
//                    top k by a warp argmax repeated k times (ties -> lower
//                    index) and the softmax over the k picks.
// The split count is chosen so that small T still spreads the read of W_r
// over many SMs and large T keeps every SM busy.
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kThreads = 256;
constexpr int kTT = 64;   // tokens per tile
constexpr int kEC = 64;   // experts per tile
constexpr int kDC = 32;   // d chunk
constexpr int kMT = 4, kME = 4;
constexpr int kTX = kEC / kME;  // 16 threads along experts
constexpr int kTY = kTT / kMT;  // 16 threads along tokens

__global__ void __launch_bounds__(kThreads) k_route_partial(const __nv_bfloat16* __restrict__ x,
                                                             const float* __restrict__ wr, int T,
                                                             int d, int E, int dk,
                                                             double* __restrict__ partial) {
  __shared__ double xs[kDC][kTT + 1];
  __shared__ double ws[kDC][kEC + 1];
  const int tid = threadIdx.x;
  const int tx = tid % kTX, ty = tid / kTX;
  const int t0 = blockIdx.x * kTT, e0 = blockIdx.y * kEC, split = blockIdx.z;
  const int kbeg = split * dk;

  double acc[kMT][kME];
#pragma unroll
  for (int i = 0; i < kMT; ++i)
#pragma unroll
    for (int j = 0; j < kME; ++j) acc[i][j] = 0.0;

  for (int k0 = kbeg; k0 < kbeg + dk; k0 += kDC) {
    __syncthreads();
    // x chunk: 64 tokens x 32 -> 2048 values, 8 per thread (one 16-byte load)
    {
      const int r = tid / 4, c = (tid % 4) * 8;
      const int t = t0 + r;
      if (t < T) {
        const uint4 v = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d + k0 + c);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(b2[j]);
          xs[c + 2 * j][r] = f.x;
          xs[c + 2 * j + 1][r] = f.y;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) xs[c + j][r] = 0.0;
      }
    }
    // W chunk: 64 experts x 32 -> 2048 values, 8 per thread (two 16-byte loads)
    {
      const int r = tid / 4, c = (tid % 4) * 8;
      const int e = e0 + r;
      if (e < E) {
        const float4 a = *reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * d + k0 + c);
        const float4 b = *reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * d + k0 + c + 4);
        ws[c + 0][r] = a.x; ws[c + 1][r] = a.y; ws[c + 2][r] = a.z; ws[c + 3][r] = a.w;
        ws[c + 4][r] = b.x; ws[c + 5][r] = b.y; ws[c + 6][r] = b.z; ws[c + 7][r] = b.w;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) ws[c + j][r] = 0.0;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kDC; ++c) {
      double xv[kMT], wv[kME];
#pragma unroll
      for (int i = 0; i < kMT; ++i) xv[i] = xs[c][i * kTY + ty];
#pragma unroll
      for (int j = 0; j < kME; ++j) wv[j] = ws[c][j * kTX + tx];
#pragma unroll
      for (int i = 0; i < kMT; ++i)
#pragma unroll
        for (int j = 0; j < kME; ++j) acc[i][j] = fma(xv[i], wv[j], acc[i][j]);
    }
  }
  double* out = partial + static_cast<size_t>(split) * T * E;
#pragma unroll
  for (int i = 0; i < kMT; ++i) {
    const int t = t0 + i * kTY + ty;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < kME; ++j) {
      const int e = e0 + j * kTX + tx;
      if (e < E) out[static_cast<size_t>(t) * E + e] = acc[i][j];
    }
  }
}

__global__ void __launch_bounds__(kThreads) k_route_select(const double* __restrict__ partial,
                                                            int splits, const float* __restrict__ bias,
                                                            const int32_t* __restrict__ forced, int T,
                                                            int E, int k, int32_t* __restrict__ out_idx,
                                                            float* __restrict__ out_w) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int t = warp;
  if (t >= T) return;
  constexpr int kPer = 8;  // E <= 256 -> at most 8 experts per lane
  double l[kPer];
#pragma unroll
  for (int m = 0; m < kPer; ++m) {
    const int e = lane + 32 * m;
    double v = -INFINITY;
    if (e < E) {
      v = 0.0;
      for (int s = 0; s < splits; ++s) v += partial[(static_cast<size_t>(s) * T + t) * E + e];
      if (bias) v += static_cast<double>(bias[e]);
    }
    l[m] = v;
  }
  int sel_e[16];
  double sel_l[16];
  if (forced) {
    for (int j = 0; j < k; ++j) {
      int e = forced[static_cast<size_t>(t) * k + j];
      e = e < 0 ? 0 : (e >= E ? E - 1 : e);
      double v = 0.0;
#pragma unroll
      for (int m = 0; m < kPer; ++m) {
        const double o = __shfl_sync(0xffffffffu, l[m], e & 31);
        if ((e >> 5) == m) v = o;
      }
      sel_e[j] = e;
      sel_l[j] = v;
    }
  } else {
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
      double best = -INFINITY;
      int best_e = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < kPer; ++m) {
        const int e = lane + 32 * m;
        if (e < E && !(taken & (1u << m))) {
          if (l[m] > best || (l[m] == best && e < best_e)) {
            best = l[m];
            best_e = e;
          }
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
  double mx = sel_l[0];
  for (int j = 1; j < k; ++j) mx = fmax(mx, sel_l[j]);
  double sum = 0.0;
  double ex[16];
  for (int j = 0; j < k; ++j) {
    ex[j] = exp(sel_l[j] - mx);
    sum += ex[j];
  }
  for (int j = 0; j < k; ++j)
    if (j == lane) {
      out_idx[static_cast<size_t>(t) * k + j] = sel_e[j];
      out_w[static_cast<size_t>(t) * k + j] = static_cast<float>(ex[j] / sum);
    }
}

}  // namespace

int route_splits(int T, int d, int E) {
  const int tiles = ceil_div(T, kTT) * ceil_div(E, kEC);
  const int chunks = d / kDC;
  const int target = ceil_div(2 * 148, tiles);
  int s = 1;
  while (s * 2 <= target && chunks % (s * 2) == 0 && s * 2 <= 64) s *= 2;
  return s;
}

size_t route_workspace_bytes(int T, int d, int E) {
  if (T <= 0 || d <= 0 || E <= 0) return 256;
  return static_cast<size_t>(route_splits(T, d, E)) * T * E * sizeof(double);
}

moe_status_t launch_route(const void* x, const float* w_router, const float* bias,
                          const int32_t* forced, int T, int d, int E, int k, int32_t* idx,
                          float* w, void* workspace, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int splits = route_splits(T, d, E);
  double* partial = static_cast<double*>(workspace);
  dim3 grid(ceil_div(T, kTT), ceil_div(E, kEC), splits);
  k_route_partial<<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), w_router, T, d, E,
                                            d / splits, partial);
  moe_status_t st = cuda_check(cudaGetLastError(), "moe_route_topk partial launch");
  if (st != MOE_OK) return st;
  k_route_select<<<ceil_div(T * 32, kThreads), kThreads, 0, s>>>(partial, splits, bias, forced, T, E,
                                                                  k, idx, w);
  return cuda_check(cudaGetLastError(), "moe_route_topk select launch");
}

}  // namespace moeq

// ---------------------------------------------------------------------------
// Allocation-free router entry point.
//
// Some callers cannot allocate device memory at the point where they route:
// code that runs while a stream is being captured into a CUDA graph (where
// cudaMalloc is not allowed), plugins and runtimes that hand us only a
// stream and have no allocator of their own to lend, and latency-critical
// serving paths that must not risk an allocation failure or an implicit
// synchronisation.  moe_route_topk_noalloc keeps the router's scratch (the
// per-slice fp64 partial logits) in a fixed device array owned by this
// library instead of a caller-provided workspace.
// ---------------------------------------------------------------------------

#include <mutex>

namespace moeq {
namespace {

constexpr size_t kRouteScratchBytes = 8u << 20;  // 8 MiB, held by every GPU that loads the library
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, resolved once
// per device (with that device current).
moe_status_t route_scratch(void** out) {
  int dev = 0;
  moe_status_t st = cuda_check(cudaGetDevice(&dev), "moe_route_topk_noalloc: cudaGetDevice");
  if (st != MOE_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("moe_route_topk_noalloc: device %d beyond the supported %d", dev, kMaxDevices);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    st = cuda_check(cudaGetSymbolAddress(&p, g_route_scratch), "moe_route_topk_noalloc: cudaGetSymbolAddress");
    if (st != MOE_OK) return st;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moeq

extern "C" moe_status_t moe_route_topk_noalloc(const void* x, const float* w_router, const float* bias,
                                                const int32_t* forced_idx, int T, int d, int E, int k,
                                                int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  using namespace moeq;
  const size_t need = route_workspace_bytes(T, d, E);
  if (T > 0 && need > kRouteScratchBytes) {
    set_error("moe_route_topk_noalloc: T=%d d=%d E=%d needs %zu bytes of scratch, above the fixed %zu",
              T, d, E, need, kRouteScratchBytes);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  void* scratch = nullptr;
  if (T > 0) {
    moe_status_t st = route_scratch(&scratch);
    if (st != MOE_OK) return st;
  }
  return moe_route_topk(x, w_router, bias, forced_idx, T, d, E, k, topk_idx, topk_w, scratch,
                        kRouteScratchBytes, stream);
}
