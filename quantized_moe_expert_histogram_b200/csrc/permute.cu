// Per-expert histogram, exclusive prefix sum and stable permutation of the
// T*k assignments, plus the gather of activation rows into expert order.
//
// Three kernels, deterministic and atomics-free:
//   k_perm_hist     CTA c owns assignments [c*CH, (c+1)*CH); each warp
//                   counts its 32-wide slices: lanes with equal keys are
//                   found with __match_any_sync and the lowest of them adds
//                   the group size to the warp's shared histogram; the CTA
//                   histogram (warps summed in order) goes to hist[bin][c].
//   k_perm_scan     one CTA: a warp per bin scans its row of hist into
//                   per-CTA start positions inside the bin and the bin
//                   total; a block scan of the totals gives offsets, which
//                   the warps then add to every start.
//   k_perm_scatter  CTA c recounts its warps, so that warp w starts at the
//                   CTA's start plus the counts of warps 0..w-1; a lane's
//                   position is its warp's cursor plus the number of lower
//                   lanes with the same key in the slice (ascending a inside
//                   a bin).  It writes perm and inv_perm.
// When all assignments fit one CTA's chunk (T*k <= 1024, decode-sized
// batches) k_perm_one does the three steps in a single launch, and for up
// to 64 K gathered elements the gather of activation rows too.  Otherwise
// the gather (bf16 -> fp16) is its own grid-wide launch: it moves
// T*k*d*2 bytes and needs every SM, while the sort needs only T*k/1024
// CTAs.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kWarps = 8;                   // per CTA
constexpr int kSlices = 4;                  // 32-assignment slices per warp
constexpr int kCH = kWarps * 32 * kSlices;  // assignments per CTA (1024)
constexpr int kMaxBins = 768;

__device__ __forceinline__ int load_key(const int32_t* idx, const uint8_t* bits, int a, int E,
                                        int32_t* status) {
  int e = idx[a];
  if (e < 0 || e >= E) {
    flag_status(status, MOE_DEV_BAD_INDEX);
    e = e < 0 ? 0 : E - 1;
  }
  if (!bits) return e;
  int b = bits[a];
  if (b < 2 || b > 4) {
    flag_status(status, MOE_DEV_BAD_INDEX);
    b = b < 2 ? 2 : 4;
  }
  return 3 * e + (b - 2);
}

// Per-warp histograms of this CTA's chunk into smem [kWarps][nbins]; the
// keys of the warp's slices are returned in `keys` (-1 past the end).
__device__ __forceinline__ void warp_hist(const int32_t* idx, const uint8_t* bits, int n, int E,
                                          int nbins, int32_t* hist_s, int32_t* status,
                                          int (&keys)[kSlices]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int base = blockIdx.x * kCH + warp * 32 * kSlices;
#pragma unroll
  for (int u = 0; u < kSlices; ++u) {
    const int a = base + 32 * u + lane;
    keys[u] = a < n ? load_key(idx, bits, a, E, status) : -1;
  }
  int32_t* my = hist_s + warp * nbins;
#pragma unroll
  for (int u = 0; u < kSlices; ++u) {
    const unsigned peers = __match_any_sync(0xffffffffu, keys[u]);
    if (keys[u] >= 0 && (peers & lt_mask) == 0) my[keys[u]] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kWarps * 32) k_perm_hist(const int32_t* __restrict__ idx,
                                                           const uint8_t* __restrict__ bits, int n,
                                                           int E, int nbins,
                                                           int32_t* __restrict__ hist,
                                                           int32_t* status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t hist_s[];  // [kWarps][nbins]
  for (int i = threadIdx.x; i < kWarps * nbins; i += blockDim.x) hist_s[i] = 0;
  __syncthreads();
  int keys[kSlices];
  warp_hist(idx, bits, n, E, nbins, hist_s, status, keys);
  __syncthreads();
  for (int b = threadIdx.x; b < nbins; b += blockDim.x) {
    int c = 0;
    for (int w = 0; w < kWarps; ++w) c += hist_s[w * nbins + b];
    hist[static_cast<size_t>(b) * gridDim.x + blockIdx.x] = c;
  }
}

__global__ void __launch_bounds__(1024) k_perm_scan(int32_t* __restrict__ hist, int ctas, int nbins,
                                                    int n, int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t total_s[kMaxBins];
  __shared__ int32_t scan_buf[32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 1. a warp per bin: exclusive scan of the bin's per-CTA counts (32 CTAs
  //    per step, shuffle scan, running carry), and the bin total
  for (int bin = warp; bin < nbins; bin += 32) {
    int32_t* row = hist + static_cast<size_t>(bin) * ctas;
    int carry = 0;
    for (int c0 = 0; c0 < ctas; c0 += 32) {
      const int c = c0 + lane;
      const int v = c < ctas ? row[c] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (c < ctas) row[c] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      total_s[bin] = carry;
      counts[bin] = carry;
    }
  }
  __syncthreads();
  // 2. block scan of the bin totals (thread = bin) -> offsets
  const int total = tid < nbins ? total_s[tid] : 0;
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scan_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = scan_buf[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    scan_buf[lane] = v;
  }
  __syncthreads();
  const int excl = incl - total + (warp > 0 ? scan_buf[warp - 1] : 0);
  if (tid < nbins) {
    offsets[tid] = excl;
    total_s[tid] = excl;
  }
  if (tid == 0) offsets[nbins] = n;
  __syncthreads();
  // 3. a warp per bin: add the bin's offset to its per-CTA starts
  for (int bin = warp; bin < nbins; bin += 32) {
    int32_t* row = hist + static_cast<size_t>(bin) * ctas;
    const int off = total_s[bin];
    for (int c = lane; c < ctas; c += 32) row[c] += off;
  }
}

// Scatter of this CTA's assignments once hist_s[w][b] holds the first
// position of warp w's keys in bin b.
__device__ __forceinline__ void scatter(const int (&keys)[kSlices], int32_t* hist_s, int nbins,
                                        int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
                                        int32_t* perm_s = nullptr) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  int32_t* my = hist_s + warp * nbins;
  const int base = blockIdx.x * kCH + warp * 32 * kSlices;
#pragma unroll
  for (int u = 0; u < kSlices; ++u) {
    const int a = base + 32 * u + lane;
    const int key = keys[u];
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (key >= 0) {
      const int p = my[key] + __popc(peers & lt_mask);
      perm[p] = a;
      inv_perm[a] = p;
      if (perm_s) perm_s[p] = a;  // single-CTA path: a copy for the gather
    }
    __syncwarp();
    if (key >= 0 && (peers & lt_mask) == 0) my[key] += __popc(peers);
    __syncwarp();
  }
}

// x_perm[p] = fp16(x[perm[p] / k]) for rows p = first, first + stride, ...:
// a warp per destination row, 16-byte loads, four in flight per lane.
// Returns whether any value was outside the fp16 range.
__device__ __forceinline__ bool gather_rows(const __nv_bfloat16* __restrict__ x, const int32_t* perm, int rows,
                                            int k, int d, __half* __restrict__ x_perm, int first, int stride) {
  const int lane = threadIdx.x & 31;
  const int vec = d / 8;
  bool bad = false;
  for (int p = first; p < rows; p += stride) {
    const int t = perm[p] / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(p) * d);
    for (int c0 = lane; c0 < vec; c0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (c0 + 32 * q < vec) v[q] = src[c0 + 32 * q];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (c0 + 32 * q >= vec) break;
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v[q]);
        uint4 o;
        __half2* h2 = reinterpret_cast<__half2*>(&o);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(b2[j]);
          bad |= fabsf(f.x) > 65504.0f || fabsf(f.y) > 65504.0f;
          h2[j] = __floats2half2_rn(f.x, f.y);
        }
        dst[c0 + 32 * q] = o;
      }
    }
  }
  return bad;
}

// The gather as its own grid-wide launch (large batches).
__global__ void __launch_bounds__(256) k_gather(const __nv_bfloat16* __restrict__ x,
                                                 const int32_t* __restrict__ perm, int rows, int k,
                                                 int d, __half* __restrict__ x_perm,
                                                 int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int first = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int stride = (gridDim.x * blockDim.x) >> 5;
  if (gather_rows(x, perm, rows, k, d, x_perm, first, stride)) flag_status(status, MOE_DEV_RANGE);
}

__global__ void __launch_bounds__(kWarps * 32) k_perm_scatter(
    const int32_t* __restrict__ idx, const uint8_t* __restrict__ bits, int n, int E, int nbins, int k,
    const int32_t* __restrict__ hist, int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t hist_s[];  // [kWarps][nbins] -> per-warp start positions
  for (int i = threadIdx.x; i < kWarps * nbins; i += blockDim.x) hist_s[i] = 0;
  __syncthreads();
  int keys[kSlices];
  warp_hist(idx, bits, n, E, nbins, hist_s, nullptr, keys);
  __syncthreads();
  for (int b = threadIdx.x; b < nbins; b += blockDim.x) {
    int start = hist[static_cast<size_t>(b) * gridDim.x + blockIdx.x];
    for (int w = 0; w < kWarps; ++w) {
      const int c = hist_s[w * nbins + b];
      hist_s[w * nbins + b] = start;
      start += c;
    }
  }
  __syncthreads();
  scatter(keys, hist_s, nbins, perm, inv_perm);
}

// All of it in one CTA when the assignments fit one chunk (n <= 1024): the
// bin totals are scanned in the block, so no workspace round trip and one
// launch instead of three.
__global__ void __launch_bounds__(kWarps * 32) k_perm_one(
    const int32_t* __restrict__ idx, const uint8_t* __restrict__ bits, int n, int E, int nbins, int k,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv_perm, int32_t* status, const __nv_bfloat16* __restrict__ x, int d,
    __half* __restrict__ x_perm) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t hist_s[];  // [kWarps][nbins]
  __shared__ int32_t warp_sum[kWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kWarps * nbins; i += blockDim.x) hist_s[i] = 0;
  __syncthreads();
  int keys[kSlices];
  warp_hist(idx, bits, n, E, nbins, hist_s, status, keys);
  __syncthreads();
  // thread t owns bins [t * per, t * per + per): total, then a block scan
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  const int b0 = tid * per;
  int own = 0;
  for (int i = 0; i < per; ++i) {
    const int b = b0 + i;
    if (b < nbins) {
      int c = 0;
      for (int w = 0; w < kWarps; ++w) c += hist_s[w * nbins + b];
      counts[b] = c;
      own += c;
    }
  }
  int incl = own;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += warp_sum[w];
  int start = before + incl - own;
  for (int i = 0; i < per; ++i) {
    const int b = b0 + i;
    if (b < nbins) {
      offsets[b] = start;
      for (int w = 0; w < kWarps; ++w) {
        const int c = hist_s[w * nbins + b];
        hist_s[w * nbins + b] = start;
        start += c;
      }
    }
  }
  if (tid == 0) offsets[nbins] = n;
  __syncthreads();
  __shared__ int32_t perm_s[kCH];  // n <= kCH here
  scatter(keys, hist_s, nbins, perm, inv_perm, perm_s);
  if (x_perm) {  // small batches: the gather too, from the block's copy of perm
    __syncthreads();
    if (gather_rows(x, perm_s, n, k, d, x_perm, warp, kWarps)) flag_status(status, MOE_DEV_RANGE);
  }
}

int sm_count_permute() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

size_t permute_workspace_bytes(int T, int k, int nbins) {
  const long n = static_cast<long>(T) * k;
  const long ctas = std::max<long>(1, (n + kCH - 1) / kCH);
  return static_cast<size_t>(std::max<long>(256, ctas * nbins * 4));
}

moe_status_t launch_permute(const int32_t* idx, const uint8_t* bits, const void* x, int T, int d,
                            int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* inv_perm, void* x_perm, int32_t* status, void* workspace,
                            cudaStream_t s) {
  const int n = T * k;
  const int nbins = bits ? 3 * E : E;
  if (nbins > kMaxBins) {
    set_error("moe_permute: %d bins exceed %d", nbins, kMaxBins);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  const int ctas = std::max(1, (n + kCH - 1) / kCH);
  int32_t* hist = static_cast<int32_t*>(workspace);
  const size_t smem = sizeof(int32_t) * kWarps * nbins;
  // The shared-memory opt-in is a per-device function attribute: set it once
  // per device, to the largest bin count.
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "moe_permute cudaGetDevice");
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    const int cap = static_cast<int>(sizeof(int32_t) * kWarps * kMaxBins);
    e = cudaFuncSetAttribute(k_perm_hist, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_perm_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_perm_one, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
    if (e != cudaSuccess) return cuda_check(e, "moe_permute smem attribute");
    attr_set.fetch_or(bit);
  }
  moe_status_t st;
  // one CTA gathers the rows itself when they are few (up to 64 K elements:
  // decode-sized batches), which saves the gather launch
  const bool fused_gather = ctas == 1 && x_perm && static_cast<long>(n) * d <= (64L << 10);
  if (ctas == 1) {
    st = cuda_check(launch_pdl(pdl_for(n), k_perm_one, dim3(1), dim3(kWarps * 32), smem, s, idx, bits, n, E, nbins, k, counts,
                               offsets, perm, inv_perm, status, static_cast<const __nv_bfloat16*>(x), d,
                               fused_gather ? static_cast<__half*>(x_perm) : static_cast<__half*>(nullptr)),
                    "moe_permute launch");
  } else {
    st = cuda_check(launch_pdl(pdl_for(n), k_perm_hist, dim3(ctas), dim3(kWarps * 32), smem, s, idx, bits, n, E, nbins, hist, status),
                    "moe_permute histogram launch");
    if (st != MOE_OK) return st;
    st = cuda_check(launch_pdl(pdl_for(n), k_perm_scan, dim3(1), dim3(1024), 0, s, hist, ctas, nbins, n, counts, offsets),
                    "moe_permute scan launch");
    if (st != MOE_OK) return st;
    st = cuda_check(launch_pdl(pdl_for(n), k_perm_scatter, dim3(ctas), dim3(kWarps * 32), smem, s, idx, bits, n, E, nbins, k,
                               static_cast<const int32_t*>(hist), perm, inv_perm),
                    "moe_permute scatter launch");
  }
  if (st != MOE_OK || !x_perm || n == 0 || fused_gather) return st;
  // a warp per row: up to 8 rows per block, at most 8 blocks per SM
  const int blocks = std::max(1, std::min((n + 7) / 8, 8 * sm_count_permute()));
  return cuda_check(launch_pdl(pdl_for(n), k_gather, dim3(blocks), dim3(256), 0, s, static_cast<const __nv_bfloat16*>(x),
                                static_cast<const int32_t*>(perm), n, k, d, static_cast<__half*>(x_perm), status),
                    "moe_permute gather launch");
}

}  // namespace moeq
