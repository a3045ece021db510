// Per-expert histogram, exclusive prefix sum and stable permutation of the
// T*k assignments, then the gather of activation rows into expert order.
//
// One CTA of 32 warps sorts all assignments without atomics:
//   pass 1  warp w counts the keys of its contiguous chunk; inside a
//           32-assignment slice the lanes with equal keys are found with
//           __match_any_sync and the lowest of them adds the group size to
//           the warp's private histogram row;
//   scan    thread b turns column b of the [warps][bins] histogram into
//           per-warp start positions and the bin total; a block scan of
//           the totals gives offsets;
//   pass 2  warp w re-reads its chunk; a lane's position is its warp's
//           cursor for the key plus the number of lower lanes with the same
//           key in the slice, so the order inside a bin is ascending a.
#include <algorithm>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kWarps = 32;
constexpr int kMaxBins = 768;
constexpr int kBatch = 16;  // 32-assignment slices whose keys are loaded together

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

__global__ void __launch_bounds__(kWarps * 32) k_permute(const int32_t* __restrict__ idx,
                                                          const uint8_t* __restrict__ bits, int n,
                                                          int E, int nbins,
                                                          int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv_perm,
                                                          int32_t* status, int stage_perm) {
  extern __shared__ int32_t hist[];  // [kWarps][nbins], then perm staging [n] when stage_perm
  int32_t* perm_s = hist + kWarps * nbins;
  __shared__ int32_t scan_buf[kWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned lt_mask = (1u << lane) - 1u;

  for (int i = tid; i < kWarps * nbins; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  const int chunk = ((n + kWarps - 1) / kWarps + 31) & ~31;
  const int begin = warp * chunk;
  const int end = min(n, begin + chunk);
  int32_t* my = hist + warp * nbins;

  // Keys are fetched kBatch slices at a time (independent loads in flight),
  // then consumed slice by slice.
  for (int base = begin; base < end; base += 32 * kBatch) {
    int keys[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int a = base + 32 * u + lane;
      keys[u] = a < end ? load_key(idx, bits, a, E, status) : -1;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const unsigned peers = __match_any_sync(0xffffffffu, keys[u]);
      if (keys[u] >= 0 && (peers & lt_mask) == 0) my[keys[u]] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();

  // Column scan over warps: start of warp w inside bin b, and bin totals.
  int total = 0;
  if (tid < nbins) {
    for (int w = 0; w < kWarps; ++w) {
      const int c = hist[w * nbins + tid];
      hist[w * nbins + tid] = total;
      total += c;
    }
    counts[tid] = total;
  }
  // Block-wide exclusive scan of the bin totals (nbins <= 1024 threads).
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
    scan_buf[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - total + (warp > 0 ? scan_buf[warp - 1] : 0);
  if (tid < nbins) {
    offsets[tid] = excl;
    for (int w = 0; w < kWarps; ++w) hist[w * nbins + tid] += excl;
  }
  if (tid == 0) offsets[nbins] = n;
  __syncthreads();

  for (int base = begin; base < end; base += 32 * kBatch) {
    int keys[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int a = base + 32 * u + lane;
      keys[u] = a < end ? load_key(idx, bits, a, E, nullptr) : -1;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int a = base + 32 * u + lane;
      const int key = keys[u];
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      if (key >= 0) {
        const int p = my[key] + __popc(peers & lt_mask);
        if (stage_perm) perm_s[p] = a; else perm[p] = a;
        inv_perm[a] = p;
      }
      __syncwarp();
      if (key >= 0 && (peers & lt_mask) == 0) my[key] += __popc(peers);
      __syncwarp();
    }
  }
  if (stage_perm) {  // scattered positions land in shared memory; write out coalesced
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) perm[i] = perm_s[i];
  }
}

// x_perm[p] = fp16(x[perm[p] / k]); a warp moves one row, 16 bytes per lane
// per step with up to four independent loads in flight.
__global__ void __launch_bounds__(256) k_gather(const __nv_bfloat16* __restrict__ x,
                                                 const int32_t* __restrict__ perm, int rows, int k,
                                                 int d, __half* __restrict__ x_perm,
                                                 int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int vec = d / 8;
  bool bad = false;
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < rows; p += (gridDim.x * blockDim.x) >> 5) {
    const int t = perm[p] / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(p) * d);
    for (int c0 = lane; c0 < vec; c0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < vec) v[u] = src[c0 + 32 * u];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (c0 + 32 * u >= vec) break;
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
        uint4 o;
        __half2* h2 = reinterpret_cast<__half2*>(&o);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(b2[j]);
          bad |= fabsf(f.x) > 65504.0f || fabsf(f.y) > 65504.0f;
          h2[j] = __floats2half2_rn(f.x, f.y);
        }
        dst[c0 + 32 * u] = o;
      }
    }
  }
  if (bad) flag_status(status, MOE_DEV_RANGE);
}

}  // namespace

moe_status_t launch_permute(const int32_t* idx, const uint8_t* bits, const void* x, int T, int d,
                            int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* inv_perm, void* x_perm, int32_t* status, cudaStream_t s) {
  const int n = T * k;
  const int nbins = bits ? 3 * E : E;
  if (nbins > kMaxBins) {
    set_error("moe_permute: %d bins exceed %d", nbins, kMaxBins);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  // Shared memory: per-warp histograms, plus the permutation itself when it
  // fits, so that its scattered positions are written to shared memory and
  // leave the SM as coalesced rows.
  constexpr size_t kSmemCap = 226 * 1024;  // 227 KB per block, less the static scan buffer
  const size_t hist_bytes = sizeof(int32_t) * kWarps * nbins;
  const int stage = hist_bytes + sizeof(int32_t) * static_cast<size_t>(n) <= kSmemCap;
  const size_t smem = hist_bytes + (stage ? sizeof(int32_t) * static_cast<size_t>(n) : 0);
  static bool attr_set = false;  // once per process, to the cap
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemCap));
    if (e != cudaSuccess) return cuda_check(e, "moe_permute smem attribute");
    attr_set = true;
  }
  k_permute<<<1, kWarps * 32, smem, s>>>(idx, bits, n, E, nbins, counts, offsets, perm, inv_perm,
                                         status, stage);
  moe_status_t st = cuda_check(cudaGetLastError(), "moe_permute launch");
  if (st != MOE_OK || !x_perm || n == 0) return st;
  const int blocks = static_cast<int>(std::min<long>((static_cast<long>(n) + 7) / 8, 148L * 8));
  k_gather<<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), perm, n, k, d,
                                  static_cast<__half*>(x_perm), status);
  return cuda_check(cudaGetLastError(), "moe_permute gather launch");
}

}  // namespace moeq
