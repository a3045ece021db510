// Shared device/host helpers of the moeq library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <utility>
#include <stdint.h>

#include "moeq.h"

namespace moeq {

// Thread-local error message (set by the API layer).
void set_error(const char* fmt, ...);
moe_status_t cuda_check(cudaError_t e, const char* what);

// Byte offsets of each section inside one expert blob (format documented
// in moeq.h).
struct BlobLayout {
  size_t codes[3];   // INT4 codes of gate, up, down
  size_t q2[3];      // PLANES: Q2 of gate, up, down
  size_t d3[3];
  size_t d4[3];
  size_t sz[3];      // (scale, zero) words of gate, up, down
  size_t bytes;
  int valid;
};
BlobLayout blob_layout(int d, int F, int group, int layout);

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ void flag_status(int32_t* status, unsigned bits) {
  if (status) atomicOr(reinterpret_cast<unsigned*>(status), bits);
}

// Programmatic dependent launch.  Every kernel of the path is launched
// with launch_pdl: it may be scheduled while the previous kernel on the
// stream still runs, and waits (pdl_wait) before it touches memory that an
// earlier kernel writes or reads; pdl_trigger lets the next kernel be
// scheduled.  A kernel triggers only after its own wait, so anything
// written two or more launches back is complete once a kernel has started.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// Byte offset, inside a blob's code region (INT4 codes, Q2, D3 or D4), of
// byte b of row `row`: the region stores tiles of 16 rows x 128 K, `tb`
// bytes per tile row (64 INT4, 32 Q2, 16 D3 / D4), row-major inside a tile,
// the tiles of a 16-row block in K order, then the next block.  A piece of
// at most 16 bytes starting 16-byte aligned stays inside one tile row.
__host__ __device__ __forceinline__ size_t code_byte(size_t row, size_t b, int K, int tb) {
  return ((row >> 4) * static_cast<size_t>(K / 128) + b / tb) * (16 * static_cast<size_t>(tb)) + (row & 15) * tb +
         b % tb;
}

// Order-preserving unsigned key of an fp32 value (a > b gives key(a) >
// key(b); -0 sorts below +0); NaN gets 0, below every other key.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(v);
  return v == v ? ((b & 0x80000000u) ? ~b : (b | 0x80000000u)) : 0u;
}

// SiLU in fp32: v / (1 + exp(-v)).
__device__ __forceinline__ float silu_f(float v) { return v / (1.0f + __expf(-v)); }

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// fp64 dot product of a bf16 row and an fp32 row (d % 8 == 0) by one warp: lanes over 8-element pieces
// of d, four pieces' loads issued before their FMAs, then a shuffle tree.
__device__ __forceinline__ double dot_bf16_f32_fp64(const __nv_bfloat16* x, const float* w, int d, int lane) {
  double a = 0.0;
  for (int i0 = lane * 8; i0 < d; i0 += 4 * 256) {
    uint4 xv[4];
    float4 w0[4], w1[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * 256;
      if (i < d) {
        xv[u] = *reinterpret_cast<const uint4*>(x + i);
        w0[u] = *reinterpret_cast<const float4*>(w + i);
        w1[u] = *reinterpret_cast<const float4*>(w + i + 4);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (i0 + u * 256 >= d) break;
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xv[u]);
      const float wv[8] = {w0[u].x, w0[u].y, w0[u].z, w0[u].w, w1[u].x, w1[u].y, w1[u].z, w1[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(b2[j]);
        a = fma(static_cast<double>(f.x), static_cast<double>(wv[2 * j]), a);
        a = fma(static_cast<double>(f.y), static_cast<double>(wv[2 * j + 1]), a);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  return a;
}


// ---- fp64 dot products of a thread-block cluster (decode-sized batches) --
//
// For a handful of rows the exact-decision dot products (router logits,
// bit-width scores) are cheapest straight in fp64: every product of a bf16
// and an fp32 is exact there, and the few thousand FMAs per row spread over
// a cluster of kClusterSlices CTAs, one slice of d each.  Partial sums go
// into CTA 0's shared memory (distributed shared memory of the cluster);
// after a cluster barrier CTA 0 adds them in slice order.
constexpr int kClusterSlices = 8;
constexpr int kClusterItems = 512;  // rows pairs of one launch (CTA 0 holds 8 x 512 fp64 partials)

__device__ __forceinline__ uint32_t cluster_map_shared(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, int v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}
// every CTA of the cluster has started (its shared memory may be written)
__device__ __forceinline__ void cluster_sync_start() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
// the stores of every CTA before the barrier are visible after it
__device__ __forceinline__ void cluster_sync_publish() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Slice partials of n dot products by one CTA: item i pairs the bf16 row
// and the fp32 row that rows(i, xr, wr) names, over elements [k0, k0 + dk)
// (k0, dk multiples of 8, rows 16-byte aligned).  Warp w takes items w,
// w + warps, ..., eight at a time: their row pointers are resolved once,
// then chunk by chunk (256 elements) the eight items' pieces are loaded
// together.  A lane takes the 8-element pieces k0 + 256 c + 8 lane, sums
// each with an fp64 FMA chain from zero and adds the piece sums in chunk
// order; the warp adds the lane sums in a shuffle tree (every lane ends
// with the same value).  Lane 0 stores item i's partial at shared::cluster
// address dst + 8 i.  The order of operations does not depend on the item,
// so identical rows give identical partials.
template <typename RowFn>
__device__ __forceinline__ void cluster_partial_dots(int n, int k0, int dk, RowFn rows, uint32_t dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int mine = n > warp ? (n - warp + nw - 1) / nw : 0;
  for (int q0 = 0; q0 < mine; q0 += 8) {
    const int gi = min(8, mine - q0);
    const __nv_bfloat16* xr[8];
    const float* wr[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      xr[j] = nullptr;
      wr[j] = nullptr;
      if (j < gi) rows(warp + nw * (q0 + j), xr[j], wr[j]);
    }
    double acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0;
    for (int off = lane * 8; off < dk; off += 256) {
      uint4 xb[8];
      float4 wa[8], wb[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < gi) {
          xb[j] = *reinterpret_cast<const uint4*>(xr[j] + k0 + off);
          wa[j] = *reinterpret_cast<const float4*>(wr[j] + k0 + off);
          wb[j] = *reinterpret_cast<const float4*>(wr[j] + k0 + off + 4);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < gi) {
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb[j]);
          const float w[8] = {wa[j].x, wa[j].y, wa[j].z, wa[j].w, wb[j].x, wb[j].y, wb[j].z, wb[j].w};
          double s = 0.0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(b2[q]);
            s = fma(static_cast<double>(f.x), static_cast<double>(w[2 * q]), s);
            s = fma(static_cast<double>(f.y), static_cast<double>(w[2 * q + 1]), s);
          }
          acc[j] += s;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < gi) {  // warp-uniform
        double a = acc[j];
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) st_cluster_f64(dst + 8u * static_cast<uint32_t>(warp + nw * (q0 + j)), a);
      }
    }
  }
}

// fp32 slice partials of n dot products by one CTA, with the sum of the
// products' magnitudes for the error bound: as cluster_partial_dots, but a
// lane sums all its products of the slice in one fp32 FMA chain (pieces in
// chunk order) and the warp adds the lane sums in a 5-level shuffle tree,
// so |S - s| <= g(m) A with m = (products per lane) + 5 and A the exact sum
// of magnitudes (the computed A errs by the same relative g(m)).  Lane 0
// stores (S, A) as a float2 at shared::cluster address dst + 8 i.
__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
template <typename RowFn>
__device__ __forceinline__ void cluster_partial_dots_f32(int n, int k0, int dk, RowFn rows, uint32_t dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int mine = n > warp ? (n - warp + nw - 1) / nw : 0;
  for (int q0 = 0; q0 < mine; q0 += 8) {
    const int gi = min(8, mine - q0);
    const __nv_bfloat16* xr[8];
    const float* wr[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      xr[j] = nullptr;
      wr[j] = nullptr;
      if (j < gi) rows(warp + nw * (q0 + j), xr[j], wr[j]);
    }
    float acc[8], mag[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = mag[j] = 0.0f;
    for (int off = lane * 8; off < dk; off += 256) {
      uint4 xb[8];
      float4 wa[8], wb[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < gi) {
          xb[j] = *reinterpret_cast<const uint4*>(xr[j] + k0 + off);
          wa[j] = *reinterpret_cast<const float4*>(wr[j] + k0 + off);
          wb[j] = *reinterpret_cast<const float4*>(wr[j] + k0 + off + 4);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < gi) {
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb[j]);
          const float w[8] = {wa[j].x, wa[j].y, wa[j].z, wa[j].w, wb[j].x, wb[j].y, wb[j].z, wb[j].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(b2[q]);
            acc[j] = fmaf(f.x, w[2 * q], acc[j]);
            mag[j] = fmaf(fabsf(f.x), fabsf(w[2 * q]), mag[j]);
            acc[j] = fmaf(f.y, w[2 * q + 1], acc[j]);
            mag[j] = fmaf(fabsf(f.y), fabsf(w[2 * q + 1]), mag[j]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < gi) {  // warp-uniform
        float a = acc[j], m = mag[j];
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          a += __shfl_xor_sync(0xffffffffu, a, o);
          m += __shfl_xor_sync(0xffffffffu, m, o);
        }
        if (lane == 0) st_cluster_f32x2(dst + 8u * static_cast<uint32_t>(warp + nw * (q0 + j)), a, m);
      }
    }
  }
}

// The k largest of E values in shared memory, in descending order,
// ties to the lower index, by one warp: each lane ranks its values
// e = lane + 32 m against all E (independent compares, no dependent
// chains) and the value of rank r < k writes its index to sel[r] (shared
// memory).  NaN values are never picked; if fewer than k values are
// comparable the remaining picks are expert 0 (the selection order of the
// warp-shuffle top-k, which takes the first maximum k times).
template <typename V>
__device__ __forceinline__ void warp_topk_rank(const V* vals, int E, int k, int lane, int32_t* sel) {
  int comparable = 0;
  for (int e = lane; e < E; e += 32) {
    const V v = vals[e];
    comparable += v == v ? 1 : 0;
    if (v != v) continue;
    int rank = 0;
    for (int o = 0; o < E; ++o) {
      const V u = vals[o];  // NaN: both compares false
      rank += (u > v || (u == v && o < e)) ? 1 : 0;
    }
    if (rank < k) sel[rank] = e;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) comparable += __shfl_xor_sync(0xffffffffu, comparable, o);
  for (int r = comparable + lane; r < k; r += 32) sel[r] = 0;
  __syncwarp();
}

// Bound factor of the fp32 cluster paths: g(m + 9), m = products per lane
// of a d-slice + 5 (tree levels); + 8 for the sum over the slices and 1 for
// the bias.
inline float cluster_gamma(int d) {
  const double u = 1.0 / 16777216.0;
  const double m = 8.0 * ((d / kClusterSlices + 255) / 256) + 5.0 + 9.0;
  return static_cast<float>(m * u / (1.0 - m * u));
}

// The bit-width gate of the smallest batches over one cluster (every CTA
// calls it after cluster_sync_start): the 3 T k width scores as fp32 slice
// partials with magnitude sums (cluster_partial_dots_f32) into CTA 0, which
// picks each assignment's width (first maximum, equal scores to the narrower
// width) when the winner's lower bound clears the others' upper bounds,
//   |L[c] - l[c]| <= D[c] = 2 g (A[c] (1 + 2^-8) + |b[c]|),  g = cluster_gamma(d);
// the assignments it leaves open are listed (CTA 0 writes the list into
// every CTA before the barrier), their scores recomputed in fp64 over the
// cluster and decided on those.  ids: the assignments' experts, in range,
// readable by every CTA.  Widths to bits (global) and, if given, bits_s
// (CTA 0's shared memory).
struct TinyGateSmem {
  float2 p32[kClusterSlices * 3 * 32];
  double p64[kClusterSlices * 3 * 32];
  int32_t cand[32];
  int32_t n_cand;
};
__device__ __forceinline__ void tiny_bit_gate(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wb,
                                              const float* __restrict__ bb, const int32_t* ids, int T, int d,
                                              int k, float gamma, uint8_t* bits, uint8_t* bits_s,
                                              TinyGateSmem& S) {
  const int rank = blockIdx.x;  // the grid is one cluster
  const int na = T * k, n = 3 * na, dk = d / kClusterSlices;
  if (threadIdx.x == 0) S.n_cand = 0;
  cluster_partial_dots_f32(
      n, rank * dk, dk,
      [&](int i, const __nv_bfloat16*& xr, const float*& w) {
        const int a = i / 3;
        xr = x + static_cast<size_t>(a / k) * d;
        w = wb + (static_cast<size_t>(ids[a]) * 3 + (i - 3 * a)) * d;
      },
      cluster_map_shared(S.p32, 0) + 8u * static_cast<uint32_t>(rank * n));
  cluster_sync_publish();
  if (rank == 0) {
    for (int a = threadIdx.x; a < na; a += blockDim.x) {
      float L[3], D[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        float s = 0.0f, m = 0.0f;
        for (int r = 0; r < kClusterSlices; ++r) {
          const float2 p = S.p32[r * n + 3 * a + c];
          s += p.x;
          m += p.y;
        }
        const float b = bb ? bb[static_cast<size_t>(ids[a]) * 3 + c] : 0.0f;
        L[c] = s + b;
        D[c] = 2.0f * gamma * (m * (1.0f + 0.00390625f) + fabsf(b)) + 1e-30f;
      }
      int best = 0;
      if (L[1] > L[best]) best = 1;
      if (L[2] > L[best]) best = 2;
      bool sure = true;  // comparisons with NaN are false: non-finite scores go to fp64
#pragma unroll
      for (int c = 0; c < 3; ++c)
        if (c != best) sure = sure && L[best] - D[best] > L[c] + D[c];
      if (sure) {
        bits[a] = static_cast<uint8_t>(2 + best);
        if (bits_s) bits_s[a] = static_cast<uint8_t>(2 + best);
      } else {
        S.cand[atomicAdd(&S.n_cand, 1)] = a;
      }
    }
    __syncthreads();  // the list is complete
    const int nc = S.n_cand;
    for (int r = 1; r < kClusterSlices; ++r) {
      for (int i = threadIdx.x; i < nc; i += blockDim.x) st_cluster_u32(cluster_map_shared(&S.cand[i], r), S.cand[i]);
      if (threadIdx.x == 0) st_cluster_u32(cluster_map_shared(&S.n_cand, r), nc);
    }
  }
  cluster_sync_publish();  // the list is in every CTA
  const int n3 = S.n_cand;
  if (n3 == 0) return;  // cluster-uniform
  cluster_partial_dots(
      3 * n3, rank * dk, dk,
      [&](int i, const __nv_bfloat16*& xr, const float*& w) {
        const int a = S.cand[i / 3];
        xr = x + static_cast<size_t>(a / k) * d;
        w = wb + (static_cast<size_t>(ids[a]) * 3 + (i - 3 * (i / 3))) * d;
      },
      cluster_map_shared(S.p64, 0) + 8u * static_cast<uint32_t>(rank * 3 * n3));
  cluster_sync_publish();
  if (rank == 0) {
    for (int j = threadIdx.x; j < n3; j += blockDim.x) {
      const int a = S.cand[j];
      double v[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        double s = S.p64[3 * j + c];
        for (int r = 1; r < kClusterSlices; ++r) s += S.p64[r * 3 * n3 + 3 * j + c];
        v[c] = s + (bb ? static_cast<double>(bb[static_cast<size_t>(ids[a]) * 3 + c]) : 0.0);
      }
      int best = 0;
      if (v[1] > v[best]) best = 1;
      if (v[2] > v[best]) best = 2;
      bits[a] = static_cast<uint8_t>(2 + best);
      if (bits_s) bits_s[a] = static_cast<uint8_t>(2 + best);
    }
  }
}

// A launch of one thread-block cluster of `cluster` CTAs (grid = cluster),
// as a programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster_pdl(void (*kernel)(KArgs...), int cluster, dim3 block, size_t smem, cudaStream_t s,
                               Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(cluster);
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launchers (each returns MOE_OK or an error already recorded).
moe_status_t launch_pack(const float* w_gate, const float* w_up, const float* w_down, int E, int d,
                         int F, int group, int layout, void* blobs, cudaStream_t s);
moe_status_t launch_route(const void* x, const float* w_router, const float* bias,
                          const int32_t* forced, int T, int d, int E, int k, int32_t* idx,
                          float* w, void* workspace, size_t workspace_bytes, cudaStream_t s);
size_t route_workspace_bytes(int T, int d, int E);
extern int g_route_fused;  // test hook: 1 default, 0 no fp64 cluster paths
constexpr int kTinyGateAssign = 32;   // assignments of the cluster bit gate (T*k)
static_assert(kTinyGateAssign <= 32, "TinyGateSmem holds 32 assignments");
bool route_tiny_ok(int T, int d, int E);
bool route_permute_fusable(int T, int d, int E, int k, bool gate);
// Router (+ bit gate) (+ permutation and gather when counts is given) of the
// smallest batches in one cluster launch (front.cu).
moe_status_t launch_front_tiny(const void* x, const float* w_router, const float* bias, const int32_t* forced,
                               const uint8_t* bits_in, const float* w_bit, const float* bias_bit, int T, int d,
                               int E, int k, int32_t* idx, float* w, uint8_t* bits_out, int32_t* counts,
                               int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* x_perm, int32_t* status,
                               cudaStream_t s);
size_t route_min_workspace_bytes(int T, int d, int E);
moe_status_t route_check_args(const void* x, const float* w_router, int T, int d, int E, int k,
                              const int32_t* topk_idx, const float* topk_w, const char* fn);
moe_status_t launch_permute(const int32_t* idx, const uint8_t* bits, const void* x, int T, int d,
                            int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* inv_perm, void* x_perm, int32_t* status, void* workspace,
                            cudaStream_t s);
size_t permute_workspace_bytes(int T, int k, int nbins);
// early: the previous launch on the stream writes none of inv_perm, w and
// residual (they may be read before the programmatic wait).
moe_status_t launch_combine(const void* y_perm, const int32_t* inv_perm, const float* w,
                            const void* residual, int T, int k, int d, void* y, cudaStream_t s, bool early = false);

struct FfnArgs {
  const __half* x_perm;
  const int32_t* offsets;
  const uint8_t* blobs;
  const int32_t* slot_of;
  int total_rows, T, E, d, F, group, layout;
  size_t blob_bytes;
  BlobLayout lay;
  __half* h;          // workspace: fp16 [total_rows][F]
  __half* y_perm;  // [total_rows][d]
  int32_t* status;
};
moe_status_t launch_ffn_gemv(const FfnArgs& a, cudaStream_t s);
moe_status_t launch_ffn_gemv_mma(const FfnArgs& a, cudaStream_t s);
moe_status_t launch_ffn_decode(const FfnArgs& a, int token_blocks, cudaStream_t s);
moe_status_t launch_bit_gate(const void* x, const float* w_bit, const float* bias_bit, const int32_t* idx,
                             int T, int d, int E, int k, uint8_t* bits, int32_t* status, cudaStream_t s);
moe_status_t launch_static_bits(const int32_t* idx, const uint8_t* width_of, int n, int E, uint8_t* bits,
                                int32_t* status, cudaStream_t s);
moe_status_t launch_ffn_tc(const FfnArgs& a, cudaStream_t s);
bool tc_supported(const FfnArgs& a);

// Programmatic dependent launch pays off where launch latency dominates:
// decode-sized batches (measured: -3 us per layer step at 1 and 16 tokens).
// At 4096 tokens it slowed the step by ~4%, so large batches launch plainly
// (the kernels' pdl_wait / pdl_trigger are then no-ops).
inline bool pdl_for(long assignments) { return assignments <= 1024; }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moeq
