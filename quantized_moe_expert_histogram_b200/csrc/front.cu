// The front of the layer for the smallest batches in one launch of a
// thread-block cluster: the softmax top-k router ([ExactMoE] the router
// decides; [D2MoE] Dual Routing: expert gate), optionally the bit-width gate
// ([D2MoE] Token-Adaptive Bit-Width Selection) and the permutation with the
// gather ([Read-ME] expert-aware batching), with the results of the
// separate kernels (the same exact decisions).
//
// Dot products.  Every CTA of the cluster (kFC of them) takes one slice of
// d of every dot product the step needs -- the router's T*E (token, expert)
// logits and, with a bit gate, the 3 T*E (token, expert, width) scores of
// every expert, so that no second round is needed once the experts are
// chosen.  Four lanes share an item: each sums its 8-element pieces of the
// slice (pieces 4 p + lane % 4) with an fp32 FMA chain, the value and the
// sum of the products' magnitudes, and two shuffle levels add the four
// lanes; a warp holds eight such groups.  Where a group would get four or
// more tokens of one weight row, it takes the row and those tokens, loading
// the row's slice once.  The (value, magnitude) pairs go into CTA 0's
// shared memory (distributed shared memory of the cluster).
//
// Error bound.  A slice partial S of an item errs by at most g(m) A (m =
// products per lane + 2 tree levels, A the exact sum of magnitudes; the
// computed A errs by the same relative g(m)); CTA 0 adds the kFC partials and
// the bias in fp32 (kFC more additions), so with g = g(m + kFC + 1)
//     |L - l| <= D = 2 g (A (1 + 2^-8) + |b|)      (factor 2: margin).
//
// Decisions (CTA 0).  Router: a warp per token picks the top k one at a
// time by warp reductions over order keys of the logits (ties to the lower
// index), lane j holding pick j, and certifies the token when consecutive
// picks and the cut after the k-th are separated by more than their
// bounds.  Gate: the
// first maximum of the three widths of each chosen expert (ties to the
// narrower width), certified when the winner's lower bound clears the
// others' upper bounds.  What is left open -- the contenders of an open
// token (its picks and every expert whose upper bound reaches the lowest
// pick's lower bound), the three scores of an open assignment -- is listed;
// CTA 0 writes the list into every CTA's shared memory before the next
// barrier, the cluster computes the listed dot products in fp64 (every
// bf16 x fp32 product exact) and CTA 0 decides those on the fp64 values.
// The gates of an open token come from its fp64 logits, so its widths are
// decided after that round: on the fp32 scores when certified, otherwise by
// CTA 0 alone in fp64 (an open assignment of an open token).
//
// Permutation and gather.  When nothing was left open, CTA 0 sends the
// final picks (and widths) with the empty list; every CTA then ranks the
// assignments itself (counting, na <= 64) and gathers its eighth of the
// (row, 8-element piece) items, CTA 0 alone writing perm, inv_perm, counts
// and offsets.  After an fp64 round CTA 0 does both alone.
//
// Shared-memory rule of the cluster: a CTA writes into another CTA's shared
// memory only before a cluster barrier that the owner also waits at, and no
// CTA reads another CTA's shared memory.
#include <atomic>
#include <cmath>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kFC = 8;               // CTAs of the cluster (slices of d)
constexpr int kFThreads = 256;       // threads of a CTA
constexpr int kFWarps = kFThreads / 32;
constexpr int kFMaxT = 8;                 // tokens
constexpr int kFMaxTE = 512;              // T*E
constexpr int kFMaxGateTE = 128;          // T*E with a bit gate (4 T*E dot products)
constexpr int kFMaxTK = 64;               // T*k
constexpr int kFMaxItems = kFMaxTE > 4 * kFMaxGateTE ? kFMaxTE : 4 * kFMaxGateTE;  // router + gate dot products
constexpr int kFMaxList = kFMaxTE + 3 * kFMaxTK;

// Groups of four lanes (kFWarps * 8 of them) over the weight rows of the
// dot products: token chunks and tokens per group (front_dots32_rows).
__host__ __device__ constexpr int front_token_chunks(int T, int n_rows) {
  return (8 * kFWarps) / n_rows < 1 ? 1 : ((8 * kFWarps) / n_rows < T ? (8 * kFWarps) / n_rows : T);
}
// Row by row where a group gets at least this many tokens (OLMoE-shaped
// layer step, row by row against item by item: 2 tokens 32.8 / 32.0 us,
// 4 tokens 39.9 / 40.6, 8 tokens 51.3 / 54.3; nested with the bit gate, 4
// tokens 60.0 / 60.9, 8 tokens 104.6 / 106.3).
constexpr int kRowsMinTokens = 4;

struct FrontArgs {
  const __nv_bfloat16* x;
  const float* wr;
  const float* bias;
  const int32_t* forced;
  const float* wbit;       // bit gate, or null
  const float* bbit;
  const uint8_t* bits_in;  // widths given by the caller, or null
  int T, d, E, k;
  float gamma;
  int32_t* idx;
  float* gw;
  uint8_t* bits_out;
  int32_t* counts;         // permutation outputs: null for the router alone
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
  __half* x_perm;          // null: no gather
  int32_t* status;
};

// Shared memory of a CTA (only CTA 0 uses most of it).
struct FrontSmem {
  float2 p32[kFC * kFMaxItems];   // (value, magnitude) per slice and item
  double p64[kFC * kFMaxList];    // fp64 partials of the listed items
  float val[kFMaxTE];             // router logits (fp32 path)
  float dev[kFMaxTE];             // their bounds
  double v64[kFMaxTE];            // fp64 logits of open tokens
  double g64[3 * kFMaxTK];        // fp64 width scores of open assignments of open tokens
  int32_t list[kFMaxList];        // listed items
  int32_t lpos[kFMaxItems];       // item -> index in list, or -1
  int32_t sel[kFMaxTK];           // picks [T][k]
  int32_t key[kFMaxTK];
  int32_t perm[kFMaxTK];
  uint8_t bits[kFMaxTK];
  int32_t open[8];                // per token: not certified
  int32_t n_list;
  int32_t n_open;
};

// Item -> (token, weight row): router items it < TE are (t, e) = divmod(it,
// E); gate items are TE + 3 (t E + e) + c, width c of expert e.
__device__ __forceinline__ void front_rows(const FrontArgs& A, int TE, int it, const __nv_bfloat16*& xr,
                                           const float*& w) {
  if (it < TE) {
    const int t = it / A.E, e = it - t * A.E;
    xr = A.x + static_cast<size_t>(t) * A.d;
    w = A.wr + static_cast<size_t>(e) * A.d;
  } else {
    const int g = it - TE, te = g / 3, c = g - 3 * te, t = te / A.E, e = te - t * A.E;
    xr = A.x + static_cast<size_t>(t) * A.d;
    w = A.wbit + (static_cast<size_t>(e) * 3 + c) * A.d;
  }
}

// fp32 slice partials of items [0, n) into CTA 0's p32 (this CTA's slice),
// item by item: a group of four lanes per item, eight items per warp at a
// time (where every group has one token: the row-major form below would
// only add work).
__device__ __forceinline__ void front_dots32_items(const FrontArgs& A, int TE, int n, int k0, int dk, uint32_t dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, q = lane >> 2, l4 = lane & 3;
  const int pieces = dk / 32;  // 8-element pieces per lane
  for (int base = warp * 8; base < n; base += kFWarps * 8) {
    const int it = base + q;
    const bool live = it < n;
    const __nv_bfloat16* xr = A.x;
    const float* w = A.wr;
    if (live) front_rows(A, TE, it, xr, w);
    float acc = 0.0f, mag = 0.0f;
    for (int p0 = 0; p0 < pieces; p0 += 8) {
      uint4 xb[8];
      float4 wa[8], wb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int off = k0 + ((p0 + u) * 4 + l4) * 8;
        if (live && p0 + u < pieces) {
          xb[u] = *reinterpret_cast<const uint4*>(xr + off);
          wa[u] = *reinterpret_cast<const float4*>(w + off);
          wb[u] = *reinterpret_cast<const float4*>(w + off + 4);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (live && p0 + u < pieces) {
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb[u]);
          const float wv[8] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w, wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(b2[j]);
            acc = fmaf(f.x, wv[2 * j], acc);
            mag = fmaf(fabsf(f.x), fabsf(wv[2 * j]), mag);
            acc = fmaf(f.y, wv[2 * j + 1], acc);
            mag = fmaf(fabsf(f.y), fabsf(wv[2 * j + 1]), mag);
          }
        }
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      acc += __shfl_xor_sync(0xffffffffu, acc, o);
      mag += __shfl_xor_sync(0xffffffffu, mag, o);
    }
    if (live && l4 == 0) st_cluster_f32x2(dst + 8u * static_cast<uint32_t>(it), acc, mag);
  }
}

// fp32 slice partials of every item into CTA 0's p32 (this CTA's slice),
// row by row.  Weight rows: the router's e < E, then (bit gate) E + 3 e +
// c; the item of (token t, row r) is t E + r for the router and
// TE + 3 t E + (r - E) for the gate.  A group of four lanes takes one
// weight row and its tokens t = tc, tc + tch, ... < T <= kFMaxT (tch token
// chunks split the tokens over groups where there are fewer rows than
// groups), so each row's slice is loaded once and reused across its
// tokens.  Lanes of a group sum their
// 8-element pieces (4 p + lane % 4) with fp32 FMA chains, the value and the
// sum of the products' magnitudes; two shuffle levels add the four lanes.
__device__ __forceinline__ void front_dots32_rows(const FrontArgs& A, int TE, int n_rows, int k0, int dk,
                                                  uint32_t dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, l4 = lane & 3;
  const int T = A.T, E = A.E;
  const int pieces = dk / 32;  // 8-element pieces per lane
  constexpr int kGroups = kFWarps * 8;
  const int g = warp * 8 + (lane >> 2);
  const int tch = front_token_chunks(T, n_rows);      // token chunks
  const int rstride = kGroups / tch;                 // rows in flight
  const int tc = g % tch;
  const int rounds = (n_rows + rstride - 1) / rstride;  // uniform across the CTA
  for (int rd = 0; rd < rounds; ++rd) {
    const int r = g / tch + rd * rstride;
    const bool live = g < tch * rstride && r < n_rows;
    const float* w = live ? (r < E ? A.wr + static_cast<size_t>(r) * A.d : A.wbit + static_cast<size_t>(r - E) * A.d)
                          : A.wr;
    float acc[kFMaxT], mag[kFMaxT];
#pragma unroll
    for (int i = 0; i < kFMaxT; ++i) acc[i] = mag[i] = 0.0f;
    for (int p0 = 0; p0 < pieces; p0 += 8) {
      float4 wa[8], wb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int off = k0 + ((p0 + u) * 4 + l4) * 8;
        if (live && p0 + u < pieces) {
          wa[u] = *reinterpret_cast<const float4*>(w + off);
          wb[u] = *reinterpret_cast<const float4*>(w + off + 4);
        }
      }
#pragma unroll
      for (int i = 0; i < kFMaxT; ++i) {
        const int t = tc + i * tch;
        if (!live || t >= T) continue;
        const __nv_bfloat16* xr = A.x + static_cast<size_t>(t) * A.d;
        uint4 xb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (p0 + u < pieces) xb[u] = *reinterpret_cast<const uint4*>(xr + k0 + ((p0 + u) * 4 + l4) * 8);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (p0 + u < pieces) {
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb[u]);
            const float wv[8] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w, wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __bfloat1622float2(b2[j]);
              acc[i] = fmaf(f.x, wv[2 * j], acc[i]);
              mag[i] = fmaf(fabsf(f.x), fabsf(wv[2 * j]), mag[i]);
              acc[i] = fmaf(f.y, wv[2 * j + 1], acc[i]);
              mag[i] = fmaf(fabsf(f.y), fabsf(wv[2 * j + 1]), mag[i]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kFMaxT; ++i) {
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
        mag[i] += __shfl_xor_sync(0xffffffffu, mag[i], o);
      }
      const int t = tc + i * tch;
      if (live && t < T && l4 == 0) {
        const int it = r < E ? t * E + r : TE + 3 * t * E + (r - E);
        st_cluster_f32x2(dst + 8u * static_cast<uint32_t>(it), acc[i], mag[i]);
      }
    }
  }
}

// fp64 slice partials of the listed items into CTA 0's p64 (same layout of
// lanes; each product exact in fp64).
__device__ __forceinline__ void front_dots64(const FrontArgs& A, int TE, const int32_t* list, int n, int k0,
                                             int dk, uint32_t dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, q = lane >> 2, l4 = lane & 3;
  const int pieces = dk / 32;
  for (int base = warp * 8; base < n; base += kFWarps * 8) {
    const int j = base + q;
    const bool live = j < n;
    const __nv_bfloat16* xr = A.x;
    const float* w = A.wr;
    if (live) front_rows(A, TE, list[j], xr, w);
    double acc = 0.0;
    for (int p = 0; live && p < pieces; ++p) {
      const int off = k0 + (p * 4 + l4) * 8;
      const uint4 xb = *reinterpret_cast<const uint4*>(xr + off);
      const float4 wa = *reinterpret_cast<const float4*>(w + off);
      const float4 wb = *reinterpret_cast<const float4*>(w + off + 4);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb);
      const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(b2[u]);
        acc = fma(static_cast<double>(f.x), static_cast<double>(wv[2 * u]), acc);
        acc = fma(static_cast<double>(f.y), static_cast<double>(wv[2 * u + 1]), acc);
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (live && l4 == 0) st_cluster_f64(dst + 8u * static_cast<uint32_t>(j), acc);
  }
}

// CTA 0: every CTA's copy of the list and its length, written before the
// barrier that follows; when the list is empty the picks and, with a bit
// gate, the widths are final, and every CTA gets them too (the permutation
// is then computed by each CTA and the gather split over the cluster).
__device__ __forceinline__ void front_publish_list(FrontSmem& S, int n, int na, bool widths) {
  for (int r = 1; r < kFC; ++r) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) st_cluster_u32(cluster_map_shared(&S.list[i], r), S.list[i]);
    if (n == 0) {
      for (int i = threadIdx.x; i < na; i += blockDim.x)
        st_cluster_u32(cluster_map_shared(&S.sel[i], r), static_cast<uint32_t>(S.sel[i]));
      const uint32_t* b4 = reinterpret_cast<const uint32_t*>(S.bits);
      if (widths)
        for (int i = threadIdx.x; i < (na + 3) / 4; i += blockDim.x)
          st_cluster_u32(cluster_map_shared(&b4[i], r), b4[i]);
    }
    if (threadIdx.x == 0) st_cluster_u32(cluster_map_shared(&S.n_list, r), n);
  }
}

// Gates of token t (warp): softmax over its picks' logits; ids and gates to
// global memory.
template <typename V>
__device__ __forceinline__ void front_gates(const FrontArgs& A, const V* vals, const int32_t* sel, int t, int lane) {
  const int k = A.k;
  const bool mine = lane < k;
  const int e = mine ? sel[lane] : 0;
  const V lv = mine ? vals[e] : static_cast<V>(-INFINITY);
  V mx = lv;
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const V ex = mine ? exp(lv - mx) : static_cast<V>(0);
  V sum = ex;
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (mine) {
    A.idx[static_cast<size_t>(t) * k + lane] = e;
    A.gw[static_cast<size_t>(t) * k + lane] = static_cast<float>(ex / sum);
  }
}

// Width of assignment a (token t, expert e) on the fp32 scores: 2..4, or 0
// when not certified.
__device__ __forceinline__ int front_width32(const FrontArgs& A, const FrontSmem& S, int TE, int nitems, int t,
                                             int e) {
  float L[3], D[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const int it = TE + 3 * (t * A.E + e) + c;
    float s = 0.0f, m = 0.0f;
    for (int r = 0; r < kFC; ++r) {
      const float2 p = S.p32[r * nitems + it];
      s += p.x;
      m += p.y;
    }
    const float b = A.bbit ? A.bbit[static_cast<size_t>(e) * 3 + c] : 0.0f;
    L[c] = s + b;
    D[c] = 2.0f * A.gamma * (m * (1.0f + 0.00390625f) + fabsf(b)) + 1e-30f;
  }
  int best = 0;
  if (L[1] > L[best]) best = 1;
  if (L[2] > L[best]) best = 2;
  bool sure = true;  // NaN: comparisons false, not certified
#pragma unroll
  for (int c = 0; c < 3; ++c)
    if (c != best) sure = sure && L[best] - D[best] > L[c] + D[c];
  return sure ? 2 + best : 0;
}

__device__ __forceinline__ void front_set_width(const FrontArgs& A, FrontSmem& S, int a, int b) {
  S.bits[a] = static_cast<uint8_t>(b);
  A.bits_out[a] = static_cast<uint8_t>(b);
}

template <bool ROWS>
__global__ void __launch_bounds__(kFThreads) k_front(const __grid_constant__ FrontArgs A) {
  extern __shared__ __align__(16) uint8_t front_smem[];
  FrontSmem& S = *reinterpret_cast<FrontSmem*>(front_smem);
  const int rank = blockIdx.x;  // the grid is one cluster
  // CTA 0's biases of the logits it sums (items threadIdx.x and + 256; T E
  // <= 512), read before the wait: no kernel of the path writes them
  float bias0 = 0.0f, bias1 = 0.0f;
  if (rank == 0 && A.bias) {
    const int te = A.T * A.E;
    if (static_cast<int>(threadIdx.x) < te) bias0 = A.bias[threadIdx.x % A.E];
    if (static_cast<int>(threadIdx.x) + kFThreads < te) bias1 = A.bias[(threadIdx.x + kFThreads) % A.E];
  }
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = A.T, E = A.E, k = A.k, TE = T * E, na = T * k, dk = A.d / kFC;
  const bool gate = A.wbit != nullptr;
  const int nitems = gate ? 4 * TE : TE;
  if (threadIdx.x == 0) S.n_list = 0;
  cluster_sync_start();
  // ---- 1. fp32 slice partials of every dot product
  if (ROWS)
    front_dots32_rows(A, TE, gate ? 4 * E : E, rank * dk, dk,
                      cluster_map_shared(S.p32, 0) + 8u * static_cast<uint32_t>(rank * nitems));
  else
    front_dots32_items(A, TE, nitems, rank * dk, dk,
                       cluster_map_shared(S.p32, 0) + 8u * static_cast<uint32_t>(rank * nitems));
  cluster_sync_publish();
  // ---- 2. decisions on the fp32 values (CTA 0)
  if (rank == 0) {
    for (int i = threadIdx.x; i < TE; i += blockDim.x) {
      float L = 0.0f, m = 0.0f;
      for (int r = 0; r < kFC; ++r) {
        const float2 p = S.p32[r * nitems + i];
        L += p.x;
        m += p.y;
      }
      const float b = i < kFThreads ? bias0 : bias1;
      S.val[i] = L + b;
      S.dev[i] = 2.0f * A.gamma * (m * (1.0f + 0.00390625f) + fabsf(b)) + 1e-30f;
    }
    for (int i = threadIdx.x; i < nitems; i += blockDim.x) S.lpos[i] = -1;
    if (threadIdx.x < T) S.open[threadIdx.x] = 0;
    if (threadIdx.x == 0) S.n_open = 0;
    __syncthreads();
    if (A.forced) {
      for (int j = threadIdx.x; j < na; j += blockDim.x) {
        const int e = A.forced[j];
        S.sel[j] = e < 0 ? 0 : (e >= E ? E - 1 : e);
      }
    } else if (warp < T) {
      // warp t decides token t, lane j holding pick j; its experts lane + 32 m
      const int t = warp, P = (E + 31) >> 5;
      const float* lv = S.val + t * E;
      const float* dv = S.dev + t * E;
      // top k, one pick per round: the largest order key (NaN never picked),
      // then the lowest expert holding it; expert 0 where fewer than k
      // logits are comparable
      uint32_t taken = 0;
      int mine = 0;
      for (int j = 0; j < k; ++j) {
        uint32_t bk = 0;
        int be = 0x7fffffff;
        for (int m = 0; m < P; ++m) {
          const int e = lane + 32 * m;
          if (e < E && !((taken >> m) & 1u)) {
            const uint32_t key = order_key(lv[e]);
            if (key > bk) {
              bk = key;
              be = e;
            }
          }
        }
        const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
        int e = __reduce_min_sync(0xffffffffu, bk == top ? be : 0x7fffffff);
        if (top == 0) e = 0;
        else if ((e & 31) == lane) taken |= 1u << (e >> 5);
        if (lane == j) mine = e;
      }
      if (lane < k) S.sel[t * k + lane] = mine;
      // certified when consecutive picks are separated by more than their
      // bounds, every pick's lower bound is finite, and every expert not
      // picked stays below the k-th pick's lower bound (NaN: not certified)
      float lo = INFINITY, up = -INFINITY;
      if (lane < k) {
        lo = lv[mine] - dv[mine];
        up = lv[mine] + dv[mine];
      }
      const float lo_prev = __shfl_up_sync(0xffffffffu, lo, 1);
      const bool order_bad = lane > 0 && lane < k && !(lo_prev > up);
      const bool fin = __all_sync(0xffffffffu, lane >= k || (lo == lo && fabsf(lo) <= 3.0e38f));
      float lo_min = lo;
#pragma unroll
      for (int o = 16; o; o >>= 1) lo_min = fminf(lo_min, __shfl_xor_sync(0xffffffffu, lo_min, o));
      const float lo_k = __shfl_sync(0xffffffffu, lo, k - 1);
      bool cut_bad = false;
      for (int m = 0; m < P; ++m) {
        const int e = lane + 32 * m;
        if (e < E && !((taken >> m) & 1u) && !(lv[e] + dv[e] < lo_k)) cut_bad = true;
      }
      const bool open = __any_sync(0xffffffffu, order_bad || cut_bad) || !fin;
      if (lane == 0) S.open[t] = open ? 1 : 0;
      if (open) {
        // contenders: its picks and every expert whose upper bound reaches the
        // lowest pick's lower bound (all of them when a bound is not finite)
        __syncwarp();
        for (int m = 0; m < P; ++m) {
          const int e = lane + 32 * m;
          bool c = false;
          if (e < E) {
            bool picked = false;
            for (int j = 0; j < k; ++j) picked = picked || S.sel[t * k + j] == e;
            c = !fin || picked || !(lv[e] + dv[e] < lo_min);
          }
          const unsigned bal = __ballot_sync(0xffffffffu, c);
          int base = 0;
          if (lane == 0 && bal) base = atomicAdd(&S.n_list, __popc(bal));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (c) {
            const int p = base + __popc(bal & ((1u << lane) - 1u));
            S.list[p] = t * E + e;
            S.lpos[t * E + e] = p;
          }
        }
      }
    }
    __syncthreads();
    // gates of the certified tokens; widths of their assignments
    if (warp < T && !S.open[warp]) front_gates(A, S.val + warp * E, S.sel + warp * k, warp, lane);
    if (gate) {
      for (int a = threadIdx.x; a < na; a += blockDim.x) {
        const int t = a / k;
        if (S.open[t]) continue;
        const int e = S.sel[a];
        const int b = front_width32(A, S, TE, nitems, t, e);
        if (b) {
          front_set_width(A, S, a, b);
        } else {  // its three scores in fp64
          const int p = atomicAdd(&S.n_list, 3);
          for (int c = 0; c < 3; ++c) {
            const int it = TE + 3 * (t * E + e) + c;
            S.list[p + c] = it;
            S.lpos[it] = p + c;
          }
        }
      }
    }
    __syncthreads();
    front_publish_list(S, S.n_list, na, gate);
  }
  cluster_sync_publish();  // the list is in every CTA
  const int nl = S.n_list;
  if (nl > 0) {  // cluster-uniform
    // ---- 3. fp64 for the listed dot products
    front_dots64(A, TE, S.list, nl, rank * dk, dk, cluster_map_shared(S.p64, 0) + 8u * static_cast<uint32_t>(rank * nl));
    cluster_sync_publish();
    if (rank == 0) {
      auto v64 = [&](int it) {
        double s = S.p64[S.lpos[it]];
        for (int r = 1; r < kFC; ++r) s += S.p64[r * nl + S.lpos[it]];
        return s;
      };
      // open tokens: select on the fp64 logits of their contenders
      for (int i = threadIdx.x; i < TE; i += blockDim.x) {
        const int t = i / E, e = i - t * E;
        if (!S.open[t]) continue;
        S.v64[i] = S.lpos[i] >= 0 ? v64(i) + (A.bias ? static_cast<double>(A.bias[e]) : 0.0) : -INFINITY;
      }
      __syncthreads();
      if (warp < T && S.open[warp]) {
        warp_topk_rank(S.v64 + warp * E, E, k, lane, S.sel + warp * k);
        front_gates(A, S.v64 + warp * E, S.sel + warp * k, warp, lane);
      }
      __syncthreads();
      if (gate) {
        // widths still open: of certified tokens (listed, fp64 from the
        // cluster), and of open tokens (fp32 if certified, else fp64 here)
        if (threadIdx.x == 0) S.n_open = 0;
        __syncthreads();
        for (int a = threadIdx.x; a < na; a += blockDim.x) {
          const int t = a / k, e = S.sel[a];
          const int it0 = TE + 3 * (t * E + e);
          if (!S.open[t]) {
            if (S.lpos[it0] < 0) continue;  // decided on the fp32 scores
            double v[3];
#pragma unroll
            for (int c = 0; c < 3; ++c)
              v[c] = v64(it0 + c) + (A.bbit ? static_cast<double>(A.bbit[static_cast<size_t>(e) * 3 + c]) : 0.0);
            int best = 0;
            if (v[1] > v[best]) best = 1;
            if (v[2] > v[best]) best = 2;
            front_set_width(A, S, a, 2 + best);
          } else {
            const int b = front_width32(A, S, TE, nitems, t, e);
            if (b) front_set_width(A, S, a, b);
            else S.key[atomicAdd(&S.n_open, 1)] = a;  // key[] is free until the permutation
          }
        }
        __syncthreads();
        // an open assignment of an open token: its three scores in fp64, a
        // warp per score (lanes over d), in this CTA alone
        const int no = S.n_open;
        for (int pc = warp; pc < 3 * no; pc += kFWarps) {
          const int a = S.key[pc / 3], c = pc % 3, t = a / k, e = S.sel[a];
          const double v = dot_bf16_f32_fp64(A.x + static_cast<size_t>(t) * A.d,
                                             A.wbit + (static_cast<size_t>(e) * 3 + c) * A.d, A.d, lane);
          if (lane == 0) S.g64[pc] = v + (A.bbit ? static_cast<double>(A.bbit[static_cast<size_t>(e) * 3 + c]) : 0.0);
        }
        __syncthreads();
        for (int j = threadIdx.x; j < no; j += blockDim.x) {
          const double* v = S.g64 + 3 * j;
          int best = 0;
          if (v[1] > v[best]) best = 1;
          if (v[2] > v[best]) best = 2;
          front_set_width(A, S, S.key[j], 2 + best);
        }
      }
    }
  }
  if (!A.counts) return;
  // with nothing open every CTA holds the final picks (and widths): each
  // computes the permutation and gathers its share of the rows; otherwise
  // CTA 0, which decided the open items, does it all
  const int nct = nl == 0 ? kFC : 1;
  if (rank >= nct) return;
  __syncthreads();  // picks and widths complete
  // ---- 4. permutation of the na assignments
  const bool nested = gate || A.bits_in;
  const int nbins = nested ? 3 * E : E;
  for (int a = threadIdx.x; a < na; a += blockDim.x) {
    int key = S.sel[a];
    if (nested) {
      int b = gate ? S.bits[a] : A.bits_in[a];
      if (b < 2 || b > 4) {
        if (rank == 0) flag_status(A.status, MOE_DEV_BAD_INDEX);
        b = b < 2 ? 2 : 4;
      }
      key = 3 * key + (b - 2);
    }
    S.key[a] = key;
  }
  __syncthreads();
  for (int a = threadIdx.x; a < na; a += blockDim.x) {
    const int key = S.key[a];
    int pos = 0;
    for (int o = 0; o < na; ++o) {
      const int ko = S.key[o];
      pos += (ko < key || (ko == key && o < a)) ? 1 : 0;
    }
    if (rank == 0) {
      A.perm[pos] = a;
      A.inv_perm[a] = pos;
    }
    S.perm[pos] = a;
  }
  for (int b = threadIdx.x; rank == 0 && b <= nbins; b += blockDim.x) {
    int below = 0, at = 0;
    for (int o = 0; o < na; ++o) {
      below += S.key[o] < b ? 1 : 0;
      at += S.key[o] == b ? 1 : 0;
    }
    A.offsets[b] = below;
    if (b < nbins) A.counts[b] = at;
  }
  if (!A.x_perm) return;
  __syncthreads();  // S.perm complete
  // gather: (row, 8-element piece) items split over the nct CTAs and their
  // threads, bf16 -> fp16
  const int vec = A.d / 8;
  bool bad = false;
  for (int v = rank * blockDim.x + threadIdx.x; v < na * vec; v += nct * blockDim.x) {
    const int p = v / vec, c = v - p * vec;
    const uint4 in = reinterpret_cast<const uint4*>(A.x + static_cast<size_t>(S.perm[p] / k) * A.d)[c];
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&in);
    uint4 o;
    __half2* h2 = reinterpret_cast<__half2*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(b2[j]);
      bad |= fabsf(f.x) > 65504.0f || fabsf(f.y) > 65504.0f;
      h2[j] = __floats2half2_rn(f.x, f.y);
    }
    reinterpret_cast<uint4*>(A.x_perm + static_cast<size_t>(p) * A.d)[c] = o;
  }
  if (bad) flag_status(A.status, MOE_DEV_RANGE);
}

// Bound factor: g(m), m = products per lane of a slice (d / (4 kFC)) + 2
// tree levels + kFC slice additions + 1 bias addition.
float front_gamma(int d) {
  const double u = std::ldexp(1.0, -24);
  const double m = static_cast<double>(d) / (4 * kFC) + 2.0 + kFC + 1.0;
  return static_cast<float>(m * u / (1.0 - m * u));
}

}  // namespace

// The smallest batches (T <= 8, T*E <= 512, d % 256 == 0: one slice of d
// per CTA is a multiple of 32 elements, 4 lanes x 8-element pieces).
bool route_tiny_ok(int T, int d, int E) {
  return g_route_fused == 1 && T >= 1 && T <= kFMaxT && T * E <= kFMaxTE && d % (32 * kFC) == 0;
}

// With a bit gate, T*E <= 128 (its 3 T*E scores join the T*E logits).
bool route_permute_fusable(int T, int d, int E, int k, bool gate) {
  return route_tiny_ok(T, d, E) && T * k <= kFMaxTK && (!gate || T * E <= kFMaxGateTE);
}

moe_status_t launch_front_tiny(const void* x, const float* w_router, const float* bias, const int32_t* forced,
                               const uint8_t* bits_in, const float* w_bit, const float* bias_bit, int T, int d,
                               int E, int k, int32_t* idx, float* w, uint8_t* bits_out, int32_t* counts,
                               int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* x_perm, int32_t* status,
                               cudaStream_t s) {
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "front cudaGetDevice");
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    e = cudaFuncSetAttribute(k_front<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sizeof(FrontSmem)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_front<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sizeof(FrontSmem)));
    if (e != cudaSuccess) return cuda_check(e, "front smem attribute");
    attr_set.fetch_or(bit);
  }
  FrontArgs A{static_cast<const __nv_bfloat16*>(x), w_router, bias, forced, w_bit, bias_bit, bits_in, T, d, E, k,
              front_gamma(d), idx, w, bits_out, counts, offsets, perm, inv_perm, static_cast<__half*>(x_perm),
              status};
  const int n_rows = w_bit ? 4 * E : E, tch = front_token_chunks(T, n_rows);
  const bool rows = (T + tch - 1) / tch >= kRowsMinTokens;
  return cuda_check(launch_cluster_pdl(rows ? k_front<true> : k_front<false>, kFC, dim3(kFThreads), sizeof(FrontSmem),
                                       s, A),
                    "front cluster launch");
}

}  // namespace moeq
