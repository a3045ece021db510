// Softmax top-k router.
//
// The expert choice must equal the top k of the exact logits
//   l[t][e] = x[t] . W_r[e] + bias[e]
// (ties -> lower index), i.e. what a plain fp64 evaluation gives.  Doing all
// T*E*d products in fp64 runs at the fp64 rate; instead:
//
//   k_route_logits  fp32 logits with blocked accumulation: a thread sums 32
//                   products with FMA into a fresh chunk sum, then adds the
//                   chunk sum to its running total; slices of d (splits)
//                   are summed later in split order.  The same CTAs also
//                   produce the sums of squares of x rows and W_r rows.
//   k_route_select  warp per token: the split sums and the bias give the
//                   fp32 logit L[e]; with the error bound
//                     |L[e] - l[e]| <= D[e]
//                       = 2 (g(32 + d/32) |x| |W_e| (1 + 2^-8) + u (|L| + |b|))
//                   (u = 2^-24, g(m) = m u / (1 - m u); Cauchy-Schwarz for
//                   sum |x_i W_ei|; the factor 2 is margin), the top k of L,
//                   in order, is that of l whenever consecutive picks are
//                   separated by more than their bounds and the last pick
//                   beats every other expert:
//                     L[k-th pick] - D  >  max over the rest (L + D).
//                   Tokens where that fails (near ties, non-finite values)
//                   are recomputed by the whole CTA in fp64 (each product of
//                   a bf16 and an fp32 is exact in fp64) and selected on the
//                   fp64 logits.  Gates are the softmax over the k picked
//                   logits (fp32 for certified tokens, fp64 for the others).
//
// For the smallest batches (T <= 8 and T*E <= 512) both steps run in one
// launch of a thread-block cluster (k_front, front.cu), each CTA one slice
// of d; the same fp32-plus-bound scheme with a tighter bound (sums of
// magnitudes, not norms), and fp64 only for the contenders of tokens it
// leaves open.
//
// Error bound of the fp32 sum: an FMA chain over m products errs by at most
// g(m) times the sum of their magnitudes; a chunk (32 products) and then the
// d/32 chunk sums in any order give g(32) + g(d/32)(1 + g(32)) <= g(32 + d/32).
// The squared norms are fp32 sums too (relative error below 2^-8 for
// d < 2^15) and the bias addition rounds once more (the u term).
#include <atomic>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kDC = 32;  // d chunk: fp32 accumulation block and shared-memory stage
constexpr int kMT = 4;   // tokens per thread (one 16-byte shared-memory load of x per k)
static_assert(kMT == 4, "x is read as float4");
constexpr int kLT = 128; // threads of a logits CTA (4 warps)

// EC experts per CTA tile (64, or 16 for E <= 16): ME per thread, TX threads
// along experts, TYW thread rows per warp; a CTA covers TT tokens.
template <int EC>
struct Tile {
  static constexpr int ME = EC == 64 ? 8 : 4;
  static constexpr int TX = EC / ME;
  static constexpr int TYW = 32 / TX;
  static constexpr int TT = (kLT / 32) * TYW * kMT;
  static constexpr int XP = TT + 4;    // x stage row pitch (floats; rows 16-byte aligned)
  static constexpr int XS = kDC * XP;  // floats per x stage ([k][token]: a thread's kMT tokens in one 16-byte load)
  static constexpr int WS = kDC * EC;  // floats per W stage ([k][expert])
  static constexpr size_t SMEM = 2 * (XS + WS) * sizeof(float);
  static constexpr int XL = TT * 4 / kLT;   // 16-byte x loads per thread per chunk
  static constexpr int WL = EC * 8 / kLT;   // 16-byte W loads per thread per chunk
};

// Workspace: partial[S][T][E] fp32, xsq[S][T], wsq[S][E].
struct RouteWs {
  float* partial;
  float* xsq;
  float* wsq;
};

__host__ __device__ inline RouteWs route_ws(void* base, int S, int T, int E) {
  float* p = static_cast<float*>(base);
  return {p, p + static_cast<size_t>(S) * T * E, p + static_cast<size_t>(S) * T * E + static_cast<size_t>(S) * T};
}

// The kLT threads of a logits tile synchronise on named barrier 1 (so that
// a kernel with more threads can run the tile on its first kLT threads).
__device__ __forceinline__ void tile_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kLT) : "memory"); }

// Partial logits of token tile bt, expert tile be, slice `split` of d (dk
// wide) into the workspace, by threads 0..kLT-1.
template <int EC>
__device__ __forceinline__ void logits_tile(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr,
                                            int T, int d, int E, int dk, RouteWs ws, int bt, int be, int split,
                                            float* sm) {
  using G = Tile<EC>;
  float* xs = sm;               // [2][kDC][XP]
  float* wsm = sm + 2 * G::XS;  // [2][kDC][EC]
  const int tid = threadIdx.x, lane = tid & 31;
  const int tx = lane % G::TX;
  const int ty = (tid >> 5) * G::TYW + lane / G::TX;
  const int t0 = bt * G::TT, e0 = be * EC;
  const int kbeg = split * dk, nch = dk / kDC;
  const bool do_x = be == 0, do_w = bt == 0;

  // loaders: x load q covers token row (tid + kLT q) / 4, columns ((tid + kLT q) % 4) * 8 .. +8;
  // W load q covers expert (tid + kLT q) % EC, columns ((tid + kLT q) / EC) * 4 .. +4
  uint4 xr[G::XL];
  float4 wv4[G::WL];
  float xsq[G::XL], wsq[G::WL];
#pragma unroll
  for (int q = 0; q < G::XL; ++q) xsq[q] = 0.f;
#pragma unroll
  for (int q = 0; q < G::WL; ++q) wsq[q] = 0.f;

  auto fetch = [&](int k0) {
#pragma unroll
    for (int q = 0; q < G::XL; ++q) {
      const int i = tid + kLT * q, t = t0 + (i >> 2);
      xr[q] = t < T ? *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d + k0 + (i & 3) * 8)
                    : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < G::WL; ++q) {
      const int i = tid + kLT * q, e = e0 + i % EC;
      wv4[q] = e < E ? *reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * d + k0 + (i / EC) * 4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto stash = [&](int b) {
    float* xb = xs + b * G::XS;
#pragma unroll
    for (int q = 0; q < G::XL; ++q) {
      const int i = tid + kLT * q, r = i >> 2, c = (i & 3) * 8;
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xr[q]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(b2[j]);
        xb[(c + 2 * j) * G::XP + r] = f.x;
        xb[(c + 2 * j + 1) * G::XP + r] = f.y;
        if (do_x) xsq[q] = fmaf(f.x, f.x, fmaf(f.y, f.y, xsq[q]));
      }
    }
    float* wb = wsm + b * G::WS;
#pragma unroll
    for (int q = 0; q < G::WL; ++q) {
      const int i = tid + kLT * q, e = i % EC, c = (i / EC) * 4;
      const float v[4] = {wv4[q].x, wv4[q].y, wv4[q].z, wv4[q].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wb[(c + j) * EC + e] = v[j];
        if (do_w) wsq[q] = fmaf(v[j], v[j], wsq[q]);
      }
    }
  };

  float acc[kMT][G::ME];
#pragma unroll
  for (int i = 0; i < kMT; ++i)
#pragma unroll
    for (int j = 0; j < G::ME; ++j) acc[i][j] = 0.f;

  fetch(kbeg);
  stash(0);
  tile_sync();
  for (int c = 0; c < nch; ++c) {
    const int b = c & 1;
    if (c + 1 < nch) fetch(kbeg + (c + 1) * kDC);
    const float* xb = xs + b * G::XS + ty * kMT;
    const float* wb = wsm + b * G::WS + tx * 4;
    // chunk sums, two experts per packed fp32 FMA (each lane of the pair is
    // an ordinary round-to-nearest FMA, so the error bound is unchanged)
    float2 cs[kMT][G::ME / 2];
#pragma unroll
    for (int i = 0; i < kMT; ++i)
#pragma unroll
      for (int j = 0; j < G::ME / 2; ++j) cs[i][j] = make_float2(0.f, 0.f);
#pragma unroll 8
    for (int kk = 0; kk < kDC; ++kk) {
      float2 wv[G::ME / 2];
#pragma unroll
      for (int j = 0; j < G::ME; j += 4) {  // experts tx*4 + (0..3) [+ EC/2]
        const float4 w4 = *reinterpret_cast<const float4*>(wb + kk * EC + (j / 4) * (EC / 2));
        wv[j / 2] = make_float2(w4.x, w4.y);
        wv[j / 2 + 1] = make_float2(w4.z, w4.w);
      }
      const float4 x4 = *reinterpret_cast<const float4*>(xb + kk * G::XP);  // tokens ty kMT .. + 3
      const float xa[kMT] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
      for (int i = 0; i < kMT; ++i) {
        const float2 x2 = make_float2(xa[i], xa[i]);
#pragma unroll
        for (int j = 0; j < G::ME / 2; ++j) cs[i][j] = __ffma2_rn(x2, wv[j], cs[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < kMT; ++i)
#pragma unroll
      for (int j = 0; j < G::ME / 2; ++j) {
        acc[i][2 * j] += cs[i][j].x;
        acc[i][2 * j + 1] += cs[i][j].y;
      }
    if (c + 1 < nch) stash(b ^ 1);
    tile_sync();
  }

  float* out = ws.partial + static_cast<size_t>(split) * T * E;
#pragma unroll
  for (int i = 0; i < kMT; ++i) {
    const int t = t0 + ty * kMT + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < G::ME; ++j) {
      const int e = e0 + tx * 4 + (j & 3) + (j / 4) * (EC / 2);
      if (e < E) out[static_cast<size_t>(t) * E + e] = acc[i][j];
    }
  }
  // squared norms: the 4 x-loader lanes of a row are adjacent; a W row's
  // loaders are the threads i with i % EC equal, reduced through shared memory
  if (do_x) {
#pragma unroll
    for (int q = 0; q < G::XL; ++q) {
      float v = xsq[q];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      const int i = tid + kLT * q, t = t0 + (i >> 2);
      if ((i & 3) == 0 && t < T) ws.xsq[static_cast<size_t>(split) * T + t] = v;
    }
  }
  if (do_w) {
    float* red = sm;  // reuse the stages (the loop ended with a barrier)
#pragma unroll
    for (int q = 0; q < G::WL; ++q) red[tid + kLT * q] = wsq[q];
    tile_sync();
    if (tid < EC) {
      float v = 0.f;
      for (int i = tid; i < EC * 8; i += EC) v += red[i];
      const int e = e0 + tid;
      if (e < E) ws.wsq[static_cast<size_t>(split) * E + e] = v;
    }
  }
}

template <int EC>
__global__ void __launch_bounds__(kLT, 4) k_route_logits(const __nv_bfloat16* __restrict__ x,
                                                       const float* __restrict__ wr, int T, int d, int E,
                                                       int dk, RouteWs ws) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) float sm[];
  logits_tile<EC>(x, wr, T, d, E, dk, ws, blockIdx.x, blockIdx.y, blockIdx.z, sm);
}

constexpr int kMaxPer = 8;  // E <= 256: at most 8 experts per lane (e = lane + 32 m)

// True on every lane of a warp when any lane lists a contender.
__device__ __forceinline__ bool contender_any(uint32_t c) { return __any_sync(0xffffffffu, c != 0); }

// Top k of the lane-distributed values v[m] (expert lane + 32 m; experts
// whose bit m of `allowed` is clear take no part), ties to the lower index;
// lane j < k receives pick j (0 where fewer than k values are comparable).
template <typename V, int P>
__device__ __forceinline__ int warp_topk(const V (&v)[P], uint32_t allowed, int E, int k, int lane) {
  uint32_t taken = 0;
  int mine = 0;
  for (int j = 0; j < k; ++j) {
    V best = -INFINITY;
    int best_e = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < P; ++m) {
      const int e = lane + 32 * m;
      if (e < E && (allowed & (1u << m)) && !(taken & (1u << m)) &&
          (v[m] > best || (v[m] == best && e < best_e))) {
        best = v[m];
        best_e = e;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const V ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oe = __shfl_xor_sync(0xffffffffu, best_e, o);
      if (ov > best || (ov == best && oe < best_e)) {
        best = ov;
        best_e = oe;
      }
    }
    if (best_e >= E) best_e = 0;  // only when fewer than k values are comparable (NaN)
    if (lane == j) mine = best_e;
    if ((best_e & 31) == lane) taken |= 1u << (best_e >> 5);
  }
  return mine;
}

// Softmax over the k picks (lane j < k holds pick j, in any order) of the
// lane-distributed values, in fp64; maximum and sum are fixed-order shuffle
// trees.
template <typename V, int P>
__device__ __forceinline__ void write_gates(const V (&v)[P], int mine, int k, int t, int lane, int32_t* out_idx,
                                            float* out_w) {
  double lv = 0.0;
#pragma unroll
  for (int m = 0; m < P; ++m) {  // the value of expert `mine`, from the lane that holds it
    const V o = __shfl_sync(0xffffffffu, v[m], mine & 31);
    if ((mine >> 5) == m) lv = static_cast<double>(o);
  }
  double mx = lane < k ? lv : -INFINITY;
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const double ex = lane < k ? exp(lv - mx) : 0.0;
  double sum = ex;
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    out_idx[static_cast<size_t>(t) * k + lane] = mine;
    out_w[static_cast<size_t>(t) * k + lane] = static_cast<float>(ex / sum);
  }
}

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

// Warp per token, P experts per lane (E <= 32 P).  The k largest fp32
// logits are picked one at a time with warp reductions (redux.sync) over
// order keys: the largest key, then the lowest expert holding it.  The
// certificate and the gates are lane-parallel: lane j < k holds pick j.  A
// token the fp32 bounds do not settle lists its contenders -- every expert
// whose upper bound reaches the lowest lower bound among the picks (all
// others are certainly out) -- and the CTA's warps recompute those logits
// in fp64; the token's warp then selects among them on the fp64 values.
// Tokens block * kSelWarps .. + kSelWarps - 1, by all kSelThreads threads.
template <int P>
__device__ __forceinline__ void select_block(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr, RouteWs ws, int splits,
    const float* __restrict__ bias, const int32_t* __restrict__ forced, int T, int d, int E, int k,
    float gamma, int32_t* __restrict__ out_idx, float* __restrict__ out_w, int block) {
  __shared__ int n_cand[kSelWarps];
  __shared__ uint8_t cand[kSelWarps][32 * P];
  __shared__ double l64[kSelWarps][32 * P];
  __shared__ float l32[kSelWarps][32 * P], d32[kSelWarps][32 * P];  // fp32 logits and bounds of each warp's token
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = block * kSelWarps + warp;
  if (lane == 0) n_cand[warp] = 0;
  uint32_t contender = 0;  // lane's experts listed for fp64
  if (t < T) {
    float L[P], D[P];
    // split sums in split order, loads of a batch of 8 splits issued together
    float xq = 0.f;
    for (int s0 = 0; s0 < splits; s0 += 8) {
      float q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = s0 + u < splits ? ws.xsq[static_cast<size_t>(s0 + u) * T + t] : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) xq += q[u];
    }
    const float xn = sqrtf(xq);
    float* ls = l32[warp];
    float* ds = d32[warp];
#pragma unroll
    for (int m = 0; m < P; ++m) {
      const int e = lane + 32 * m;
      L[m] = -INFINITY;
      D[m] = 0.f;
      if (e < E) {
        float v = 0.f, wq = 0.f;
        for (int s0 = 0; s0 < splits; s0 += 8) {
          float pv[8], qv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const bool in = s0 + u < splits;
            pv[u] = in ? ws.partial[(static_cast<size_t>(s0 + u) * T + t) * E + e] : 0.f;
            qv[u] = in ? ws.wsq[static_cast<size_t>(s0 + u) * E + e] : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            v += pv[u];
            wq += qv[u];
          }
        }
        const float b = bias ? bias[e] : 0.f;
        v += b;
        L[m] = v;
        D[m] = 2.0f * (gamma * xn * sqrtf(wq) * (1.0f + 0.00390625f) +
                       5.9604645e-8f * (fabsf(v) + fabsf(b))) + 1e-30f;
        ls[e] = L[m];
        ds[e] = D[m];
      }
    }
    __syncwarp();
    int mine = 0;        // lane j < k: pick j
    uint32_t taken = 0;  // the lane's picked experts (bit m: expert lane + 32 m)
    bool sure = true;
    if (forced) {
      if (lane < k) {
        const int e = forced[static_cast<size_t>(t) * k + lane];
        mine = e < 0 ? 0 : (e >= E ? E - 1 : e);
      }
    } else {
      uint32_t key[P];
#pragma unroll
      for (int m = 0; m < P; ++m) key[m] = lane + 32 * m < E ? order_key(L[m]) : 0u;
      for (int j = 0; j < k; ++j) {
        uint32_t bk = 0;
        int be = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < P; ++m)
          if (!((taken >> m) & 1u) && key[m] > bk) {  // the lane's lowest expert on equal keys
            bk = key[m];
            be = lane + 32 * m;
          }
        const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
        int e = __reduce_min_sync(0xffffffffu, bk == top ? be : 0x7fffffff);
        if (e >= E) e = 0;  // only when fewer than k values are comparable (NaN)
        if (top != 0 && (e & 31) == lane) taken |= 1u << (e >> 5);
        if (lane == j) mine = e;
      }
      // Certified when the order of the picks and the cut after the k-th are
      // both wider than the bounds: pick j beats pick j + 1, and the last
      // pick beats every other expert (comparisons with NaN are false, so
      // non-finite values fall through to fp64).
      float lo = INFINITY, up = -INFINITY;
      if (lane < k) {
        lo = ls[mine] - ds[mine];
        up = ls[mine] + ds[mine];
      }
      const float lo_prev = __shfl_up_sync(0xffffffffu, lo, 1);
      const bool ok = lane >= k || lane == 0 || lo_prev > up;
      float hi = -INFINITY;
#pragma unroll
      for (int m = 0; m < P; ++m)
        if (lane + 32 * m < E && !(taken & (1u << m))) hi = fmaxf(hi, L[m] + D[m]);
#pragma unroll
      for (int o = 16; o; o >>= 1) hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      float lo_min = lo;
#pragma unroll
      for (int o = 16; o; o >>= 1) lo_min = fminf(lo_min, __shfl_xor_sync(0xffffffffu, lo_min, o));
      const float lo_last = __shfl_sync(0xffffffffu, lo, k - 1);
      sure = __all_sync(0xffffffffu, ok) && (k < E ? lo_last > hi : lo_last == lo_last);
      if (!sure) {
        // contenders: picks, and every other expert whose upper bound reaches
        // the lowest pick's lower bound (all of them when a value is not finite)
        const bool finite = lo_min == lo_min && fabsf(lo_min) <= 3.0e38f;
#pragma unroll
        for (int m = 0; m < P; ++m) {
          const int e = lane + 32 * m;
          if (e < E && (!finite || (taken & (1u << m)) || !(L[m] + D[m] < lo_min))) contender |= 1u << m;
        }
        int base = 0;
#pragma unroll
        for (int m = 0; m < P; ++m) {
          const unsigned bal = __ballot_sync(0xffffffffu, (contender >> m) & 1u);
          if ((contender >> m) & 1u) cand[warp][base + __popc(bal & ((1u << lane) - 1u))] = lane + 32 * m;
          base += __popc(bal);
        }
        if (lane == 0) n_cand[warp] = base;
      }
    }
    if (sure) {  // gates: the softmax over the picks' fp32 logits, in fp32
      const float lv = lane < k ? ls[mine] : -INFINITY;
      float mx = lv;
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float ex = lane < k ? expf(lv - mx) : 0.0f;
      float sum = ex;
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane < k) {
        out_idx[static_cast<size_t>(t) * k + lane] = mine;
        out_w[static_cast<size_t>(t) * k + lane] = ex / sum;
      }
    }
  }
  __syncthreads();
  // fp64 logits of all listed (token, expert) pairs of this CTA, spread over its warps
  int total = 0;
  for (int w = 0; w < kSelWarps; ++w) total += n_cand[w];
  if (total == 0) return;  // CTA-uniform
  for (int item = warp; item < total; item += kSelWarps) {
    int w = 0, r = item;
    while (r >= n_cand[w]) r -= n_cand[w++];
    const int tu = block * kSelWarps + w, e = cand[w][r];
    const double v = dot_bf16_f32_fp64(x + static_cast<size_t>(tu) * d, wr + static_cast<size_t>(e) * d, d, lane);
    if (lane == 0) l64[w][e] = v + (bias ? static_cast<double>(bias[e]) : 0.0);
  }
  __syncthreads();
  if (contender_any(contender)) {
    double v[P];
#pragma unroll
    for (int m = 0; m < P; ++m) v[m] = ((contender >> m) & 1u) ? l64[warp][lane + 32 * m] : -INFINITY;
    write_gates(v, warp_topk(v, contender, E, k, lane), k, t, lane, out_idx, out_w);
  }
}

// Scratch bytes of a route with S slices of d.
size_t route_ws_for(size_t S, int T, int E) {
  return std::max<size_t>(256, S * (static_cast<size_t>(T) * E + T + E) * sizeof(float));
}

// Slices of d: enough CTAs for about four per SM, halved while the scratch
// they need exceeds `cap` bytes (one slice always remains; the error bound
// of the logits holds for any slicing, since slices are sums of 32-product
// chunk sums).

template <int P>
__global__ void __launch_bounds__(kSelThreads, 4) k_route_select(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr, RouteWs ws, int splits,
    const float* __restrict__ bias, const int32_t* __restrict__ forced, int T, int d, int E, int k,
    float gamma, int32_t* __restrict__ out_idx, float* __restrict__ out_w) {
  pdl_wait();
  pdl_trigger();
  select_block<P>(x, wr, ws, splits, bias, forced, T, d, E, k, gamma, out_idx, out_w, blockIdx.x);
}

int route_splits(int T, int d, int E, size_t cap = static_cast<size_t>(-1)) {
  const int ec = E <= 16 ? 16 : 64;
  const int tt = ec == 64 ? Tile<64>::TT : Tile<16>::TT;
  const int tiles = ceil_div(T, tt) * ceil_div(E, ec);
  const int chunks = d / kDC;
  const int target = ceil_div(4 * 148, tiles);  // about four CTAs per SM
  int s = 1;
  while (s * 2 <= target && chunks % (s * 2) == 0 && s * 2 <= 16) s *= 2;
  while (s > 1 && route_ws_for(s, T, E) > cap) s /= 2;
  return s;
}

float route_gamma(int d) {
  const double u = std::ldexp(1.0, -24);
  const double m = kDC + d / kDC;
  return static_cast<float>(m * u / (1.0 - m * u));
}

template <int EC>
moe_status_t launch_logits(const __nv_bfloat16* x, const float* wr, int T, int d, int E, int k_route, int splits,
                           RouteWs ws, cudaStream_t s) {
  using G = Tile<EC>;
  // the shared-memory opt-in is a per-device attribute: set once per device
  // (the first call on a device precedes any stream capture)
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "moe_route_topk cudaGetDevice");
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    e = cudaFuncSetAttribute(k_route_logits<EC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(G::SMEM));
    if (e != cudaSuccess) return cuda_check(e, "moe_route_topk smem attribute");
    attr_set.fetch_or(bit);
  }
  dim3 grid(ceil_div(T, G::TT), ceil_div(E, EC), splits);
  return cuda_check(launch_pdl(pdl_for(static_cast<long>(T) * k_route), k_route_logits<EC>, grid, dim3(kLT), G::SMEM, s, x, wr, T, d, E, d / splits, ws),
                    "moe_route_topk logits launch");
}

}  // namespace

int g_route_fused = 1;

size_t route_workspace_bytes(int T, int d, int E) {
  if (T <= 0 || d <= 0 || E <= 0) return 256;
  return route_ws_for(static_cast<size_t>(route_splits(T, d, E)), T, E);
}

size_t route_min_workspace_bytes(int T, int d, int E) {
  if (T <= 0 || d <= 0 || E <= 0) return 256;
  return route_ws_for(1, T, E);
}

moe_status_t launch_route(const void* x, const float* w_router, const float* bias,
                          const int32_t* forced, int T, int d, int E, int k, int32_t* idx,
                          float* w, void* workspace, size_t workspace_bytes, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int splits = route_splits(T, d, E, workspace_bytes);
  const RouteWs ws = route_ws(workspace, splits, T, E);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  // the smallest batches: one cluster launch (no workspace)
  if (route_tiny_ok(T, d, E))
    return launch_front_tiny(x, w_router, bias, forced, nullptr, nullptr, nullptr, T, d, E, k, idx, w, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, s);
  moe_status_t st = E <= 16 ? launch_logits<16>(xb, w_router, T, d, E, k, splits, ws, s)
                            : launch_logits<64>(xb, w_router, T, d, E, k, splits, ws, s);
  if (st != MOE_OK) return st;
  auto sel = E <= 32 ? k_route_select<1> : E <= 64 ? k_route_select<2> : E <= 128 ? k_route_select<4>
                                                                           : k_route_select<kMaxPer>;
  return cuda_check(launch_pdl(pdl_for(static_cast<long>(T) * k), sel, dim3(ceil_div(T, kSelWarps)), dim3(kSelThreads),
                               0, s, xb, w_router, ws, splits, bias, forced, T, d, E, k, route_gamma(d), idx, w),
                    "moe_route_topk select launch");
}

}  // namespace moeq

// ---------------------------------------------------------------------------
// Allocation-free router entry point.
//
// Some callers cannot allocate device memory at the point where they route:
// plugins and runtimes that hand us only a stream and have no allocator of
// their own to lend, and latency-critical serving paths that must not risk
// an allocation failure or an implicit synchronisation.  moe_route_topk_noalloc keeps the router's scratch (the
// per-slice fp32 partial logits and squared norms) in a fixed device array
// owned by this library instead of a caller-provided workspace; the number
// of d slices is capped so that the scratch fits the array.
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

extern "C" void moe_debug_route_fused(int mode) { moeq::g_route_fused = mode == 0 ? 0 : 1; }

extern "C" moe_status_t moe_route_topk_noalloc(const void* x, const float* w_router, const float* bias,
                                                const int32_t* forced_idx, int T, int d, int E, int k,
                                                int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  using namespace moeq;
  moe_status_t st = route_check_args(x, w_router, T, d, E, k, topk_idx, topk_w, "moe_route_topk_noalloc");
  if (st != MOE_OK) return st;
  const size_t need = route_min_workspace_bytes(T, d, E);
  if (T > 0 && need > kRouteScratchBytes) {
    set_error("moe_route_topk_noalloc: T=%d d=%d E=%d needs %zu bytes of scratch, above the fixed %zu",
              T, d, E, need, kRouteScratchBytes);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (T == 0) return MOE_OK;
  void* scratch = nullptr;
  st = route_scratch(&scratch);
  if (st != MOE_OK) return st;
  return launch_route(x, w_router, bias, forced_idx, T, d, E, k, topk_idx, topk_w, scratch,
                      kRouteScratchBytes, static_cast<cudaStream_t>(stream));
}
