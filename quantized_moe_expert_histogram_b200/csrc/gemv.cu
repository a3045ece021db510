// Decode-regime grouped expert FFN: a warp per group of weight rows.
//
// Used for one token (bins of one row; any T when the regime is forced):
// the layer is then bound by the bytes of the routed experts' codes, so
// each weight row is streamed once with 16-byte loads and dotted against
// the bin's (at most MAXR) activation rows, which stay in L1.  Dequantisation happens in
// registers: a 4-bit code q becomes the fp32 value 1 + q/16 by OR-ing it
// into the mantissa of 1.0f, so the row dot product needs no int->float
// conversion; per 8 elements the exact  sum (q - z) * s * x  is recovered as
//   s * (16 * (sum (1 + q/16) x - sum x) - z * sum x).
// Accumulation is fp32.  blockIdx.y enumerates the non-empty (and, in slot
// mode, resident) bins; blockIdx.x a block of 8 warps x RW output rows.
//
// Both passes are programmatic dependent launches (launch_pdl).  The down
// pass starts while the gate/up pass runs, locates its bin and issues the
// loads of its weight codes (which do not depend on h), and only then waits
// for the gate/up grid before reading h.  The gate/up pass triggers after
// its own wait, so everything the down pass reads before its wait
// (offsets, slot table, weights) is complete by then.
//
//   gate/up pass:  h[p][f]      = silu(Wg[f] . x_p) * (Wu[f] . x_p)   (fp16)
//   down pass:     y_perm[p][n] = Wd[n] . h_p                          (fp16)
#include <algorithm>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kChunkSteps = 2;  // 32-element steps whose loads are issued together

struct GemvParams {
  const __half* act;        // x_perm [rows][K] or h [rows][K]
  const int32_t* offsets;   // [nbins+1]
  const uint8_t* blobs;
  const int32_t* slot_of;
  size_t blob_bytes;
  size_t code_off[2];       // INT4 codes (or Q2) of the 1-2 matrices
  size_t d3_off[2];
  size_t d4_off[2];
  size_t sz_off[2];
  int K, N, nbins, planes_mult;  // planes_mult: 1 for INT4 bins, 3 for (e,b) bins
  int rows;                 // activation rows: bin ranges are clamped into [0, rows]
  int group;
  __half* h_out;            // gate/up pass output [rows][N]
  __half* y_out;            // down pass output [rows][N]
  int32_t* status;
};

// Nibble i of `w` as the float 1 + q/16.
template <int I>
__device__ __forceinline__ float nib_as_float(uint32_t w) {
  constexpr int sh = 19 - 4 * I;
  const uint32_t m = sh >= 0 ? (w << sh) : (w >> (-sh));
  return __uint_as_float((m & 0x00780000u) | 0x3F800000u);
}

// Locate the blockIdx.y-th non-empty, resident bin.  Returns false when
// there is none (the block has no work).
__device__ __forceinline__ bool find_bin(const GemvParams& P, int ordinal, int& bin, int& row0,
                                         int& nrows, int& blob_index, int& bits) {
  const int lane = threadIdx.x & 31;
  int seen = 0;
  for (int b0 = 0; b0 < P.nbins; b0 += 32) {
    const int b = b0 + lane;
    bool ok = false;
    int slot = 0;
    if (b < P.nbins) {
      const int n = min(max(P.offsets[b + 1], 0), P.rows) - min(max(P.offsets[b], 0), P.rows);
      const int e = b / P.planes_mult;
      slot = P.slot_of ? P.slot_of[e] : e;
      ok = n > 0 && slot >= 0;
    }
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    const int cnt = __popc(m);
    if (ordinal < seen + cnt) {
      // the (ordinal-seen)-th set bit of m
      int want = ordinal - seen;
      unsigned mm = m;
      for (int i = 0; i < want; ++i) mm &= mm - 1;
      const int src = __ffs(mm) - 1;
      bin = b0 + src;
      slot = __shfl_sync(0xffffffffu, slot, src);
      row0 = min(max(P.offsets[bin], 0), P.rows);
      nrows = max(0, min(max(P.offsets[bin + 1], 0), P.rows) - row0);
      blob_index = slot;
      bits = P.planes_mult == 3 ? 2 + bin % 3 : 4;
      return true;
    }
    seen += cnt;
  }
  return false;
}

// Load the 32 codes of row `r` at element offset k0 as 4 code words (INT4:
// nibble i = element i; planes: element 2j in nibble j, 2j+1 in nibble 4+j).
template <bool PLANES>
__device__ __forceinline__ uint4 load_codes(const GemvParams& P, const uint8_t* blob, int m,
                                            int row, int k0, int bits) {
  if (!PLANES) {
    const uint32_t* c = reinterpret_cast<const uint32_t*>(blob + P.code_off[m] + code_byte(row, k0 / 2, P.K, 64));
    return ldg_nc_v4(c);
  } else {
    const uint32_t* q2 = reinterpret_cast<const uint32_t*>(blob + P.code_off[m] + code_byte(row, k0 / 4, P.K, 32));
    uint2 base;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(base.x), "=r"(base.y)
                 : "l"(q2));
    uint32_t r3 = 0, r4 = 0;
    if (bits >= 3)
      r3 = ldg_nc_u32(blob + P.d3_off[m] + code_byte(row, k0 / 8, P.K, 16));
    if (bits >= 4)
      r4 = ldg_nc_u32(blob + P.d4_off[m] + code_byte(row, k0 / 8, P.K, 16));
    // plane-order code words (element 2j in nibble j, 2j+1 in nibble 4+j):
    // word wd takes the base from bits 2(wd & 1) of each nibble of Q2 word
    // wd >> 1 and the residuals from bit wd of the D3/D4 word
    uint4 out;
    out.x = (base.x << 2) & 0xCCCCCCCCu;
    out.y = base.x & 0xCCCCCCCCu;
    out.z = (base.y << 2) & 0xCCCCCCCCu;
    out.w = base.y & 0xCCCCCCCCu;
    if (bits >= 3) {
      out.x |= (r3 << 1) & 0x22222222u;
      out.y |= r3 & 0x22222222u;
      out.z |= (r3 >> 1) & 0x22222222u;
      out.w |= (r3 >> 2) & 0x22222222u;
    }
    if (bits >= 4) {
      out.x |= r4 & 0x11111111u;
      out.y |= (r4 >> 1) & 0x11111111u;
      out.z |= (r4 >> 2) & 0x11111111u;
      out.w |= (r4 >> 3) & 0x11111111u;
    }
    return out;
  }
}

// RW output rows per warp; NM matrices (2 = gate+up, 1 = down).
template <int MAXR, int NM, int RW, bool PLANES>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, MAXR == 1 ? 2 : (MAXR == 2 ? 3 : 1)) k_gemv(const GemvParams P) {
  constexpr int ROWS = NM * RW;  // weight rows per warp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // gate/up: wait for the earlier kernels, then let the down pass launch;
  // down: h is read only after the wait below (the weight codes before it)
  if (NM == 2) {
    pdl_wait();
    pdl_trigger();
  }
  bool dep_waited = NM == 2;
  int bin, row0, nrows, blob_index, bits;
  if (!find_bin(P, blockIdx.y, bin, row0, nrows, blob_index, bits)) return;
  const uint8_t* blob = P.blobs + static_cast<size_t>(blob_index) * P.blob_bytes;
  const int n0 = (blockIdx.x * kWarpsPerBlock + warp) * RW;  // first output row of this warp
  if (n0 >= P.N) return;

  // Bins with more than MAXR rows (only when this regime is used beyond its
  // intended T) are processed MAXR rows at a time.
  const int bin_row0 = row0, bin_rows = nrows;
  for (int rc = 0; rc < bin_rows; rc += MAXR) {
  row0 = bin_row0 + rc;
  nrows = min(MAXR, bin_rows - rc);
  float acc[ROWS][MAXR];
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int t = 0; t < MAXR; ++t) acc[r][t] = 0.0f;

  const int G = P.K / P.group;
  for (int kc = 0; kc < P.K; kc += kChunkSteps * 1024) {
    uint4 codes[kChunkSteps][ROWS];
    uint32_t sz[kChunkSteps][ROWS];
#pragma unroll
    for (int s = 0; s < kChunkSteps; ++s) {
      const int k0 = kc + s * 1024 + lane * 32;
      if (k0 < P.K) {
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
          const int m = r % NM, row = n0 + r / NM;
          codes[s][r] = load_codes<PLANES>(P, blob, m, row, k0, bits);
          const uint32_t* szp = reinterpret_cast<const uint32_t*>(blob + P.sz_off[m]);
          sz[s][r] = ldg_nc_u32(szp + (static_cast<size_t>(row >> 7) * G + k0 / P.group) * 128 + (row & 127));
        }
      }
    }
    if (!dep_waited) {
      pdl_wait();
      pdl_trigger();
      dep_waited = true;
    }
#pragma unroll
    for (int s = 0; s < kChunkSteps; ++s) {
      const int k0 = kc + s * 1024 + lane * 32;
      if (k0 >= P.K) continue;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {  // 8 elements per word
        float xv[MAXR][8], px[MAXR];
#pragma unroll
        for (int t = 0; t < MAXR; ++t) {
          px[t] = 0.0f;
          if (t < nrows) {
            const uint4 raw = *reinterpret_cast<const uint4*>(P.act + static_cast<size_t>(row0 + t) * P.K + k0 + wi * 8);
            const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
            float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __half22float2(h2[j]);
              xv[t][2 * j] = f.x;
              xv[t][2 * j + 1] = f.y;
              s2 = __fadd2_rn(s2, f);
            }
            px[t] = s2.x + s2.y;
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) xv[t][j] = 0.0f;
          }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
          const uint32_t w = wi == 0 ? codes[s][r].x : wi == 1 ? codes[s][r].y : wi == 2 ? codes[s][r].z : codes[s][r].w;
          // element e of the word: nibble e (INT4) or nibble (e >> 1) + 4 (e & 1) (planes)
          const float f0 = nib_as_float<0>(w), f1 = nib_as_float<PLANES ? 4 : 1>(w),
                      f2 = nib_as_float<PLANES ? 1 : 2>(w), f3 = nib_as_float<PLANES ? 5 : 3>(w),
                      f4 = nib_as_float<PLANES ? 2 : 4>(w), f5 = nib_as_float<PLANES ? 6 : 5>(w),
                      f6 = nib_as_float<PLANES ? 3 : 6>(w), f7 = nib_as_float<7>(w);
          const float sc = __uint_as_float(sz[s][r] << 16);
          const float zp = __uint_as_float(sz[s][r] & 0xFFFF0000u);
#pragma unroll
          for (int t = 0; t < MAXR; ++t) {
            // even and odd elements as the two lanes of packed fp32 FMAs
            float2 p2 = __fmul2_rn(make_float2(f0, f1), make_float2(xv[t][0], xv[t][1]));
            p2 = __ffma2_rn(make_float2(f2, f3), make_float2(xv[t][2], xv[t][3]), p2);
            p2 = __ffma2_rn(make_float2(f4, f5), make_float2(xv[t][4], xv[t][5]), p2);
            p2 = __ffma2_rn(make_float2(f6, f7), make_float2(xv[t][6], xv[t][7]), p2);
            const float p = p2.x + p2.y;
            // sum (q - z) x = 16 (p - px) - z px
            const float qx = 16.0f * (p - px[t]);
            acc[r][t] = fmaf(sc, fmaf(-zp, px[t], qx), acc[r][t]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int t = 0; t < MAXR; ++t) {
      float v = acc[r][t];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[r][t] = v;
    }
  if (lane == 0) {
#pragma unroll
    for (int t = 0; t < MAXR; ++t) {
      if (t >= nrows) break;
      const size_t p = static_cast<size_t>(row0 + t);
#pragma unroll
      for (int j = 0; j < RW; ++j) {
        if (NM == 2) {
          const float g = acc[2 * j][t], u = acc[2 * j + 1][t];
          P.h_out[p * P.N + n0 + j] = __float2half_rn(silu_f(g) * u);
        } else {
          if (!(fabsf(acc[j][t]) <= 65504.0f)) flag_status(P.status, MOE_DEV_RANGE);
          P.y_out[p * P.N + n0 + j] = __float2half_rn(acc[j][t]);
        }
      }
    }
  }
  }
}

template <int MAXR, bool PLANES>
moe_status_t run_pair(GemvParams gu, GemvParams dn, int max_bins, cudaStream_t s) {
  // one token per bin: twice the rows per warp, so that the grid (8 warps
  // per block) fits the resident blocks of one wave
  constexpr int RW_GU = MAXR == 1 ? 4 : 2, RW_DN = MAXR == 1 ? 8 : 4;
  dim3 g1(ceil_div(gu.N, kWarpsPerBlock * RW_GU), max_bins);
  moe_status_t st = cuda_check(launch_pdl(true, k_gemv<MAXR, 2, RW_GU, PLANES>, g1, dim3(kWarpsPerBlock * 32), 0, s, gu),
                               "ffn gemv gate/up launch");
  if (st != MOE_OK) return st;
  dim3 g2(ceil_div(dn.N, kWarpsPerBlock * RW_DN), max_bins);
  return cuda_check(launch_pdl(true, k_gemv<MAXR, 1, RW_DN, PLANES>, g2, dim3(kWarpsPerBlock * 32), 0, s, dn),
                    "ffn gemv down launch");
}

}  // namespace

moe_status_t launch_ffn_gemv(const FfnArgs& a, cudaStream_t s) {
  const bool planes = a.layout == MOE_LAYOUT_PLANES;
  const int mult = planes ? 3 : 1;
  const int nbins = a.E * mult;
  GemvParams gu{};
  gu.act = a.x_perm;
  gu.offsets = a.offsets;
  gu.blobs = a.blobs;
  gu.slot_of = a.slot_of;
  gu.blob_bytes = a.blob_bytes;
  gu.K = a.d;
  gu.N = a.F;
  gu.nbins = nbins;
  gu.planes_mult = mult;
  gu.group = a.group;
  gu.h_out = a.h;
  gu.rows = a.total_rows;
  gu.status = a.status;
  for (int m = 0; m < 2; ++m) {
    gu.code_off[m] = planes ? a.lay.q2[m] : a.lay.codes[m];
    gu.d3_off[m] = a.lay.d3[m];
    gu.d4_off[m] = a.lay.d4[m];
    gu.sz_off[m] = a.lay.sz[m];
  }
  GemvParams dn = gu;
  dn.act = a.h;
  dn.K = a.F;
  dn.N = a.d;
  dn.h_out = nullptr;
  dn.y_out = a.y_perm;
  dn.code_off[0] = planes ? a.lay.q2[2] : a.lay.codes[2];
  dn.d3_off[0] = a.lay.d3[2];
  dn.d4_off[0] = a.lay.d4[2];
  dn.sz_off[0] = a.lay.sz[2];
  const int max_bins = std::min(nbins, a.total_rows);
  if (max_bins == 0) return MOE_OK;
  const int T = a.T;
  if (planes) {
    if (T <= 1) return run_pair<1, true>(gu, dn, max_bins, s);
    if (T <= 2) return run_pair<2, true>(gu, dn, max_bins, s);
    if (T <= 4) return run_pair<4, true>(gu, dn, max_bins, s);
    return run_pair<8, true>(gu, dn, max_bins, s);
  }
  if (T <= 1) return run_pair<1, false>(gu, dn, max_bins, s);
  if (T <= 2) return run_pair<2, false>(gu, dn, max_bins, s);
  if (T <= 4) return run_pair<4, false>(gu, dn, max_bins, s);
  return run_pair<8, false>(gu, dn, max_bins, s);
}

}  // namespace moeq
