// Small-batch grouped expert FFN: weight rows streamed through shared
// memory, dot products on the tensor cores (mma.sync m16n8k16).
//
// Used for batches of a few to a few tens of tokens, where a bin holds too
// few rows for a 128-row tensor-core tile to pay for its dequantisation but
// more than the one-token GEMV handles well: the cost per weight does not
// grow with the bin's rows (up to 16 per pass).  A warp owns 16 weight rows
// (8 features x {gate, up}, or 16 rows of W_down) and streams them in
// stages of 256 K (128 B per row) with cp.async into a ring of S
// shared-memory stages (S = 4 or 8: the whole K when it fits, so that a
// warp's weights are requested at once); the bytes in flight do not depend
// on registers.  Each lane dequantises its own 64 K of each row: lane
// (g, c) = (lane / 4, lane % 4) holds MMA operand B for weight row g of an
// 8-row group and the K slots of quad c; the four nibble pairs of a code
// word become fp16 (code - z) * s (one rounding, as in the 128-row kernel)
// and feed two MMAs.  Operand A holds the bin's token rows (16 per pass);
// since the MMA sums over K, A takes the activations in the same K order as
// the pairs B holds (INT4 words give pairs (0,4), (1,5), ...; plane-order
// words give (0,1), (2,3), ...).  Accumulation is fp32 in the MMA.
// blockIdx.y enumerates the non-empty (and, in slot mode, resident) bins;
// blockIdx.x a block of kWarps warps x 16 rows.
//
// Both passes are programmatic dependent launches (launch_pdl).  The down
// pass starts while the gate/up pass runs, locates its bin and issues the
// copies of its first weight stages (which do not depend on h), and only
// then waits for the gate/up grid before reading h.  The gate/up pass
// triggers after its own wait, so everything the down pass reads before
// its wait (offsets, slot table, weights) is complete by then.
//
//   gate/up pass:  h[p][f]      = silu(Wg[f] . x_p) * (Wu[f] . x_p)   (fp16)
//   down pass:     y_perm[p][n] = Wd[n] . h_p                          (fp16)
#include <algorithm>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kWarps = 4;        // warps per block
constexpr int kStageK = 256;     // K per stage
constexpr int kRowPitch = 144;   // bytes per row per stage: 128 + 16 (bank spread)
constexpr int kStageBytes = 16 * kRowPitch;                 // 16 rows
constexpr int kSzWords = 2 * 32;                            // 2 fragments x 32 lanes
constexpr int warp_smem(int S) { return S * (kStageBytes + kSzWords * 4); }
constexpr int kMaxRows = 16;     // token rows per pass (MMA M)

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

// (a & m) | c in one instruction.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t c) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(m), "r"(c));
  return r;
}

// The four nibble pairs (0,4), (1,5), (2,6), (3,7) of a 32-bit code word as
// fp16 (code - z) * s, in that order.  Masking nibbles (j, 4+j) into
// 0x6400 gives the half2 (1024 + n_j, 1024 + n_4+j); nibbles at bits 4..7
// of each half, masked into 0x5400, read as (64 + n, 64 + n) (their unit at
// exponent 64 is 1/16).  Subtracting (1024 + z) or (64 + z) is exact; one
// multiply by s rounds each product once.  z_lo = (1024 + z) twice, z_hi =
// (64 + z) twice.
__device__ __forceinline__ uint4 dequant_pairs(uint32_t w, __half2 z_lo, __half2 z_hi, __half2 s2) {
  const uint32_t w8 = w >> 8;
  const uint32_t r[4] = {and_or(w, 0x000F000Fu, 0x64006400u), and_or(w, 0x00F000F0u, 0x54005400u),
                         and_or(w8, 0x000F000Fu, 0x64006400u), and_or(w8, 0x00F000F0u, 0x54005400u)};
  uint32_t v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __half2 h = *reinterpret_cast<const __half2*>(&r[j]);
    h = __hmul2(__hsub2(h, (j & 1) ? z_hi : z_lo), s2);
    v[j] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte pieces of one row's stage: INT4 pieces 0..7 = codes of K 32p..;
// planes: 0..3 Q2 (64 K each), 4..5 D3 (128 K each), 6..7 D4.
template <bool PLANES>
__device__ __forceinline__ bool piece_src(const GemvParams& P, const uint8_t* blob, int m, int row, int k0,
                                          int p, int bits, const uint8_t*& src) {
  const int kv = min(kStageK, P.K - k0);  // 256, or 128 at a ragged end
  if (!PLANES) {
    if (32 * p >= kv) return false;
    src = blob + P.code_off[m] + code_byte(row, k0 / 2 + 16 * p, P.K, 64);
    return true;
  }
  if (p < 4) {
    if (64 * p >= kv) return false;
    src = blob + P.code_off[m] + code_byte(row, k0 / 4 + 16 * p, P.K, 32);
    return true;
  }
  const int q = (p - 4) & 1;
  if (128 * q >= kv) return false;
  if (p < 6) {
    if (bits < 3) return false;
    src = blob + P.d3_off[m] + code_byte(row, k0 / 8 + 16 * q, P.K, 16);
  } else {
    if (bits < 4) return false;
    src = blob + P.d4_off[m] + code_byte(row, k0 / 8 + 16 * q, P.K, 16);
  }
  return true;
}

// NM matrices (2 = gate+up of the same 8 features, 1 = down); RG 8-row
// groups per matrix; NM * RG = 2 fragments (16 rows) per warp.  HI: bins
// may hold more than 8 rows (T > 8: the tensor-core kernel does not take
// the shape, or the regime is forced), and token rows 8..15 of the MMA are
// used; without it the activations of stage i + 1 are loaded while stage i
// is computed.
template <int NM, int RG, bool PLANES, bool HI, int S>
__global__ void __launch_bounds__(kWarps * 32) k_gemv(const GemvParams P) {
  static_assert(NM * RG == 2, "two 8-row fragments per warp");
  constexpr int kStages = S;
  constexpr int kWarpSmem = warp_smem(S);
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
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
  const int n0 = (blockIdx.x * kWarps + warp) * 8 * RG;  // first output row of this warp
  if (n0 >= P.N) return;
  uint8_t* wsm = smem_raw + warp * kWarpSmem;
  const uint32_t wsm_u = static_cast<uint32_t>(__cvta_generic_to_shared(wsm));
  const int G = P.K / P.group;
  const int n_stages = (P.K + kStageK - 1) / kStageK;

  // fragment b: matrix b % NM, rows n0 + 8 (b / NM) + 0..7
  auto frag_row = [&](int b, int j) { return n0 + 8 * (b / NM) + j; };
  // copies of stage i into ring slot i % kStages: 16 rows x 8 pieces over
  // the 32 lanes, plus each lane's own two scale/zero words
  auto issue = [&](int i) {
    if (i < n_stages) {
      const int k0 = i * kStageK;
      const int slot = i % kStages;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = lane + 32 * u;   // 0..127
        const int rr = q >> 3, p = q & 7;
        const int b = rr >> 3;
        const uint8_t* src;
        if (piece_src<PLANES>(P, blob, b % NM, frag_row(b, rr & 7), k0, p, bits, src))
          cp_async16(wsm_u + slot * kStageBytes + rr * kRowPitch + 16 * p, src);
      }
      const int kl = k0 + 64 * c;
      if (kl < P.K) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int row = frag_row(b, g);
          const uint8_t* szp = blob + P.sz_off[b % NM] +
                               ((static_cast<size_t>(row >> 7) * G + kl / P.group) * 128 + (row & 127)) * 4;
          cp_async4(wsm_u + kStages * kStageBytes + (slot * kSzWords + b * 32 + lane) * 4, szp);
        }
      }
    }
    cp_async_commit();  // an empty group past the end keeps the count uniform
  };

  const int bin_row0 = row0, bin_rows = nrows;
  for (int rc = 0; rc < bin_rows; rc += kMaxRows) {
    row0 = bin_row0 + rc;
    nrows = min(kMaxRows, bin_rows - rc);
    __syncwarp();  // the previous pass's reads of the ring are done
#pragma unroll
    for (int i = 0; i < kStages; ++i) issue(i);
    if (!dep_waited) {
      pdl_wait();
      pdl_trigger();
      dep_waited = true;
    }
    float acc[2][4];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[b][j] = 0.0f;
    const bool tok_lo = g < nrows, tok_hi = HI && g + 8 < nrows;
    const __half* xlo = P.act + static_cast<size_t>(row0 + g) * P.K;
    const __half* xhi = P.act + static_cast<size_t>(row0 + g + 8) * P.K;
    // this lane's 64 K of the token rows g and g + 8 for one stage
    auto load_x = [&](int i, const __half* xr, bool tok, uint4 (&xv)[8]) {
      const int kl = i * kStageK + 64 * c;
      const bool in = tok && i < n_stages && kl < P.K;
#pragma unroll
      for (int w = 0; w < 8; ++w)
        xv[w] = in ? *reinterpret_cast<const uint4*>(xr + kl + 8 * w) : make_uint4(0, 0, 0, 0);
    };
    uint4 xl[8], xh[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) xh[w] = make_uint4(0, 0, 0, 0);
    if (!HI) load_x(0, xlo, tok_lo, xl);
    for (int i = 0; i < n_stages; ++i) {
      uint4 nl[8];
      if (!HI) {
        load_x(i + 1, xlo, tok_lo, nl);
      } else {
        load_x(i, xlo, tok_lo, xl);
        load_x(i, xhi, tok_hi, xh);
      }
      cp_async_wait<kStages - 1>();
      __syncwarp();  // every lane's copies of stage i have landed
      const int slot = i % kStages;
      // lanes whose 64 K lie past a ragged K end feed zeros (the MMA is
      // warp-wide, so every lane issues it)
      const bool kin = i * kStageK + 64 * c < P.K;
      {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const uint8_t* rowp = wsm + slot * kStageBytes + (8 * b + g) * kRowPitch;
          const uint32_t word = reinterpret_cast<const uint32_t*>(wsm + kStages * kStageBytes)[slot * kSzWords + b * 32 + lane];
          const float zf = __uint_as_float(word & 0xFFFF0000u);
          const __half2 s2 = __half2half2(__float2half_rn(__uint_as_float(word << 16)));
          const __half2 zlo = __half2half2(__float2half_rn(1024.0f + zf));
          const __half2 zhi = __half2half2(__float2half_rn(64.0f + zf));
          uint32_t cw[8];  // this lane's 8 code words (64 K)
          if (!PLANES) {
            const uint4 c0 = *reinterpret_cast<const uint4*>(rowp + 32 * c);
            const uint4 c1 = *reinterpret_cast<const uint4*>(rowp + 32 * c + 16);
            cw[0] = c0.x; cw[1] = c0.y; cw[2] = c0.z; cw[3] = c0.w;
            cw[4] = c1.x; cw[5] = c1.y; cw[6] = c1.z; cw[7] = c1.w;
          } else {
            // plane-order words: base from bits 2(w & 1) of each nibble of
            // Q2 word w >> 1, residuals from bit (w & 3) of D3/D4 word w >> 2
            const uint4 q2 = *reinterpret_cast<const uint4*>(rowp + 16 * c);
            const uint32_t qw[4] = {q2.x, q2.y, q2.z, q2.w};
            uint2 d3 = make_uint2(0, 0), d4 = make_uint2(0, 0);
            if (bits >= 3) d3 = *reinterpret_cast<const uint2*>(rowp + 64 + 8 * c);
            if (bits >= 4) d4 = *reinterpret_cast<const uint2*>(rowp + 96 + 8 * c);
            const uint32_t r3[2] = {d3.x, d3.y}, r4[2] = {d4.x, d4.y};
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              uint32_t v = (qw[w >> 1] << (2 - 2 * (w & 1))) & 0xCCCCCCCCu;
              const int sh = 1 - (w & 3);
              if (bits >= 3) v = and_or(sh >= 0 ? r3[w >> 2] << sh : r3[w >> 2] >> -sh, 0x22222222u, v);
              if (bits >= 4) v = and_or(r4[w >> 2] >> (w & 3), 0x11111111u, v);
              cw[w] = v;
            }
          }
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            uint4 pr = dequant_pairs(cw[w], zlo, zhi, s2);
            if (!kin) pr = make_uint4(0, 0, 0, 0);
            // activations in the K order of the pairs
            uint32_t a0, a2, a0b, a2b, a1, a3, a1b, a3b;
            if (PLANES) {
              a0 = xl[w].x; a2 = xl[w].y; a0b = xl[w].z; a2b = xl[w].w;
              a1 = xh[w].x; a3 = xh[w].y; a1b = xh[w].z; a3b = xh[w].w;
            } else {
              a0 = __byte_perm(xl[w].x, xl[w].z, 0x5410); a2 = __byte_perm(xl[w].x, xl[w].z, 0x7632);
              a0b = __byte_perm(xl[w].y, xl[w].w, 0x5410); a2b = __byte_perm(xl[w].y, xl[w].w, 0x7632);
              a1 = __byte_perm(xh[w].x, xh[w].z, 0x5410); a3 = __byte_perm(xh[w].x, xh[w].z, 0x7632);
              a1b = __byte_perm(xh[w].y, xh[w].w, 0x5410); a3b = __byte_perm(xh[w].y, xh[w].w, 0x7632);
            }
            mma16816(acc[b], a0, a1, a2, a3, pr.x, pr.y);
            mma16816(acc[b], a0b, a1b, a2b, a3b, pr.z, pr.w);
          }
        }
      }
      __syncwarp();  // every lane is done with slot i % kStages
      issue(i + kStages);
      if (!HI) {
#pragma unroll
        for (int w = 0; w < 8; ++w) xl[w] = nl[w];
      }
    }
    cp_async_wait<0>();
    // D[token][n]: lane holds tokens g (acc[.][0..1]) and g + 8 (acc[.][2..3])
    // for rows 2c, 2c + 1 of each fragment
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
      const int tok = g + 8 * hi;
      if (tok >= nrows) continue;
      const size_t p = static_cast<size_t>(row0 + tok);
      if (NM == 2) {
        const float h0 = silu_f(acc[0][2 * hi]) * acc[1][2 * hi];
        const float h1 = silu_f(acc[0][2 * hi + 1]) * acc[1][2 * hi + 1];
        *reinterpret_cast<__half2*>(P.h_out + p * P.N + n0 + 2 * c) = __floats2half2_rn(h0, h1);
      } else {
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          const float y0 = acc[r][2 * hi], y1 = acc[r][2 * hi + 1];
          if (!(fmaxf(fabsf(y0), fabsf(y1)) <= 65504.0f)) flag_status(P.status, MOE_DEV_RANGE);
          *reinterpret_cast<__half2*>(P.y_out + p * P.N + n0 + 8 * r + 2 * c) = __floats2half2_rn(y0, y1);
        }
      }
    }
  }
}

template <int NM, int RG, bool PLANES, bool HI, int S>
moe_status_t run_one(const GemvParams& p, int max_bins, cudaStream_t s, const char* what) {
  constexpr int smem = kWarps * warp_smem(S);
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_gemv<NM, RG, PLANES, HI, S>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_check(e, what);
    if (dev < 64) attr_set[dev] = true;
  }
  const dim3 grid(ceil_div(p.N, kWarps * 8 * RG), max_bins);
  return cuda_check(launch_pdl(true, k_gemv<NM, RG, PLANES, HI, S>, grid, dim3(kWarps * 32), smem, s, p), what);
}

// Ring depth: the whole K of a row up to 8 stages (2048 K); deeper rings
// (16 stages, 160 KB per block) left one block per SM and measured slower.
template <int NM, int RG, bool PLANES, bool HI>
moe_status_t run_pass(const GemvParams& p, int max_bins, cudaStream_t s, const char* what) {
  const int stages = ceil_div(p.K, kStageK);
  if (stages <= 4) return run_one<NM, RG, PLANES, HI, 4>(p, max_bins, s, what);
  return run_one<NM, RG, PLANES, HI, 8>(p, max_bins, s, what);
}

template <bool PLANES, bool HI>
moe_status_t run_pair(const GemvParams& gu, const GemvParams& dn, int max_bins, cudaStream_t s) {
  const moe_status_t st = run_pass<2, 1, PLANES, HI>(gu, max_bins, s, "ffn gemv gate/up launch");
  if (st != MOE_OK) return st;
  return run_pass<1, 2, PLANES, HI>(dn, max_bins, s, "ffn gemv down launch");
}

}  // namespace

moe_status_t launch_ffn_gemv_mma(const FfnArgs& a, cudaStream_t s) {
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
  // HI: a bin may hold more than 8 rows (bins never hold more than T)
  if (a.T <= 8) return planes ? run_pair<true, false>(gu, dn, max_bins, s) : run_pair<false, false>(gu, dn, max_bins, s);
  return planes ? run_pair<true, true>(gu, dn, max_bins, s) : run_pair<false, true>(gu, dn, max_bins, s);
}

}  // namespace moeq
