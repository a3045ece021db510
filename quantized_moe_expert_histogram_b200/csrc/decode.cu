// Decode-regime grouped expert FFN: short bins (a few token rows each; a
// bin longer than a pass takes several passes), where the layer is bound by
// the bytes of the routed experts' weights.
//
// Swap-AB tensor-core dot products (mma.sync m16n8k16, fp32 accumulate):
// dequantised weight rows are operand A (16 rows x 16 K per instruction)
// and the bin's token rows operand B (N = 8 tokens), so one instruction
// consumes 256 weights whatever the number of tokens up to 8 (two per A
// fragment for 9-16 tokens).  A holds (code - zero) in fp16, which is exact;
// the scale of a 128-wide group is applied to the fp32 partial sum of that
// group, acc += s * sum_k (q_k - z) x_k (for groups of 64, where one lane's
// K run spans two groups, A holds (q - z) * s rounded once to fp16, as in
// the 128-row kernel).
//
// Work split: a work unit is (bin, block of weight rows, pass over 8 NB of
// the bin's token rows): 16 features x {gate, up} in the first GEMM, 16 or
// 32 rows of W_down in the second.  The grid is persistent (as many CTAs as
// fit on the GPU at once); CTA b takes units b, b + grid, ...  The W warps
// of a CTA (8, or 12 where that balances the units better) split each
// unit's K: warp w takes the 128-K stages w, w+W, w+2W, ... of every row of
// the unit (so a 14336-long row is all the warps' work; a stage of a
// 16-row fragment is one contiguous 1 KB code tile of the blob).  Each
// warp streams its stages with cp.async into a shared-memory ring (the bytes
// in flight take no registers), and the stream runs on across units: the
// next unit's first stages are in flight while the current unit's partial
// sums are added (in shared memory, in a fixed order: deterministic) and its
// epilogue writes h = silu(gate) * up or y_perm (fp16).  The non-empty,
// resident bins are listed once per CTA in shared memory.
//
// Register layout of one MMA, lane = (g, c) = (lane / 4, lane % 4): A rows g
// and g + 8, K slots {2c, 2c+1, 2c+8, 2c+9}; B token g at the same slots;
// D rows g, g + 8 x tokens 2c, 2c + 1.  The sum runs over K, so each lane
// feeds its K slots from its own run of 32 consecutive elements of the
// stage: a code word (8 elements) gives four fp16 pairs by masking nibble
// pairs into the mantissa of 1024 (low nibbles) or 64 (high nibbles), and
// the activations are paired the same way -- elements (j, j + 4) for INT4
// words, (2j, 2j + 1) for plane-order words.
//
// Both passes are programmatic dependent launches (launch_pdl).  The down
// pass lists its bins and issues the copies of its first weight stages
// (which do not depend on h) before it waits for the gate/up grid.
//
//   gate/up pass:  h[p][f]      = silu(Wg[f] . x_p) * (Wu[f] . x_p)   (fp16)
//   down pass:     y_perm[p][n] = Wd[n] . h_p                          (fp16)
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kStageK = 128;       // K per stage (one group of 128, two of 64)
constexpr int kFragBytes = 1024;   // one stage of one 16-row fragment: 16 rows x 64 B
constexpr int kSzBytes = 128;      // its scale/zero words: 16 rows x up to 2 groups
constexpr int kRing = 2;           // stages in flight per warp (3 measured 0.5-2 % slower)

struct DecParams {
  const __half* act;        // x_perm or h: fp16 [rows][K]
  const int32_t* offsets;   // [nbins + 1]
  const uint8_t* blobs;
  const int32_t* slot_of;
  size_t blob_bytes;
  size_t code_off[2];       // INT4 codes (or Q2) of matrix 0 / 1
  size_t d3_off[2];
  size_t d4_off[2];
  size_t sz_off[2];
  int K, N, nbins, planes_mult;
  int rows;                 // activation rows: bin ranges are clamped into [0, rows]
  int group;
  int row_blocks;           // weight-row blocks per bin
  int max_ent;              // capacity of the bin list (>= non-empty bins)
  __half* out;              // h (gate/up) or y_perm (down): fp16 [rows][N]
  int32_t* status;
};

// One listed bin: its rows, blob, width and its first work unit.
struct BinEnt {
  int row0, nrows, slot, bits, unit0;
};

__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t c) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(m), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// The four fp16 pairs of a code word: nibbles (0,4), (1,5), (2,6), (3,7)
// minus the zero-point.  Nibbles masked into 0x6400 read as 1024 + n, those
// at bits 4..7 of a half masked into 0x5400 as 64 + n (unit 1/16 at 64);
// z_lo = 1024 + z, z_hi = 64 + z (both exact), so each pair is exactly
// (n - z).  For an INT4 word these are elements (j, j + 4); for a
// plane-order word elements (2j, 2j + 1).
__device__ __forceinline__ void pairs(uint32_t w, __half2 z_lo, __half2 z_hi, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = h2u(__hsub2(u2h(and_or(w, 0x000F000Fu, 0x64006400u)), z_lo));
  p[1] = h2u(__hsub2(u2h(and_or(w, 0x00F000F0u, 0x54005400u)), z_hi));
  p[2] = h2u(__hsub2(u2h(and_or(w8, 0x000F000Fu, 0x64006400u)), z_lo));
  p[3] = h2u(__hsub2(u2h(and_or(w8, 0x00F000F0u, 0x54005400u)), z_hi));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// D += A B (register-only: the compiler may schedule it freely)
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A B (a fresh accumulator)
__device__ __forceinline__ void mma16816_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ uint4 ldg_act(const __half* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
  return r;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
  return r;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(a));
  return r;
}

// Shared-memory layout of a CTA: the warps' rings, the reduction buffer,
// the bin list.
template <int FW, int NB, int W>
struct Smem {
  static constexpr int kSlot = FW * (kFragBytes + kSzBytes);  // one ring stage of a warp
  static constexpr int kVals = FW * NB * 4;                    // partial sums per lane
  static constexpr int kRing0 = 0;
  static constexpr int kRed0 = W * kRing * kSlot;
  static constexpr int kEnt0 = kRed0 + W * kVals * 32 * 4;
  static constexpr size_t bytes(int max_ent) { return kEnt0 + static_cast<size_t>(max_ent) * sizeof(BinEnt); }
};

// GU: first GEMM (fragment 0 = gate rows, 1 = up rows of 16 features);
// else the second GEMM (FW fragments of 16 consecutive W_down rows).  NB
// token blocks of 8 per pass over K.
// Residency: 24 warps per SM (<= 80 registers) with one token block (three
// CTAs of 8 warps or two of 12); two CTAs of 8 warps with two token blocks,
// whose B operands need more registers.
template <bool GU, bool PLANES, bool G64, int FW, int NB, int W>
__global__ void __launch_bounds__(W * 32, NB == 1 && W == 8 ? 3 : 2) k_dec(const DecParams P) {
  static_assert(!GU || FW == 2, "gate and up fragments");
  static_assert(W == 8 || W == 12, "warps per CTA");
  constexpr int kWarps = W;
  using L = Smem<FW, NB, W>;
  constexpr int kSlot = L::kSlot;
  constexpr int kVals = L::kVals;
  extern __shared__ __align__(16) uint8_t smem[];
  float* red = reinterpret_cast<float*>(smem + L::kRed0);
  BinEnt* ent = reinterpret_cast<BinEnt*>(smem + L::kEnt0);
  __shared__ int n_ent_s, n_units_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  if (GU) {  // x_perm comes from the previous launch
    pdl_wait();
    pdl_trigger();
  }
  // ---- the non-empty, resident bins and their work units (warp 0): units
  // of a bin = passes x row blocks, passes = ceil(rows / (8 NB))
  if (warp == 0) {
    int n_ent = 0, n_units = 0;
    for (int b0 = 0; b0 < P.nbins; b0 += 32) {
      const int b = b0 + lane;
      int r0 = 0, nr = 0, sl = 0;
      if (b < P.nbins) {
        r0 = min(max(P.offsets[b], 0), P.rows);
        nr = max(0, min(max(P.offsets[b + 1], 0), P.rows) - r0);
        sl = P.slot_of ? P.slot_of[b / P.planes_mult] : b / P.planes_mult;
      }
      const bool ok = nr > 0 && sl >= 0;
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      const int units = ok ? ((nr + 8 * NB - 1) / (8 * NB)) * P.row_blocks : 0;
      int incl = units;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (ok) {
        const int pos = n_ent + __popc(m & ((1u << lane) - 1u));
        if (pos < P.max_ent)
          ent[pos] = BinEnt{r0, nr, sl, P.planes_mult == 3 ? 2 + b % 3 : 4, n_units + incl - units};
      }
      n_ent += __popc(m);
      n_units += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      n_ent_s = min(n_ent, P.max_ent);  // the list holds at most max_ent bins
      n_units_s = n_ent <= P.max_ent ? n_units : 0;
      if (n_ent > P.max_ent) flag_status(P.status, MOE_DEV_BAD_INDEX);
    }
  }
  __syncthreads();
  const int n_ent = n_ent_s, n_units = n_units_s;
  const int my_units = static_cast<int>(blockIdx.x) < n_units ? (n_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (my_units == 0) {
    if (!GU) pdl_wait();  // CTA-uniform; keeps the wait/trigger order of every CTA
    return;
  }
  const int n_stages = P.K / kStageK;
  const int G = P.K / P.group;
  const int my_stages = n_stages > warp ? (n_stages - warp + kWarps - 1) / kWarps : 0;
  const uint32_t ring_u = static_cast<uint32_t>(__cvta_generic_to_shared(smem + L::kRing0 + warp * (kRing * kSlot)));
  const int rows_per_unit = GU ? 16 : 16 * FW;
  auto mat = [](int f) { return GU ? f : 0; };

  // unit u -> (listed bin, pass, row block)
  auto locate = [&](int u, int& e, int& pass, int& rb) {
    int lo = 0, hi = n_ent;  // largest e with ent[e].unit0 <= u
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (ent[mid].unit0 <= u) lo = mid; else hi = mid;
    }
    e = lo;
    const int local = u - ent[lo].unit0;
    pass = local / P.row_blocks;
    rb = local - pass * P.row_blocks;
  };

  // ---- copy side: this warp's stream of stages, unit by unit.  Per
  // fragment: INT4 16 rows x 64 B of codes; planes 16 rows x (32 B Q2 + 16 B
  // D3 + 16 B D4); then 16 rows x 1 or 2 groups of (scale, zero) words,
  // contiguous.  The blob stores code words in tiles of 16 rows x 128 K, so a
  // fragment's stage is one contiguous tile of each kind (1 KB of INT4
  // codes; 512 B of Q2, 256 B of D3, of D4).  A lane copies 16 bytes at ring
  // offset lane * 16 (piece 0) and 512 + lane * 16 (piece 1) of each
  // fragment: bytes lane * 16 and 512 + lane * 16 of the INT4 tile, or of the
  // Q2 tile and of the D3 (lanes below 16) / D4 tile (planes; a null base:
  // plane not needed), and a scale/zero piece (lanes below 4, or 8 for groups
  // of 64).  Fragment f's sources are fragment 0's plus f times a fixed
  // stride (the up matrix, or the next 16-row block), so the stream keeps one
  // base per kind of piece.
  constexpr int kStep0 = PLANES ? 512 : 1024;  // piece 0 advance per stage: the next tile of codes, or Q2
  constexpr int kStep1 = 256;                  // planes' piece 1: D3 / D4
  const int sz_step = (kStageK / P.group) * 512;
  const size_t fs_c = GU ? P.code_off[1] - P.code_off[0] : static_cast<size_t>(PLANES ? 4 : 8) * P.K;
  const size_t fs_d = GU ? P.d3_off[1] - P.d3_off[0] : 2 * static_cast<size_t>(P.K);
  const size_t fs_sz = GU ? P.sz_off[1] - P.sz_off[0] : 64;
  const uint8_t* cp = nullptr;   // piece 0 of fragment 0 (codes or Q2)
  const uint8_t* dp = nullptr;   // planes: piece 1 of fragment 0 (D3 / D4), null when not needed
  const uint8_t* szp = nullptr;  // scale/zero piece of fragment 0
  const bool sz_lane = lane < (G64 ? 8 : 4);
  const uint32_t sz_dst = FW * kFragBytes + ((lane >> 2) & 1) * 64 + (lane & 3) * 16;
  int iq = 0, ii = 0;  // unit (of this CTA) and stage (of this warp) of the next copy
  // copy bases of this warp's first stage of unit q
  auto bases = [&](int q) {
    int e, pass, rb;
    locate(blockIdx.x + q * gridDim.x, e, pass, rb);
    const BinEnt be = ent[e];
    const uint8_t* blob = P.blobs + static_cast<size_t>(be.slot) * P.blob_bytes;
    const int n0 = rb * rows_per_unit;
    const size_t tile = static_cast<size_t>(n0 >> 4) * (P.K / kStageK) + warp;  // (16-row block, first stage)
    cp = blob + P.code_off[0] + tile * kStep0 + lane * 16;
    if (PLANES) {
      const bool want = lane < 16 ? be.bits >= 3 : be.bits >= 4;
      dp = want ? blob + (lane < 16 ? P.d3_off[0] : P.d4_off[0]) + tile * kStep1 + (lane & 15) * 16 : nullptr;
    }
    szp = blob + P.sz_off[0] + (static_cast<size_t>(n0 >> 7) * G + ((lane >> 2) & 1)) * 512 + (n0 & 127) * 4 +
          (lane & 3) * 16 + warp * sz_step;
  };
  // the next stage of the stream into ring slot j % kRing (j = 0, 1, ... in
  // order); past the stream's end an empty group keeps the count uniform
  auto issue = [&](int j) {
    if (iq < my_units && my_stages > 0) {
      if (ii == 0) bases(iq);
      const uint32_t slot = ring_u + (j % kRing) * kSlot;
#pragma unroll
      for (int f = 0; f < FW; ++f) {
        const uint32_t d0 = slot + f * kFragBytes + lane * 16;
        cp_async16(d0, cp + f * fs_c);
        if (!PLANES) cp_async16(d0 + 512, cp + f * fs_c + 512);
        else if (dp) cp_async16(d0 + 512, dp + f * fs_d);
        if (sz_lane) cp_async16(slot + sz_dst + f * kSzBytes, szp + f * fs_sz);
      }
      cp += kWarps * kStep0;
      if (PLANES && dp) dp += kWarps * kStep1;
      szp += kWarps * sz_step;
      if (++ii == my_stages) {
        ii = 0;
        ++iq;
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int j = 0; j < kRing; ++j) issue(j);
  if (!GU) {  // down pass: h is read only from here on
    pdl_wait();
    pdl_trigger();
  }

  int j = 0;  // stream position of the stage being computed
  for (int q = 0; q < my_units; ++q) {
    int e, pass, rb;
    locate(blockIdx.x + q * gridDim.x, e, pass, rb);
    const BinEnt be = ent[e];
    const int t0 = pass * 8 * NB, n0 = rb * rows_per_unit;
    const int ntok = min(8 * NB, be.nrows - t0);  // token rows of this unit
    // this lane's run of each token row it feeds (token g of each 8-token
    // block), advanced by one stage of this warp (8 x 128 K) per stage
    bool tok_in[NB];
    const __half* xp[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      tok_in[nb] = 8 * nb + g < ntok;
      xp[nb] = P.act + static_cast<size_t>(be.row0 + t0 + (tok_in[nb] ? 8 * nb + g : 0)) * P.K + warp * kStageK + 32 * c;
    }
    // the unit's activation runs into L1 ahead of their use when they fit
    // (a stage's 128 K of one token row is two 128-byte lines)
    if (ntok * P.K * 2 <= (48 << 10) && (c & 1) == 0) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        if (tok_in[nb])
          for (int i = 0; i < my_stages; ++i)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(xp[nb] + i * kWarps * kStageK));
    }
    float acc[FW][NB][4];
#pragma unroll
    for (int f = 0; f < FW; ++f)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[f][nb][jj] = 0.0f;
    for (int i = 0; i < my_stages; ++i, ++j) {
      // activations (4 x 8 elements per token block), loaded before the wait
      uint4 xv[NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int wd = 0; wd < 4; ++wd)
          xv[nb][wd] = tok_in[nb] ? ldg_act(xp[nb] + 8 * wd) : make_uint4(0, 0, 0, 0);
        xp[nb] += kWarps * kStageK;
      }
      cp_async_wait<kRing - 1>();
      __syncwarp();
      const uint32_t sb = ring_u + (j % kRing) * kSlot;  // this stage's ring slot
#pragma unroll
      for (int f = 0; f < FW; ++f) {
        const uint32_t fb = sb + f * kFragBytes;
        const uint32_t szw = sb + FW * kFragBytes + f * kSzBytes + (G64 ? (c >> 1) * 64 : 0) + g * 4;
        const uint32_t wlo = lds32(szw), whi = lds32(szw + 32);  // rows g and g + 8
        const float slo = __uint_as_float(wlo << 16), shi = __uint_as_float(whi << 16);
        // zero-points are integers 0..15: 1024 + z and 64 + z as fp16 bit
        // patterns (units 1 and 1/16 of the mantissa), in both halves
        const uint32_t zi_lo = static_cast<uint32_t>(__float2int_rz(__uint_as_float(wlo & 0xFFFF0000u)));
        const uint32_t zi_hi = static_cast<uint32_t>(__float2int_rz(__uint_as_float(whi & 0xFFFF0000u)));
        const __half2 za_lo = u2h(0x64006400u + zi_lo * 0x10001u);
        const __half2 za_hi = u2h(0x54005400u + (zi_lo << 4) * 0x10001u);
        const __half2 zb_lo = u2h(0x64006400u + zi_hi * 0x10001u);
        const __half2 zb_hi = u2h(0x54005400u + (zi_hi << 4) * 0x10001u);
        // this lane's 32 elements of rows g and g + 8 as four code words each
        uint32_t ca[4], cb[4];
        if (!PLANES) {
          const uint4 va = lds128(fb + g * 64 + c * 16);
          const uint4 vb = lds128(fb + (g + 8) * 64 + c * 16);
          ca[0] = va.x; ca[1] = va.y; ca[2] = va.z; ca[3] = va.w;
          cb[0] = vb.x; cb[1] = vb.y; cb[2] = vb.z; cb[3] = vb.w;
        } else {
          // plane-order words: base from bits 2 (wd & 1) of each nibble of Q2
          // word wd >> 1, residuals from bit wd of the D3 / D4 word
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int r = g + 8 * half;
            const uint2 q2 = lds64(fb + r * 32 + c * 8);
            const uint32_t d3 = be.bits >= 3 ? lds32(fb + 512 + r * 16 + c * 4) : 0u;
            const uint32_t d4 = be.bits >= 4 ? lds32(fb + 768 + r * 16 + c * 4) : 0u;
            uint32_t* cw = half ? cb : ca;
            const uint32_t qw[2] = {q2.x, q2.y};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              uint32_t v = (qw[wd >> 1] << (2 - 2 * (wd & 1))) & 0xCCCCCCCCu;
              const int sh = 1 - wd;
              v = and_or(sh >= 0 ? d3 << sh : d3 >> -sh, 0x22222222u, v);
              v = and_or(d4 >> wd, 0x11111111u, v);
              cw[wd] = v;
            }
          }
        }
        // two accumulation chains per token block (even and odd MMAs of the
        // stage), so that consecutive MMAs do not wait for each other; the
        // first MMA of each chain starts from zero
        float dsum[NB][2][4];
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          uint32_t pa[4], pb[4];
          pairs(ca[wd], za_lo, za_hi, pa);
          pairs(cb[wd], zb_lo, zb_hi, pb);
          if (G64) {  // groups of 64: the scale goes into A (one fp16 rounding)
            const __half2 sa = __half2half2(__float2half_rn(slo)), sb2 = __half2half2(__float2half_rn(shi));
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              pa[jj] = h2u(__hmul2(u2h(pa[jj]), sa));
              pb[jj] = h2u(__hmul2(u2h(pb[jj]), sb2));
            }
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              const uint4 x = xv[nb][wd];
              uint32_t b0, b1;
              if (PLANES) {
                b0 = hh ? x.z : x.x;
                b1 = hh ? x.w : x.y;
              } else {  // (x_j, x_j+4) pairs
                b0 = hh ? __byte_perm(x.y, x.w, 0x5410) : __byte_perm(x.x, x.z, 0x5410);
                b1 = hh ? __byte_perm(x.y, x.w, 0x7632) : __byte_perm(x.x, x.z, 0x7632);
              }
              if (G64)
                mma16816(acc[f][nb], pa[2 * hh], pb[2 * hh], pa[2 * hh + 1], pb[2 * hh + 1], b0, b1);
              else if (wd == 0)
                mma16816_first(dsum[nb][hh], pa[2 * hh], pb[2 * hh], pa[2 * hh + 1], pb[2 * hh + 1], b0, b1);
              else
                mma16816(dsum[nb][hh], pa[2 * hh], pb[2 * hh], pa[2 * hh + 1], pb[2 * hh + 1], b0, b1);
            }
          }
        }
        if (!G64) {
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            acc[f][nb][0] = fmaf(slo, dsum[nb][0][0] + dsum[nb][1][0], acc[f][nb][0]);
            acc[f][nb][1] = fmaf(slo, dsum[nb][0][1] + dsum[nb][1][1], acc[f][nb][1]);
            acc[f][nb][2] = fmaf(shi, dsum[nb][0][2] + dsum[nb][1][2], acc[f][nb][2]);
            acc[f][nb][3] = fmaf(shi, dsum[nb][0][3] + dsum[nb][1][3], acc[f][nb][3]);
          }
        }
      }
      __syncwarp();  // every lane is done with ring slot j % kRing
      issue(j + kRing);
    }
    // the unit's partial sums of all warps, added in warp order
#pragma unroll
    for (int f = 0; f < FW; ++f)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) red[(warp * kVals + (f * NB + nb) * 4 + jj) * 32 + lane] = acc[f][nb][jj];
    __syncthreads();
    for (int v = threadIdx.x; v < 32 * NB * 4; v += kWarps * 32) {
      const int ln = v & 31, nb = (v >> 5) / 4, jj = (v >> 5) & 3;
      const int gg = ln >> 2, cc = ln & 3;
      const int row = gg + 8 * (jj >> 1);               // weight row inside the fragment
      const int tk = t0 + 8 * nb + 2 * cc + (jj & 1);   // token row inside the bin
      float sum[FW];
#pragma unroll
      for (int f = 0; f < FW; ++f) {
        float a = 0.0f;
        for (int w = 0; w < kWarps; ++w) a += red[(w * kVals + (f * NB + nb) * 4 + jj) * 32 + ln];
        sum[f] = a;
      }
      if (tk < be.nrows) {
        const size_t p = static_cast<size_t>(be.row0 + tk);
        if (GU) {
          P.out[p * P.N + n0 + row] = __float2half_rn(silu_f(sum[0]) * sum[1]);
        } else {
#pragma unroll
          for (int f = 0; f < FW; ++f) {
            if (!(fabsf(sum[f]) <= 65504.0f)) flag_status(P.status, MOE_DEV_RANGE);
            P.out[p * P.N + n0 + 16 * f + row] = __float2half_rn(sum[f]);
          }
        }
      }
    }
    __syncthreads();  // the reduction buffer is reused by the next unit
  }
  cp_async_wait<0>();  // only empty groups remain
}

// CTAs of a k_dec variant resident on the device at once (found once per device).
template <bool GU, bool PLANES, bool G64, int FW, int NB, int W>
int resident_ctas(const char* what, moe_status_t* st) {
  auto kern = k_dec<GU, PLANES, G64, FW, NB, W>;
  // the dynamic shared memory depends on max_ent: set the opt-in to the
  // largest this variant can need (768 bins), once per device
  static std::atomic<uint64_t> attr_set{0};
  static int resident[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) { *st = cuda_check(e, what); return 0; }
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Smem<FW, NB, W>::bytes(768)));
    if (e != cudaSuccess) { *st = cuda_check(e, what); return 0; }
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, W * 32, Smem<FW, NB, W>::bytes(256));
    if (e != cudaSuccess) { *st = cuda_check(e, what); return 0; }
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) { *st = cuda_check(e, what); return 0; }
    if (dev < 64) resident[dev] = std::max(1, per_sm) * std::max(1, sms);
    attr_set.fetch_or(bit);
  }
  *st = MOE_OK;
  return dev < 64 && resident[dev] > 0 ? resident[dev] : 148;
}

// The grid is the number of CTAs that fit at once (persistent), or fewer
// when there are fewer units.
template <bool GU, bool PLANES, bool G64, int FW, int NB, int W>
moe_status_t run_dec(const DecParams& p, int units_upper, int fit, cudaStream_t s, const char* what) {
  const int grid = std::max(1, std::min(units_upper, fit));
  return cuda_check(launch_pdl(true, k_dec<GU, PLANES, G64, FW, NB, W>, dim3(grid), dim3(W * 32),
                               Smem<FW, NB, W>::bytes(p.max_ent), s, p),
                    what);
}

// Warps per CTA: a unit's K stages are split over the CTA's warps, and the
// units over the resident CTAs; the time is about (rounds of units) x
// (stages of the busiest warp).  With one token block both 8 warps (three
// CTAs per SM) and 12 (two) are built, and the cheaper is taken: 12 where
// the units come to just over a whole number of rounds of 8-warp CTAs and
// rows are long (the Mixtral-shaped down GEMM: 512 units of 112 stages on
// 444 or 296 CTAs, 2 x 14 against 2 x 10).
template <bool GU, bool PLANES, bool G64, int FW>
moe_status_t run_nb(const DecParams& p, int nb, int units_upper, cudaStream_t s, const char* what) {
  moe_status_t st = MOE_OK;
  if (nb != 1) {
    const int fit = resident_ctas<GU, PLANES, G64, FW, 2, 8>(what, &st);
    if (st != MOE_OK) return st;
    return run_dec<GU, PLANES, G64, FW, 2, 8>(p, units_upper, fit, s, what);
  }
  const int fit8 = resident_ctas<GU, PLANES, G64, FW, 1, 8>(what, &st);
  if (st != MOE_OK) return st;
  const int fit12 = resident_ctas<GU, PLANES, G64, FW, 1, 12>(what, &st);
  if (st != MOE_OK) return st;
  const int n_st = p.K / kStageK;
  const long cost8 = static_cast<long>(ceil_div(units_upper, fit8)) * ceil_div(n_st, 8);
  const long cost12 = static_cast<long>(ceil_div(units_upper, fit12)) * ceil_div(n_st, 12);
  return cost12 < cost8 ? run_dec<GU, PLANES, G64, FW, 1, 12>(p, units_upper, fit12, s, what)
                        : run_dec<GU, PLANES, G64, FW, 1, 8>(p, units_upper, fit8, s, what);
}

// units_upper: an upper bound of the work units (listed bins x passes x row
// blocks), which sizes the grid when there are fewer units than CTA slots
template <bool PLANES, bool G64>
moe_status_t run_pair(DecParams gu, DecParams dn, int max_bins, int passes, int nb, int sms, cudaStream_t s) {
  gu.row_blocks = gu.N / 16;
  moe_status_t st = run_nb<true, PLANES, G64, 2>(gu, nb, max_bins * passes * gu.row_blocks, s,
                                                 "ffn decode gate/up launch");
  if (st != MOE_OK) return st;
  // 32-row units unless that leaves fewer than two units per SM
  const bool wide = static_cast<long>(max_bins) * (dn.N / 32) >= 2L * sms && dn.N % 32 == 0;
  dn.row_blocks = dn.N / (wide ? 32 : 16);
  const int units = max_bins * passes * dn.row_blocks;
  return wide ? run_nb<false, PLANES, G64, 2>(dn, nb, units, s, "ffn decode down launch")
              : run_nb<false, PLANES, G64, 1>(dn, nb, units, s, "ffn decode down launch");
}

int sm_count_dec() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev].load() > 0) return cached[dev].load();
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cached[dev].store(n);
  return n;
}

}  // namespace

moe_status_t launch_ffn_decode(const FfnArgs& a, int token_blocks, cudaStream_t s) {
  const bool planes = a.layout == MOE_LAYOUT_PLANES;
  const int mult = planes ? 3 : 1;
  DecParams gu{};
  gu.act = a.x_perm;
  gu.offsets = a.offsets;
  gu.blobs = a.blobs;
  gu.slot_of = a.slot_of;
  gu.blob_bytes = a.blob_bytes;
  gu.K = a.d;
  gu.N = a.F;
  gu.nbins = a.E * mult;
  gu.planes_mult = mult;
  gu.rows = a.total_rows;
  gu.group = a.group;
  gu.out = a.h;
  gu.status = a.status;
  for (int m = 0; m < 2; ++m) {
    gu.code_off[m] = planes ? a.lay.q2[m] : a.lay.codes[m];
    gu.d3_off[m] = a.lay.d3[m];
    gu.d4_off[m] = a.lay.d4[m];
    gu.sz_off[m] = a.lay.sz[m];
  }
  if (planes && a.lay.d4[1] - a.lay.d4[0] != a.lay.d3[1] - a.lay.d3[0]) {  // one stride for D3 and D4 pieces
    set_error("ffn decode: gate-to-up offsets of D3 and D4 differ");
    return MOE_ERR_INVALID_ARG;
  }
  const int max_bins = std::min(gu.nbins, a.total_rows);
  if (max_bins == 0) return MOE_OK;
  gu.max_ent = max_bins;  // no more bins than rows are non-empty
  DecParams dn = gu;
  dn.act = a.h;
  dn.K = a.F;
  dn.N = a.d;
  dn.out = a.y_perm;
  dn.code_off[0] = planes ? a.lay.q2[2] : a.lay.codes[2];
  dn.d3_off[0] = a.lay.d3[2];
  dn.d4_off[0] = a.lay.d4[2];
  dn.sz_off[0] = a.lay.sz[2];
  const int nb = token_blocks <= 1 ? 1 : 2;
  // passes per bin: a bin never holds more than T rows
  const int passes = std::max(1, (std::min(a.T, a.total_rows) + 8 * nb - 1) / (8 * nb));
  const int sms = sm_count_dec();
  const bool g64 = a.group == 64;
  if (planes)
    return g64 ? run_pair<true, true>(gu, dn, max_bins, passes, nb, sms, s)
               : run_pair<true, false>(gu, dn, max_bins, passes, nb, sms, s);
  return g64 ? run_pair<false, true>(gu, dn, max_bins, passes, nb, sms, s)
             : run_pair<false, false>(gu, dn, max_bins, passes, nb, sms, s);
}

}  // namespace moeq
