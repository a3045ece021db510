// Prefill-regime grouped expert FFN on the 5th-generation tensor cores.
//
// One persistent CTA per SM walks a tile list built on the device from the
// bin offsets (no host sync).  A tile is (bin, token block of up to 128
// rows, weight block).  The MMA is issued "swap-AB": dequantised weight
// rows are the M side (operand A) and the bin's tokens the N side (operand
// B, fp16 activation rows loaded by TMA), so a bin of any size is covered
// with at most 15 padded token columns; D[weight row][token] accumulates in
// TMEM (fp32).
//
// Operand A lives in tensor memory, not shared memory: a dequantiser thread
// owns one weight row, which is one TMEM lane, and stores its fp16 values
// there with tcgen05.st (two per 32-bit column, K ascending).  The MMA
// reads A from TMEM and only B from shared memory.  At N = 128 a 128-row
// MMA that took both operands from shared memory would already use the
// whole shared-memory bandwidth of the SM (A + B slices every 64 cycles),
// and building A there as well (dequantiser stores) would double that.
//
// Each k-block issues two M=128 MMAs that share one B tile: the gate and
// up rows of the same 128 features (first GEMM), or two adjacent 128-row
// blocks of W_down (second GEMM).  Sharing B halves the activation bytes
// per MAC, and in the first GEMM lane i of both accumulators belongs to
// feature i, so the SwiGLU epilogue needs no exchange.  The MMA warp issues
// the eight MMAs of a k-block back to back from fixed descriptor bases plus
// constant offsets: address arithmetic between tcgen05.mma instructions
// (descriptors rebuilt per MMA) was measured to cost 3-6x the MMA time.
//
// TMEM (512 columns) holds the two accumulators (2 x 128 columns) and four
// A stages (4 x 2 matrices x 32 columns), so there is one accumulator
// buffer.  To keep the MMA waiting as little as possible for the
// epilogue, the epilogue only moves the accumulators through registers
// into a shared-memory staging buffer (h and y_perm as fp16, both
// double-buffered), releases them, and then writes the staged rows out with
// 16-byte stores while the next tile's MMAs run.
//
// Warp roles (16 warps):
//   warp 0      codes producer: packed codes (5-D tensor maps over the
//               blob pool's 16-row x 128-K code tiles, one box of 128 rows
//               per 128 K per matrix) and their scale/zero words (1-D bulk
//               copies)
//   warp 3      activation producer: one 128-row TMA box (128B swizzle)
//               per 64 K of the tile's fp16 activation rows
//   warp 1      MMA issuer: the whole warp waits, one elected lane issues
//               tcgen05.mma (M=128, N=tokens, K=16) and tcgen05.commit
//   warp 2      TMEM allocator
//   warps 4-7   dequantisers of matrix 0, warps 8-11 of matrix 1: thread i
//               turns weight row i of a staged codes block into fp16
//               ((code - zero) * scale, one rounding) and stores it to TMEM
//               lane i (the warp's lane quadrant is warp % 4)
//   warps 12-15 epilogue: tcgen05.ld of its TMEM lane quadrant; gate/up
//               pass stages h = silu(gate) * up (fp16), down pass y_perm
//               (fp16); then the four warps copy the staged rows out
// Pipelines: codes (3 / 2 stages of 128 K) -> dequant -> A in TMEM (4
// stages of 64 K); activations B (6 / 3 stages of 64 K, first / second
// GEMM); both -> MMA -> accumulators -> epilogue staging -> global.  Every
// wait is bounded; on a timeout the CTA raises MOE_DEV_TIMEOUT, drains its
// copies and MMAs, frees TMEM and returns.  Warps reconverge after every
// wait, before any warp-aligned instruction.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace moeq {
namespace {

// ------------------------------------------------------------ PTX utils --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try, but lets the hardware suspend the thread for up to
// `hint_ns` while the phase is incomplete (it resumes as soon as the phase
// completes), so waiting warps do not spin on the issue slots that the
// working warps of the same SM sub-partition need.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: only reached when something is broken

// Bounded wait.  Returns false when the CTA is aborting (flag set here on
// timeout, or by another role).
// Where the first timeout of a CTA happened (test hook, see trace_put).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, int* trace = nullptr, uint32_t bar0 = 0,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_sleep(bar, parity, 20000u)) return true;
    if ((i & 7) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        flag_status(status, MOE_DEV_TIMEOUT);
        if (trace) {  // slot 8: barrier index and parity of the wait that gave up
          reinterpret_cast<volatile int*>(trace)[blockIdx.x * 16 + 8] =
              (0x7F << 24) | (static_cast<int>((bar - bar0) / 8) << 4) | static_cast<int>(parity);
          __threadfence_system();
        }
        return false;
      }
    }
  }
}

// Bounded wait by a whole warp: every lane observes the barrier, then the
// warp reconverges and agrees on the outcome, so the warp-aligned
// instructions that follow (tcgen05.ld, barriers) run converged.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, int* trace = nullptr, uint32_t bar0 = 0,
                                          uint64_t limit_ns = kWaitLimitNs) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status, trace, bar0, limit_ns);
  __syncwarp();
  return __all_sync(0xffffffffu, ok);
}

// Optional progress record (a test hook): slot `role` of this CTA holds
// (site << 24) | (tile & 0xfff) << 12 | (kb & 0xfff), written through to
// host-visible memory so that a stalled launch can be inspected.
__device__ __forceinline__ void trace_put(int* trace, int role, int site, int tile, int kb) {
  if (trace) {
    reinterpret_cast<volatile int*>(trace)[blockIdx.x * 16 + role] =
        (site << 24) | ((tile & 0xfff) << 12) | (kb & 0xfff);
    __threadfence_system();
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// UMMA shared-memory descriptor: K-major, 128B swizzle, 8-row atoms 1024 B
// apart (SBO), version 1.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 D,
// M = 128, N = n.
__device__ __forceinline__ uint32_t umma_idesc_f16(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}


// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}



__device__ __forceinline__ void umma_commit_elect(uint32_t bar) {
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void umma_f16_ts_elect(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------ config ----

constexpr int kThreads = 512;  // 16 warps
constexpr int kMaxBins = 768;
constexpr int kNT = 128;       // largest token block (MMA N)

// The epilogue stages a tile's outputs in shared memory (h fp16, 32 KB; y
// fp16, 64 KB; both double-buffered), releases the accumulators, and then
// writes them out with 16-byte stores while the next tile's MMAs run.
template <bool GATEUP>
struct Cfg {
  static constexpr int AK = 64;       // K of one A stage (TMEM)
  static constexpr int SA = 4;        // A stages
  static constexpr int ACC = 1;       // accumulator buffers (each: 2 matrices x kNT columns)
  static constexpr int SB = GATEUP ? 6 : 3;        // B (activation) stages of 64 K
  static constexpr int CSTAGES = GATEUP ? 3 : 2;   // codes stages of 128 K
  static constexpr int OUT_BYTES = GATEUP ? kNT * 128 * 2 : kNT * 256 * 2;  // one staging buffer
  static constexpr int OUT_BUFS = 2;
  static constexpr int B_BYTES = kNT * 128;     // 128 token rows x 64 fp16
  static constexpr int C_BYTES = 8192;          // per matrix: 128 rows x 128 K of codes
  static constexpr int SZ_BYTES = 1024;         // per matrix: 128 rows x up to 2 groups x 4 B
  static constexpr int OFF_B = 0;
  static constexpr int OFF_C = OFF_B + SB * B_BYTES;
  static constexpr int OFF_SZ = OFF_C + CSTAGES * 2 * C_BYTES;
  static constexpr int OFF_OUT = OFF_SZ + CSTAGES * 2 * SZ_BYTES;
  static constexpr int OFF_TILE = OFF_OUT + OUT_BUFS * OUT_BYTES;  // int tile_start[769], off[769]
  static constexpr int OFF_BAR = OFF_TILE + 2 * (kMaxBins + 1) * 4 + 8;
  static constexpr int N_BARS = 2 * CSTAGES + 2 * SA + 2 * SB + 2 * ACC + 1 + 1 + 1;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem base, abort flag
  static constexpr int SMEM = OFF_MISC + 16 + 1024;      // + alignment slack
  static constexpr int A_COLS = AK / 2;                  // TMEM columns of one matrix's A stage
  static constexpr int ACOL = ACC * 2 * kNT;             // first A column
  static constexpr int TMEM_COLS = 512;
};
static_assert(Cfg<true>::SMEM <= 232448 && Cfg<false>::SMEM <= 232448, "shared memory budget");
static_assert(Cfg<true>::ACOL + Cfg<true>::SA * 2 * Cfg<true>::A_COLS <= Cfg<true>::TMEM_COLS, "TMEM budget");
static_assert(Cfg<true>::AK == 64, "one A stage per B stage of 64 K");

struct TcParams {
  CUtensorMap act;       // fp16 [rows][K], box 64 x 16, 128B swizzle
  CUtensorMap codes[2];  // INT4: u32 [nblob][N][K/8];   PLANES: Q2 u32 [nblob][N][K/16]
  CUtensorMap d3[2];     // PLANES only: u32 [nblob][N][K/32]
  CUtensorMap d4[2];
  const int32_t* offsets;
  const int32_t* slot_of;
  const uint8_t* blobs;
  size_t blob_bytes;
  size_t sz_off[2];
  int K, N, nbins, planes_mult, group;
  int rows;  // activation rows (= total_rows): every bin range is clamped into [0, rows]
  __half* h_out;
  __half* y_out;
  int32_t* status;
  int* trace;  // optional progress record (null in normal use)
  uint64_t wait_ns;  // limit of every wait (2 s; shorter under the timeout test hook)
  int debug_stall;   // test hook: CTA 0's epilogue withholds its first accumulator release
};

struct Tile {
  int bin, slot, bits, row0, nrows, nt, mb;
};

__device__ __forceinline__ Tile decode_tile(int t, const int* tile_start, const int* off, int nbins,
                                            int MB, int planes_mult, const int32_t* slot_of) {
  int lo = 0, hi = nbins;  // largest b with tile_start[b] <= t (tile_start[nbins] = total)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid;
  }
  Tile T;
  T.bin = lo;
  const int local = t - tile_start[lo];
  const int tb = local / MB;
  T.mb = local - tb * MB;
  const int n = max(0, off[lo + 1] - off[lo]);
  const int nb = (n + kNT - 1) / kNT;
  const int per = (((n + nb - 1) / nb) + 15) & ~15;
  T.row0 = off[lo] + tb * per;
  T.nrows = min(per, n - tb * per);
  T.nt = (T.nrows + 15) & ~15;
  const int e = lo / planes_mult;
  T.slot = slot_of ? slot_of[e] : e;
  T.bits = planes_mult == 3 ? 2 + lo % 3 : 4;
  return T;
}

// (a & m) | c in one instruction.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t c) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(m), "r"(c));
  return r;
}

// Eight 4-bit codes (nibble i = element i) -> (code - z) * s as fp16,
// elements in order.  Byte j holds the pair (e_2j, e_2j+1); replicated
// into both halves and masked, it reads as the half2 (1024 + e_2j,
// 64 + e_2j+1) (the high nibble lands at mantissa bits 4..7, whose unit at
// exponent 64 is 1/16).  Subtracting (1024 + z, 64 + z) is exact, and one
// multiply by s rounds each product once.
__device__ __forceinline__ uint4 dequant8(uint32_t w, __half2 zoff, __half2 s2) {
  uint32_t v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t rep = __byte_perm(w, 0u, 0x1111u * j);
    uint32_t raw;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(raw) : "r"(rep), "r"(0x00F0000Fu), "r"(0x54006400u));
    __half2 h = *reinterpret_cast<const __half2*>(&raw);
    h = __hmul2(__hsub2(h, zoff), s2);
    v[j] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(v[0], v[1], v[2], v[3]);
}

// Eight 4-bit codes in plane order (element 2j in nibble j, element 2j+1
// in nibble 4+j) -> (code - z) * s as fp16, elements in order.  Masking
// nibbles (j, 4+j) into 0x6400 gives the half2 (1024 + e_2j, 1024 + e_2j+1);
// nibbles at bits 4..7 of each half, masked into 0x5400, read as (64 + e,
// 64 + e) (their unit at exponent 64 is 1/16).  Subtracting (1024 + z) or
// (64 + z) is exact; one multiply by s rounds each product once.
__device__ __forceinline__ uint4 dequant8_planes(uint32_t w, __half2 z_lo, __half2 z_hi, __half2 s2) {
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

// GATEUP: matrix 0 = gate rows, matrix 1 = up rows of features
// [128 mb, 128 mb + 128).  DOWN: matrix 0 = W_down rows [256 mb, +128),
// matrix 1 = rows [256 mb + 128, +128) when they exist (d % 256 may be 128).
template <bool GATEUP, bool PLANES>
__global__ void __launch_bounds__(kThreads, 1) k_ffn_tc(const __grid_constant__ TcParams P) {
  using C = Cfg<GATEUP>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int* tile_start = reinterpret_cast<int*>(smem + C::OFF_TILE);
  int* off_s = tile_start + (kMaxBins + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t bar0 = smem_u32(bars);
  auto codes_full = [&](int i) { return bar0 + 8u * i; };
  auto codes_empty = [&](int i) { return bar0 + 8u * (C::CSTAGES + i); };
  constexpr int kA = 2 * C::CSTAGES, kB = kA + 2 * C::SA, kR = kB + 2 * C::SB, kE = kR + 2 * C::ACC;
  auto a_full = [&](int i) { return bar0 + 8u * (kA + i); };
  auto a_empty = [&](int i) { return bar0 + 8u * (kA + C::SA + i); };
  auto b_full = [&](int i) { return bar0 + 8u * (kB + i); };
  auto b_empty = [&](int i) { return bar0 + 8u * (kB + C::SB + i); };
  auto acc_full = [&](int i) { return bar0 + 8u * (kR + i); };
  auto acc_empty = [&](int i) { return bar0 + 8u * (kR + C::ACC + i); };
  const uint32_t drain_bar = bar0 + 8u * kE;
  const uint32_t exit_bar = bar0 + 8u * (kE + 1);
  const uint32_t epi_bar = bar0 + 8u * (kE + 2);  // the 4 epilogue warps, once per tile
  int* trace = P.trace ? P.trace + (GATEUP ? 0 : gridDim.x * 16) : nullptr;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbins = P.nbins;
  const int rows_per_block = GATEUP ? 128 : 256;      // weight rows of one matrix pair
  const int MB = (P.N + rows_per_block - 1) / rows_per_block;
  const int KC = P.K / 128;
  auto has_m1 = [&](int mb) { return GATEUP || mb * 256 + 128 < P.N; };
  auto row_base = [&](int mb, int m) { return GATEUP ? mb * 128 : mb * 256 + 128 * m; };

  // ---- set-up: barriers, TMEM, tile table --------------------------------
  if (tid == 0) {
    for (int i = 0; i < C::CSTAGES; ++i) {
      mbar_init(codes_full(i), 1);
      mbar_init(codes_empty(i), 8);
    }
    for (int i = 0; i < C::SA; ++i) {
      mbar_init(a_full(i), 8);
      mbar_init(a_empty(i), 1);
    }
    for (int i = 0; i < C::SB; ++i) {
      mbar_init(b_full(i), 1);
      mbar_init(b_empty(i), 1);
    }
    for (int i = 0; i < C::ACC; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 4);
    }
    mbar_init(drain_bar, 1);
    mbar_init(exit_bar, kThreads / 32);
    mbar_init(epi_bar, 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // barrier set-up and the TMEM allocation may overlap the previous kernel;
  // everything below reads what earlier kernels wrote
  pdl_wait();
  pdl_trigger();
  // offsets come from the caller: clamp them into [0, rows] so that no
  // inconsistent table (e.g. one built for another bin layout) can send a
  // tile outside the activation rows; such a table is flagged
  for (int b = tid; b <= nbins; b += kThreads) {
    const int v = P.offsets[b];
    const int c = min(max(v, 0), P.rows);
    if (c != v || (b == nbins && v != P.rows)) flag_status(P.status, MOE_DEV_BAD_INDEX);
    off_s[b] = c;
  }
  __syncwarp();
  __syncthreads();
  if (warp == 0) {
    // tiles per bin -> exclusive scan (lane owns a contiguous run of bins)
    const int per_lane = (nbins + 31) / 32;
    const int b0 = lane * per_lane;
    int run = 0;
    for (int i = 0; i < per_lane; ++i) {
      const int b = b0 + i;
      if (b < nbins) {
        int n = max(0, off_s[b + 1] - off_s[b]);
        if (P.slot_of && P.slot_of[b / P.planes_mult] < 0) n = 0;
        const int tiles = ((n + kNT - 1) / kNT) * MB;
        tile_start[b] = run;
        run += tiles;
      }
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int base = incl - run;
    for (int i = 0; i < per_lane; ++i) {
      const int b = b0 + i;
      if (b < nbins) tile_start[b] += base;
    }
    if (lane == 31) tile_start[nbins] = incl;
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = tile_start[nbins];

  // ---- producers: codes (warp 0) and activations (warp 3) ----------------
  if (warp == 0 || warp == 3) {
    if (lane == 0) {
      const bool codes_role = warp == 0;
      int cs = 0, cph = 0, s = 0, sph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile(t, tile_start, off_s, nbins, MB, P.planes_mult, P.slot_of);
        if (codes_role) {
          const uint8_t* blob = P.blobs + static_cast<size_t>(T.slot) * P.blob_bytes;
          const int gpc = 128 / P.group;  // groups per codes stage
          const int G = P.K / P.group;
          const int nm = has_m1(T.mb) ? 2 : 1;
          uint32_t code_bytes = 8192;
          if (PLANES) code_bytes = 4096 + (T.bits >= 3 ? 2048 : 0) + (T.bits >= 4 ? 2048 : 0);
          for (int kc = 0; kc < KC && ok; ++kc) {
            trace_put(trace, 0, 1, t, kc);
            ok = mbar_wait(codes_empty(cs), cph ^ 1, abort_flag, P.status, trace, bar0, P.wait_ns);
            if (!ok) break;
            mbar_expect_tx(codes_full(cs), nm * (code_bytes + gpc * 512));
            for (int m = 0; m < nm; ++m) {
              const int r0 = row_base(T.mb, m);
              const uint32_t cdst = smem_u32(smem + C::OFF_C + (cs * 2 + m) * C::C_BYTES);
              const CUtensorMap* cm = &P.codes[GATEUP ? m : 0];
              // the blob's code tiles (16 rows x 128 K): row blocks r0/16 .. + 7 of K stage kc
              tma_load_5d(cdst, cm, 0, 0, kc, r0 >> 4, T.slot, codes_full(cs));
              if (PLANES && T.bits >= 3)
                tma_load_5d(cdst + 4096, &P.d3[GATEUP ? m : 0], 0, 0, kc, r0 >> 4, T.slot, codes_full(cs));
              if (PLANES && T.bits >= 4)
                tma_load_5d(cdst + 6144, &P.d4[GATEUP ? m : 0], 0, 0, kc, r0 >> 4, T.slot, codes_full(cs));
              const uint8_t* src = blob + P.sz_off[GATEUP ? m : 0] +
                                   (static_cast<size_t>(r0 >> 7) * G + kc * gpc) * 512;
              bulk_load(smem_u32(smem + C::OFF_SZ + (cs * 2 + m) * C::SZ_BYTES), src, gpc * 512,
                        codes_full(cs));
            }
            if (++cs == C::CSTAGES) { cs = 0; cph ^= 1; }
          }
        } else {
          for (int kb = 0; kb < 2 * KC && ok; ++kb) {
            trace_put(trace, 2, 2, t, kb);
            ok = mbar_wait(b_empty(s), sph ^ 1, abort_flag, P.status, trace, bar0, P.wait_ns);
            if (!ok) break;
            // one 128-row box: rows past this tile's are loaded but not read
            // by the MMA (N = nt); rows past the tensor are zero-filled
            mbar_expect_tx(b_full(s), C::B_BYTES);
            tma_load_2d(smem_u32(smem + C::OFF_B + s * C::B_BYTES), &P.act, kb * 64, T.row0, b_full(s));
            if (++s == C::SB) { s = 0; sph ^= 1; }
          }
        }
      }
      trace_put(trace, codes_role ? 0 : 2, ok ? 12 : 13, 0, 0);
      if (!ok) {
        // drain: the most recent arming of every stage must land before exit
        const uint64_t t0 = global_ns();
        if (codes_role) {
          for (int idx = 0; idx < C::CSTAGES; ++idx) {
            const int ph = (idx < cs) ? cph : cph ^ 1;
            while (!mbar_try(codes_full(idx), ph) && global_ns() - t0 < P.wait_ns) {}
          }
        } else {
          for (int idx = 0; idx < C::SB; ++idx) {
            const int ph = (idx < s) ? sph : sph ^ 1;
            while (!mbar_try(b_full(idx), ph) && global_ns() - t0 < P.wait_ns) {}
          }
        }
      }
    }
  }
  // ---- MMA issuer --------------------------------------------------------
  else if (warp == 1) {
    {
      int sa = 0, saph = 0, sb = 0, sbph = 0, acc = 0, aph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile(t, tile_start, off_s, nbins, MB, P.planes_mult, P.slot_of);
        const uint32_t idesc = umma_idesc_f16(T.nt);
        const int nm = has_m1(T.mb) ? 2 : 1;
        if (lane == 0) trace_put(trace, 1, 3, t, 0);
        ok = warp_wait(acc_empty(acc), aph ^ 1, abort_flag, P.status, trace, bar0, P.wait_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t dcol = tmem_base + acc * (2 * kNT);
        // operand addresses: fixed bases plus stage offsets, so that the
        // MMAs of a k-block issue back to back
        const uint64_t bdesc0 = umma_desc_sw128(smem_u32(smem + C::OFF_B));
        const uint32_t acol0 = tmem_base + C::ACOL;
        for (int kb = 0; kb < 2 * KC && ok; ++kb) {
          ok = warp_wait(a_full(sa), saph, abort_flag, P.status, trace, bar0, P.wait_ns);
          if (!ok) break;
          ok = warp_wait(b_full(sb), sbph, abort_flag, P.status, trace, bar0, P.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(sb * (C::B_BYTES >> 4));
          const uint32_t acol = acol0 + sa * (2 * C::A_COLS);
          const uint32_t first = kb != 0;
          umma_f16_ts_elect(dcol, acol, bdesc, idesc, first);
          umma_f16_ts_elect(dcol, acol + 8, bdesc + 2, idesc, 1u);
          umma_f16_ts_elect(dcol, acol + 16, bdesc + 4, idesc, 1u);
          umma_f16_ts_elect(dcol, acol + 24, bdesc + 6, idesc, 1u);
          if (nm == 2) {
            umma_f16_ts_elect(dcol + kNT, acol + C::A_COLS, bdesc, idesc, first);
            umma_f16_ts_elect(dcol + kNT, acol + C::A_COLS + 8, bdesc + 2, idesc, 1u);
            umma_f16_ts_elect(dcol + kNT, acol + C::A_COLS + 16, bdesc + 4, idesc, 1u);
            umma_f16_ts_elect(dcol + kNT, acol + C::A_COLS + 24, bdesc + 6, idesc, 1u);
          }
          umma_commit_elect(a_empty(sa));
          umma_commit_elect(b_empty(sb));
          if (++sa == C::SA) { sa = 0; saph ^= 1; }
          if (++sb == C::SB) { sb = 0; sbph ^= 1; }
        }
        if (!ok) break;
        umma_commit_elect(acc_full(acc));
        if (++acc == C::ACC) { acc = 0; aph ^= 1; }
      }
      if (lane == 0) trace_put(trace, 1, ok ? 12 : 13, 0, 0);
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit_elect(drain_bar);
      const uint64_t t0 = global_ns();
      while (!mbar_try(drain_bar, 0) && global_ns() - t0 < P.wait_ns) {}
      __syncwarp();
    }
  }
  // ---- dequantisers: warps 4-7 matrix 0, warps 8-11 matrix 1 -------------
  else if (warp >= 4 && warp < 12) {
    const int m = (warp - 4) >> 2;
    const int i = tid - 128 - 128 * m;   // weight row inside the 128-row block = TMEM lane
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    int cs = 0, cph = 0, s = 0, sph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const Tile T = decode_tile(t, tile_start, off_s, nbins, MB, P.planes_mult, P.slot_of);
      const bool live = m == 0 || has_m1(T.mb);  // matrix 1 may be absent in the last W_down block
      for (int kc = 0; kc < KC && ok; ++kc) {
        if (lane == 0) trace_put(trace, 3 + m, 6, t, kc);
        ok = warp_wait(codes_full(cs), cph, abort_flag, P.status, trace, bar0, P.wait_ns);
        if (!ok) break;
        const uint8_t* cb = smem + C::OFF_C + (cs * 2 + m) * C::C_BYTES;
        uint32_t w[16];
        if (!PLANES) {
          // row i: 64 B, 64B swizzle (chunk j at j ^ ((i >> 1) & 3))
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(cb + i * 64 + ((j ^ ((i >> 1) & 3)) << 4));
            w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
          }
        } else {
          // Q2 row i: 32 B, 32B swizzle (chunk j at j ^ ((i >> 2) & 1)); D3, D4 rows 16 B
          uint32_t qw[8];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(cb + i * 32 + ((j ^ ((i >> 2) & 1)) << 4));
            qw[4 * j] = v.x; qw[4 * j + 1] = v.y; qw[4 * j + 2] = v.z; qw[4 * j + 3] = v.w;
          }
          uint4 r3 = make_uint4(0, 0, 0, 0), r4 = make_uint4(0, 0, 0, 0);
          if (T.bits >= 3) r3 = *reinterpret_cast<const uint4*>(cb + 4096 + i * 16);
          if (T.bits >= 4) r4 = *reinterpret_cast<const uint4*>(cb + 6144 + i * 16);
          const uint32_t d3w[4] = {r3.x, r3.y, r3.z, r3.w};
          const uint32_t d4w[4] = {r4.x, r4.y, r4.z, r4.w};
          // word wd = elements 8wd..8wd+7 as a plane-order code word: the
          // base sits at bits 2wd' (wd' = wd & 1) of each nibble of Q2 word
          // wd >> 1, the residuals at bit wd & 3 of D3/D4 word wd >> 2;
          // residual planes only up to the bin's width (uniform across the
          // warp)
#pragma unroll
          for (int wd = 0; wd < 16; ++wd) w[wd] = (qw[wd >> 1] << (2 - 2 * (wd & 1))) & 0xCCCCCCCCu;
          if (T.bits >= 3) {
#pragma unroll
            for (int wd = 0; wd < 16; ++wd) {
              const int sh = 1 - (wd & 3);
              w[wd] = and_or(sh >= 0 ? d3w[wd >> 2] << sh : d3w[wd >> 2] >> -sh, 0x22222222u, w[wd]);
            }
          }
          if (T.bits >= 4) {
#pragma unroll
            for (int wd = 0; wd < 16; ++wd) w[wd] = and_or(d4w[wd >> 2] >> (wd & 3), 0x11111111u, w[wd]);
          }
        }
        const uint32_t* szb = reinterpret_cast<const uint32_t*>(smem + C::OFF_SZ + (cs * 2 + m) * C::SZ_BYTES);
        const uint32_t sz0 = szb[i];
        const uint32_t sz1 = P.group == 64 ? szb[128 + i] : sz0;
        __syncwarp();
        if (lane == 0) mbar_arrive(codes_empty(cs));
        if (++cs == C::CSTAGES) { cs = 0; cph ^= 1; }
        for (int h = 0; h < 2 && ok; ++h) {
          if (lane == 0) trace_put(trace, 3 + m, 7, t, 2 * kc + h);
          ok = warp_wait(a_empty(s), sph ^ 1, abort_flag, P.status, trace, bar0, P.wait_ns);
          if (!ok) break;
          tc_fence_after();  // the MMAs that read this stage have completed
          if (live) {
            const uint32_t word = h ? sz1 : sz0;
            const __half sc = __float2half_rn(__uint_as_float(word << 16));
            const float zf = __uint_as_float(word & 0xFFFF0000u);
            const __half2 s2 = __half2half2(sc);
            const __half z1024 = __float2half_rn(1024.0f + zf), z64 = __float2half_rn(64.0f + zf);
            uint32_t v[32];  // column c = elements (2c, 2c + 1) of this 64-K slice of row i
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint4 o = PLANES ? dequant8_planes(w[8 * h + j], __half2half2(z1024), __half2half2(z64), s2)
                                     : dequant8(w[8 * h + j], __halves2half2(z1024, z64), s2);
              v[4 * j] = o.x; v[4 * j + 1] = o.y; v[4 * j + 2] = o.z; v[4 * j + 3] = o.w;
            }
            tmem_st32(lane_base + C::ACOL + (s * 2 + m) * C::A_COLS, v);
            tmem_st_wait();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(a_full(s));
          if (++s == C::SA) { s = 0; sph ^= 1; }
        }
      }
    }
  }
  // ---- epilogue: warps 12-15, TMEM lane quadrant = warp % 4 ---------------
  else if (warp >= 12) {
    const int q = warp & 3;
    int acc = 0, aph = 0, ep_tile = 0, ep_ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const Tile T = decode_tile(t, tile_start, off_s, nbins, MB, P.planes_mult, P.slot_of);
      const bool m1 = has_m1(T.mb);
      if (lane == 0) trace_put(trace, 5, 8, t, 0);
      ok = warp_wait(acc_full(acc), aph, abort_flag, P.status, trace, bar0, P.wait_ns);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * (2 * kNT);
      const int r = 32 * q + lane;  // row of the weight block
      // 16-token chunks; the TMEM loads of chunk c + 1 are in flight while
      // chunk c is converted and written to the staging buffer
      uint8_t* stage = smem + C::OFF_OUT + (C::OUT_BUFS == 2 ? (ep_tile & 1) : 0) * C::OUT_BYTES;
      float ymax = 0.0f;  // largest |y_perm| of this tile's rows (fp16 range check)
      auto emit = [&](const uint32_t (&a0)[16], const uint32_t (&a1)[16], int j0) {
        if (GATEUP) {
          // [token pair][128 features] words of fp16 (token 2p, token 2p + 1)
          uint32_t* hs = reinterpret_cast<uint32_t*>(stage);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float g0 = __uint_as_float(a0[j]), u0 = __uint_as_float(a1[j]);
            const float g1 = __uint_as_float(a0[j + 1]), u1 = __uint_as_float(a1[j + 1]);
            const __half2 hv = __floats2half2_rn(__fdividef(g0, 1.0f + __expf(-g0)) * u0,
                                                 __fdividef(g1, 1.0f + __expf(-g1)) * u1);
            hs[((j0 + j) >> 1) * 128 + r] = *reinterpret_cast<const uint32_t*>(&hv);
          }
        } else {
          // [token pair][256 outputs] words of fp16 (token 2p, token 2p + 1)
          uint32_t* ys = reinterpret_cast<uint32_t*>(stage);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const int pr = (j0 + j) >> 1;
            const float y00 = __uint_as_float(a0[j]), y01 = __uint_as_float(a0[j + 1]);
            const float y10 = __uint_as_float(a1[j]), y11 = __uint_as_float(a1[j + 1]);
            // rows past the tile's (padding up to a multiple of 16) do not count;
            // matrix 1 is absent in a last 128-row W_down block
            const float m0 = fmaxf(j0 + j < T.nrows ? fabsf(y00) : 0.0f, j0 + j + 1 < T.nrows ? fabsf(y01) : 0.0f);
            const float m1v = fmaxf(j0 + j < T.nrows ? fabsf(y10) : 0.0f, j0 + j + 1 < T.nrows ? fabsf(y11) : 0.0f);
            ymax = fmaxf(ymax, m1 ? fmaxf(m0, m1v) : m0);
            const __half2 v0 = __floats2half2_rn(y00, y01), v1 = __floats2half2_rn(y10, y11);
            ys[pr * 256 + r] = *reinterpret_cast<const uint32_t*>(&v0);
            ys[pr * 256 + 128 + r] = *reinterpret_cast<const uint32_t*>(&v1);
          }
        }
      };
      uint32_t g0[16], u0[16], g1[16], u1[16];
      tmem_ld16(tbase, g0);
      if (m1) tmem_ld16(tbase + kNT, u0);
      tmem_ld_wait();
      for (int j0 = 0; j0 < T.nrows; j0 += 32) {
        const bool more1 = j0 + 16 < T.nrows;
        if (more1) {
          tmem_ld16(tbase + j0 + 16, g1);
          if (m1) tmem_ld16(tbase + kNT + j0 + 16, u1);
        }
        emit(g0, u0, j0);
        tmem_ld_wait();
        if (more1) {
          const bool more2 = j0 + 32 < T.nrows;
          if (more2) {
            tmem_ld16(tbase + j0 + 32, g0);
            if (m1) tmem_ld16(tbase + kNT + j0 + 32, u0);
          }
          emit(g1, u1, j0 + 16);
          tmem_ld_wait();
        }
      }
      // NaN compares false: flagged too
      if (!GATEUP && !(ymax <= 65504.0f)) flag_status(P.status, MOE_DEV_RANGE);
      // accumulators read: the MMA may start the next tile
      tc_fence_before();
      __syncwarp();
      // (test hook: withheld once, so that the MMA warp's wait for the next
      // tile's accumulators runs out -- the arrive has no copy behind it)
      const bool withhold = GATEUP && P.debug_stall && blockIdx.x == 0 && t == static_cast<int>(blockIdx.x);
      if (lane == 0 && !withhold) mbar_arrive(acc_empty(acc));
      if (++acc == C::ACC) { acc = 0; aph ^= 1; }
      // all four warps have staged their rows
      if (lane == 0) mbar_arrive(epi_bar);
      ok = warp_wait(epi_bar, ep_ph, abort_flag, P.status, trace, bar0, P.wait_ns);
      ep_ph ^= 1;
      if (!ok) break;
      // 16-byte stores of the staged rows (tokens) that belong to this tile
      const int et = tid - 12 * 32;  // 0..127
      // features / outputs 8 col .. 8 col + 7 of a token are the low (even
      // token) or high (odd token) halves of 8 staged words
      auto unpair = [](const uint32_t* wds, int row) {
        const uint4 lo = reinterpret_cast<const uint4*>(wds)[0], hi = reinterpret_cast<const uint4*>(wds)[1];
        const uint32_t sel = (row & 1) ? 0x7632u : 0x5410u;
        return make_uint4(__byte_perm(lo.x, lo.y, sel), __byte_perm(lo.z, lo.w, sel),
                          __byte_perm(hi.x, hi.y, sel), __byte_perm(hi.z, hi.w, sel));
      };
      if (GATEUP) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(stage);
        const size_t f0 = static_cast<size_t>(T.mb) * 128;
        for (int c = et; c < T.nrows * 16; c += 128) {
          const int row = c >> 4, col = c & 15;
          *reinterpret_cast<uint4*>(P.h_out + static_cast<size_t>(T.row0 + row) * P.N + f0 + col * 8) =
              unpair(src + (row >> 1) * 128 + col * 8, row);
        }
      } else {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(stage);
        const int n0 = row_base(T.mb, 0);
        const int per_row = m1 ? 32 : 16;  // 16-byte pieces (8 outputs) of a row's 256 (or 128)
        for (int c = et; c < T.nrows * 32; c += 128) {
          const int row = c >> 5, col = c & 31;
          if (col < per_row)
            *reinterpret_cast<uint4*>(P.y_out + static_cast<size_t>(T.row0 + row) * P.N + n0 + col * 8) =
                unpair(src + (row >> 1) * 256 + col * 8, row);
        }
      }
      if (C::OUT_BUFS == 1) {
        // a single buffer is rewritten by the next tile: wait for every warp's copy
        if (lane == 0) mbar_arrive(epi_bar);
        ok = warp_wait(epi_bar, ep_ph, abort_flag, P.status, trace, bar0, P.wait_ns);
        ep_ph ^= 1;
        if (!ok) break;
      }
      ++ep_tile;
    }
  }

  // Exit: every warp reconverges (single-lane roles included) and reports;
  // the allocator warp frees TMEM once all have left their loops.
  __syncwarp();
  tc_fence_before();
  if (lane == 0) mbar_arrive(exit_bar);
  if (warp == 2) {
    if (lane == 0) trace_put(trace, 7, 14, 0, 0);
    {  // not cut short by an abort: every warp must have left before TMEM goes
      const uint64_t t0 = global_ns();
      while (!mbar_try(exit_bar, 0) && global_ns() - t0 < P.wait_ns) {}
      __syncwarp();
    }
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                 : "memory");
    if (lane == 0) trace_put(trace, 7, 15, 0, 0);
  }
}

// ------------------------------------------------------------ host side --

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = get_encode();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, dt, rank, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int* g_trace = nullptr;  // test hook: host-mapped progress record
int g_debug_stall = 0;   // test hook: a withheld arrive and a 20 ms wait limit

// SM count of the current device (cached per device).
int sm_count() {
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

// act: fp16 [rows][K]; weight matrices `mats` of the pass (N x K each),
// `box_rows` weight rows per matrix per tile.
moe_status_t make_params(TcParams& P, const FfnArgs& a, const __half* act, int rows, int K, int N,
                         const int* mats, int nmat, int box_rows, int n_blobs) {
  const bool planes = a.layout == MOE_LAYOUT_PLANES;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t str[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, 128};
    if (!encode(&P.act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, act, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) {
      set_error("tensor map (activations) could not be encoded");
      return MOE_ERR_CUDA;
    }
  }
  const cuuint32_t br = static_cast<cuuint32_t>(box_rows);
  for (int i = 0; i < nmat; ++i) {
    const int m = mats[i];
    // code tiles of 16 rows x 128 K: {words of a tile row, 16 rows, K / 128
    // tiles, N / 16 row blocks, blobs}; a box is one K tile of box_rows rows,
    // which lands in shared memory row after row as a row-major
    // [box_rows][words] block
    const cuuint64_t nk = static_cast<cuuint64_t>(K / 128), nr = static_cast<cuuint64_t>(N / 16);
    auto tiles = [&](CUtensorMap* map, size_t off, cuuint64_t words, CUtensorMapSwizzle sw) {
      const cuuint64_t row = words * 4;
      cuuint64_t dims[5] = {words, 16, nk, nr, static_cast<cuuint64_t>(n_blobs)};
      cuuint64_t str[4] = {row, 16 * row, nk * 16 * row, static_cast<cuuint64_t>(a.blob_bytes)};
      cuuint32_t box[5] = {static_cast<cuuint32_t>(words), 16, 1, br / 16, 1};
      return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 5, a.blobs + off, dims, str, box, sw);
    };
    if (!planes) {
      if (!tiles(&P.codes[i], a.lay.codes[m], 16, CU_TENSOR_MAP_SWIZZLE_64B)) {
        set_error("tensor map (codes) could not be encoded");
        return MOE_ERR_CUDA;
      }
    } else {
      if (!tiles(&P.codes[i], a.lay.q2[m], 8, CU_TENSOR_MAP_SWIZZLE_32B) ||
          !tiles(&P.d3[i], a.lay.d3[m], 4, CU_TENSOR_MAP_SWIZZLE_NONE) ||
          !tiles(&P.d4[i], a.lay.d4[m], 4, CU_TENSOR_MAP_SWIZZLE_NONE)) {
        set_error("tensor map (bit planes) could not be encoded");
        return MOE_ERR_CUDA;
      }
    }
    P.sz_off[i] = a.lay.sz[m];
  }
  P.offsets = a.offsets;
  P.slot_of = a.slot_of;
  P.blobs = a.blobs;
  P.blob_bytes = a.blob_bytes;
  P.K = K;
  P.rows = rows;
  P.N = N;
  P.planes_mult = planes ? 3 : 1;
  P.nbins = a.E * P.planes_mult;
  P.group = a.group;
  P.status = a.status;
  P.trace = g_trace;
  P.wait_ns = g_debug_stall ? 20000000ull : kWaitLimitNs;
  P.debug_stall = g_debug_stall;
  return MOE_OK;
}

template <bool GATEUP, bool PLANES>
moe_status_t launch_one(const TcParams& P, bool pdl, cudaStream_t s) {
  auto kern = k_ffn_tc<GATEUP, PLANES>;
  // The shared-memory opt-in is a per-device attribute: set once per device
  // (the first call on a device must precede any stream capture).
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "tc ffn cudaGetDevice");
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<GATEUP>::SMEM);
    if (e != cudaSuccess) return cuda_check(e, "tc ffn smem attribute");
    attr_set.fetch_or(bit);
  }
  return cuda_check(launch_pdl(pdl, kern, dim3(sm_count()), dim3(kThreads), Cfg<GATEUP>::SMEM, s, P), "tc ffn launch");
}

}  // namespace

bool tc_supported(const FfnArgs& a) {
  return get_encode() != nullptr && a.d % 128 == 0 && a.F % 128 == 0 &&
         a.E * (a.layout == MOE_LAYOUT_PLANES ? 3 : 1) <= kMaxBins;
}

moe_status_t launch_ffn_tc(const FfnArgs& a, cudaStream_t s) {
  const bool pdl = pdl_for(a.total_rows);
  const int n_blobs = a.slot_of ? 65536 : a.E;
  const bool planes = a.layout == MOE_LAYOUT_PLANES;
  TcParams gu{};
  const int m_gu[2] = {0, 1};
  moe_status_t st = make_params(gu, a, a.x_perm, a.total_rows, a.d, a.F, m_gu, 2, 128, n_blobs);
  if (st != MOE_OK) return st;
  gu.h_out = a.h;
  gu.y_out = nullptr;
  st = planes ? launch_one<true, true>(gu, pdl, s) : launch_one<true, false>(gu, pdl, s);
  if (st != MOE_OK) return st;
  TcParams dn{};
  const int m_dn[1] = {2};
  st = make_params(dn, a, a.h, a.total_rows, a.F, a.d, m_dn, 1, 128, n_blobs);
  if (st != MOE_OK) return st;
  dn.h_out = nullptr;
  dn.y_out = a.y_perm;
  return planes ? launch_one<false, true>(dn, pdl, s) : launch_one<false, false>(dn, pdl, s);
}

}  // namespace moeq

extern "C" void moe_debug_set_trace(void* host_mapped_ints) {
  moeq::g_trace = static_cast<int*>(host_mapped_ints);
}

extern "C" void moe_debug_ffn_timeout(int enable) { moeq::g_debug_stall = enable ? 1 : 0; }
