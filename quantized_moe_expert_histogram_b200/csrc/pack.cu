// Offline quantiser: fp32 expert weights -> blob format (moeq.h).
//
// One warp quantises one (row, group): lane l holds elements l, l+32, ...
// of the group, so the min/max is a warp reduction and each packed word is
// an OR-reduction over the lanes that own its elements.  The arithmetic is
// the asymmetric 4-bit rule of moe_quant_pack, in IEEE fp32 with
// round-half-even, so the codes are bit-identical to any other IEEE
// implementation of the same rule.
#include "common.cuh"

namespace moeq {
namespace {

template <int G>
__global__ void __launch_bounds__(256) k_pack(const float* __restrict__ w, int rows_per_expert,
                                               int K, int n_items, uint8_t* __restrict__ blobs,
                                               size_t blob_bytes, size_t off_codes, size_t off_q2,
                                               size_t off_d3, size_t off_d4, size_t off_sz,
                                               int planes) {
  constexpr int PER_LANE = G / 32;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_items) return;
  const int groups = K / G;
  const int c = warp % groups;                 // group along K
  const long row_all = warp / groups;          // expert * N + n
  const int e = static_cast<int>(row_all / rows_per_expert);
  const int n = static_cast<int>(row_all % rows_per_expert);
  const float* src = w + row_all * static_cast<long>(K) + static_cast<long>(c) * G;

  float v[PER_LANE];
  float mn = 0.0f, mx = 0.0f;  // the range always includes 0
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    v[i] = src[lane + 32 * i];
    mn = fminf(mn, v[i]);
    mx = fmaxf(mx, v[i]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  __nv_bfloat16 sb = __float2bfloat16_rn(s32);
  float s = __bfloat162float(sb);
  if (s == 0.0f) {
    s = 1.0f;
    sb = __float2bfloat16_rn(1.0f);
  }
  // + 0 turns a -0 zero-point (from mn = -0) into +0: an integer has no sign
  const float z = __fadd_rn(fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.0f), 15.0f), 0.0f);

  uint32_t q[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const float r = __fadd_rn(rintf(__fdiv_rn(v[i], s)), z);
    q[i] = static_cast<uint32_t>(fminf(fmaxf(r, 0.0f), 15.0f));
  }

  uint8_t* blob = blobs + static_cast<size_t>(e) * blob_bytes;
  // element index inside the row of this lane's i-th value: c*G + lane + 32 i.
  // Code words are stored in tiles of 16 rows x 128 elements (`per` words a
  // tile row): word w of row n at tile_word(n, w, per).
  auto tile_word = [&](int w, int per) {
    return (static_cast<size_t>(n >> 4) * (K / 128) + w / per) * (16 * per) + (n & 15) * per + w % per;
  };
  if (!planes) {
    uint32_t* codes = reinterpret_cast<uint32_t*>(blob + off_codes);
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
      uint32_t part = q[i] << (4 * (lane & 7));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) part |= __shfl_xor_sync(0xffffffffu, part, o);
      if ((lane & 7) == 0) codes[tile_word((c * G + 32 * i + lane) / 8, 16)] = part;
    }
  } else {
    uint32_t* q2 = reinterpret_cast<uint32_t*>(blob + off_q2);
    uint32_t* d3 = reinterpret_cast<uint32_t*>(blob + off_d3);
    uint32_t* d4 = reinterpret_cast<uint32_t*>(blob + off_d4);
    // plane order: element i of a run of 8 in nibble (i >> 1) + 4 (i & 1);
    // Q2 shifts the second run of its 16 by 2 bits, D3/D4 run g of 32 by g
    const int nib = 4 * (((lane & 7) >> 1) + 4 * (lane & 1));
    const int sh2 = 2 * ((lane >> 3) & 1) + nib;
    const int sh1 = (lane >> 3) + nib;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
      uint32_t part = (q[i] >> 2) << sh2;
      uint32_t p3 = ((q[i] >> 1) & 1u) << sh1;
      uint32_t p4 = (q[i] & 1u) << sh1;
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) part |= __shfl_xor_sync(0xffffffffu, part, o);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        p3 |= __shfl_xor_sync(0xffffffffu, p3, o);
        p4 |= __shfl_xor_sync(0xffffffffu, p4, o);
      }
      if ((lane & 15) == 0) q2[tile_word((c * G + 32 * i + lane) / 16, 8)] = part;
      if (lane == 0) {
        d3[tile_word((c * G + 32 * i) / 32, 4)] = p3;
        d4[tile_word((c * G + 32 * i) / 32, 4)] = p4;
      }
    }
  }
  if (lane == 0) {
    const __nv_bfloat16 zb = __float2bfloat16_rn(z);
    const uint32_t word = static_cast<uint32_t>(__bfloat16_as_ushort(sb)) |
                          (static_cast<uint32_t>(__bfloat16_as_ushort(zb)) << 16);
    uint32_t* sz = reinterpret_cast<uint32_t*>(blob + off_sz);
    sz[(static_cast<size_t>(n / 128) * groups + c) * 128 + (n % 128)] = word;
  }
}

}  // namespace

moe_status_t launch_pack(const float* w_gate, const float* w_up, const float* w_down, int E, int d,
                         int F, int group, int layout, void* blobs, cudaStream_t s) {
  const BlobLayout L = blob_layout(d, F, group, layout);
  const float* mats[3] = {w_gate, w_up, w_down};
  const int rows[3] = {F, F, d};
  const int Ks[3] = {d, d, F};
  for (int m = 0; m < 3; ++m) {
    const long items = static_cast<long>(E) * rows[m] * (Ks[m] / group);
    if (items > (1L << 31) / 32) {
      set_error("moe_quant_pack: matrix too large (%ld groups)", items);
      return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    const int threads = 256;
    const int blocks = static_cast<int>((items * 32 + threads - 1) / threads);
    auto kern = group == 64 ? k_pack<64> : k_pack<128>;
    kern<<<blocks, threads, 0, s>>>(mats[m], rows[m], Ks[m], static_cast<int>(items),
                                    static_cast<uint8_t*>(blobs), L.bytes, L.codes[m], L.q2[m],
                                    L.d3[m], L.d4[m], L.sz[m], layout == MOE_LAYOUT_PLANES);
    moe_status_t st = cuda_check(cudaGetLastError(), "moe_quant_pack launch");
    if (st != MOE_OK) return st;
  }
  return MOE_OK;
}

}  // namespace moeq
