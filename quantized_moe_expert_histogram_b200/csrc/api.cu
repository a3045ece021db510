// C ABI entry points: argument validation, regime dispatch, error strings.
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>

#include "common.cuh"

namespace moeq {

namespace {
thread_local char g_err[512] = "no error";

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}

// Argument checks shared by the router entry points (everything except
// the scratch, which each entry point provides its own way).
moe_status_t route_check_args(const void* x, const float* w_router, int T, int d, int E, int k,
                              const int32_t* topk_idx, const float* topk_w, const char* fn) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0) {
    set_error("%s: bad sizes T=%d d=%d E=%d k=%d", fn, T, d, E, k);
    return MOE_ERR_INVALID_ARG;
  }
  if (T > 0 && (!x || !w_router || !topk_idx || !topk_w)) {
    set_error("%s: null pointer", fn);
    return MOE_ERR_INVALID_ARG;
  }
  if (k > E || k > 16 || E > 256) {
    set_error("%s: need k <= E, k <= 16, E <= 256 (k=%d E=%d)", fn, k, E);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (d % 32) {
    set_error("%s: d=%d must be a multiple of 32", fn, d);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (T > 0 && (!aligned16(x) || !aligned16(w_router))) {
    set_error("%s: x and w_router must be 16-byte aligned", fn);
    return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

moe_status_t cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MOE_OK;
  set_error("%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
  return MOE_ERR_CUDA;
}

BlobLayout blob_layout(int d, int F, int group, int layout) {
  BlobLayout L{};
  L.valid = 0;
  if (d <= 0 || F <= 0 || d % 128 || F % 128) return L;
  if (group != 64 && group != 128) return L;
  if (d % group || F % group) return L;
  if (layout != MOE_LAYOUT_INT4 && layout != MOE_LAYOUT_PLANES) return L;
  const size_t N[3] = {(size_t)F, (size_t)F, (size_t)d};
  const size_t K[3] = {(size_t)d, (size_t)d, (size_t)F};
  // INT4: codes of gate, up, down, then their scales.  PLANES, width by
  // width: Q2 of the three matrices, their scales, then D3 of the three,
  // then D4 -- the planes of a b-bit read are the blob's first bytes.
  size_t pos = 0;
  for (int m = 0; m < 3; ++m) {
    if (layout == MOE_LAYOUT_INT4) {
      L.codes[m] = pos;
      pos += N[m] * K[m] / 2;
    } else {
      L.q2[m] = pos;
      pos += N[m] * K[m] / 4;
    }
  }
  for (int m = 0; m < 3; ++m) {
    L.sz[m] = pos;
    pos += N[m] * (K[m] / group) * 4;
  }
  if (layout == MOE_LAYOUT_PLANES) {
    for (int m = 0; m < 3; ++m) {
      L.d3[m] = pos;
      pos += N[m] * K[m] / 8;
    }
    for (int m = 0; m < 3; ++m) {
      L.d4[m] = pos;
      pos += N[m] * K[m] / 8;
    }
  }
  L.bytes = pos;
  L.valid = 1;
  return L;
}

}  // namespace moeq

using namespace moeq;

namespace {

inline cudaStream_t S(moe_stream_t s) { return static_cast<cudaStream_t>(s); }

// Regime by T (bins never hold more than T rows): up to kDecMaxT tokens ->
// the decode kernel (weight-streaming, split-K over warps, mma.sync with one
// or two 8-token blocks); above -> the tensor-core grouped GEMM (128-row
// weight tiles, tcgen05).
constexpr int kDecMaxT = 16;

// Above kDecMaxT tokens the decode kernel still wins on layers with long
// rows (d >= 4096) while bins stay short: up to 64 tokens with bins of at
// most 12 rows on average (T k <= 12 E mult; measured FFN, decode against
// tensor cores: Mixtral-shaped 24 tokens 242 / 340 us, 32 tokens 278 / 340,
// 48 tokens 327 / 341, 64 tokens 423 / 342; nested 64 tokens 162 / 169).  On
// the OLMoE-shaped layer (d = 2048: units of two stages per warp) the
// tensor cores win from 32 tokens (71 against 79 us).
inline bool decode_fits(int T, int k, int E, int mult, int d) {
  return T <= kDecMaxT || (T <= 64 && d >= 4096 && static_cast<long>(T) * k <= 12L * E * mult);
}

// Token blocks of the decode kernel: one 8-token block per pass over the
// weights (three CTAs per SM) unless bins are likely to hold more than 8
// rows, where two blocks read each weight stage once for 16 rows.  Bins
// hold T k / (E mult) rows on average; up to 6, a second pass is rare
// (measured FFN, one block against two: OLMoE-shaped 16 tokens 50.9 / 55.5
// us, nested 16 tokens 110.0 / 130.2, Mixtral-shaped 24 tokens 242 / 272;
// at 32 tokens, 8 rows a bin, two blocks win: 278 against 288).
inline int decode_regime(int T, int k, int E, int mult) {
  return T <= 8 || static_cast<long>(T) * k <= 6L * E * mult ? 1 : 3;
}

// 0: pick by T; 1: the decode kernel with one 8-token block per pass; 2:
// tensor cores whenever possible; 3: the decode kernel with two 8-token
// blocks; 4, 5: the earlier CUDA-core GEMV and the earlier small-batch
// kernel (comparison only).
int g_force_regime = 0;

size_t workspace_for(int total_rows, int F) {
  size_t h = static_cast<size_t>(total_rows) * F * sizeof(__half);
  return (h + 255) & ~static_cast<size_t>(255);
}

}  // namespace

extern "C" {

const char* moe_last_error(void) { return g_err; }

void moe_debug_force_regime(int regime) { g_force_regime = (regime >= 0 && regime <= 5) ? regime : 0; }

size_t moe_blob_bytes(int d, int F, int group, int layout) {
  const BlobLayout L = blob_layout(d, F, group, layout);
  return L.valid ? L.bytes : 0;
}

moe_status_t moe_quant_pack(const float* w_gate, const float* w_up, const float* w_down, int E,
                            int d, int F, int group, int layout, void* blobs,
                            moe_stream_t stream) {
  if (!w_gate || !w_up || !w_down || !blobs || E <= 0) {
    set_error("moe_quant_pack: null pointer or E <= 0");
    return MOE_ERR_INVALID_ARG;
  }
  const BlobLayout L = blob_layout(d, F, group, layout);
  if (!L.valid) {
    set_error("moe_quant_pack: unsupported shape d=%d F=%d group=%d layout=%d", d, F, group, layout);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (!aligned16(blobs)) {
    set_error("moe_quant_pack: blobs must be 16-byte aligned");
    return MOE_ERR_INVALID_ARG;
  }
  return launch_pack(w_gate, w_up, w_down, E, d, F, group, layout, blobs, S(stream));
}

size_t moe_route_workspace_bytes(int T, int d, int E) { return route_workspace_bytes(T, d, E); }

moe_status_t moe_route_topk(const void* x, const float* w_router, const float* bias,
                            const int32_t* forced_idx, int T, int d, int E, int k,
                            int32_t* topk_idx, float* topk_w, void* workspace,
                            size_t workspace_bytes, moe_stream_t stream) {
  moe_status_t st = route_check_args(x, w_router, T, d, E, k, topk_idx, topk_w, "moe_route_topk");
  if (st != MOE_OK) return st;
  if (T > 0 && (!workspace || workspace_bytes < route_workspace_bytes(T, d, E))) {
    set_error("moe_route_topk: workspace %zu < %zu bytes", workspace_bytes,
              route_workspace_bytes(T, d, E));
    return MOE_ERR_WORKSPACE;
  }
  if (T > 0 && !aligned16(workspace)) {
    set_error("moe_route_topk: workspace must be 16-byte aligned");
    return MOE_ERR_INVALID_ARG;
  }
  return launch_route(x, w_router, bias, forced_idx, T, d, E, k, topk_idx, topk_w, workspace,
                      workspace_bytes, S(stream));
}

size_t moe_permute_workspace_bytes(int T, int E, int k, int nested) {
  if (T < 0 || E <= 0 || k <= 0) return 0;
  return permute_workspace_bytes(T, k, nested ? 3 * E : E);
}

moe_status_t moe_permute(const int32_t* topk_idx, const uint8_t* bits, const void* x, int T,
                         int d, int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv_perm, void* x_perm, int32_t* status, void* workspace,
                         size_t workspace_bytes, moe_stream_t stream) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) {
    set_error("moe_permute: bad sizes T=%d E=%d k=%d", T, E, k);
    return MOE_ERR_INVALID_ARG;
  }
  if (!counts || !offsets || (T > 0 && (!topk_idx || !perm || !inv_perm))) {
    set_error("moe_permute: null pointer");
    return MOE_ERR_INVALID_ARG;
  }
  if (static_cast<long>(T) * k > (1L << 24)) {
    set_error("moe_permute: T*k = %ld exceeds 2^24", static_cast<long>(T) * k);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if ((x == nullptr) != (x_perm == nullptr)) {
    set_error("moe_permute: x and x_perm must both be given or both be NULL");
    return MOE_ERR_INVALID_ARG;
  }
  if (x_perm && (d <= 0 || d % 8 || !aligned16(x) || !aligned16(x_perm))) {
    set_error("moe_permute: gather needs d %% 8 == 0 and 16-byte aligned x / x_perm");
    return MOE_ERR_INVALID_ARG;
  }
  const size_t need = permute_workspace_bytes(T, k, bits ? 3 * E : E);
  if (!workspace || workspace_bytes < need) {
    set_error("moe_permute: workspace %zu < %zu bytes", workspace_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  return launch_permute(topk_idx, bits, x, T, d, E, k, counts, offsets, perm, inv_perm, x_perm,
                        status, workspace, S(stream));
}

size_t moe_route_permute_workspace_bytes(int T, int d, int E, int k, int nested) {
  if (T <= 0 || d <= 0 || E <= 0 || k <= 0) return 256;
  const size_t r = (route_workspace_bytes(T, d, E) + 255) / 256 * 256;
  return r + permute_workspace_bytes(T, k, nested ? 3 * E : E);
}

moe_status_t moe_route_permute(const void* x, const float* w_router, const float* bias, const int32_t* forced_idx,
                               const uint8_t* bits_in, const float* w_bit, const float* bias_bit, int T, int d,
                               int E, int k, int32_t* topk_idx, float* topk_w, uint8_t* bits_out,
                               int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* x_perm,
                               int32_t* status, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  moe_status_t st = route_check_args(x, w_router, T, d, E, k, topk_idx, topk_w, "moe_route_permute");
  if (st != MOE_OK) return st;
  if (bits_in && w_bit) {
    set_error("moe_route_permute: give the widths (bits_in) or the bit gate (w_bit), not both");
    return MOE_ERR_INVALID_ARG;
  }
  if (w_bit && !bits_out) {
    set_error("moe_route_permute: the bit gate needs bits_out");
    return MOE_ERR_INVALID_ARG;
  }
  if (!counts || !offsets || (T > 0 && (!perm || !inv_perm))) {
    set_error("moe_route_permute: null pointer");
    return MOE_ERR_INVALID_ARG;
  }
  if (w_bit && (d % 8 || !aligned16(w_bit))) {
    set_error("moe_route_permute: the bit gate needs d %% 8 == 0 and a 16-byte aligned w_bit");
    return MOE_ERR_INVALID_ARG;
  }
  if (x_perm && (d % 8 || !aligned16(x_perm))) {
    set_error("moe_route_permute: gather needs d %% 8 == 0 and a 16-byte aligned x_perm");
    return MOE_ERR_INVALID_ARG;
  }
  if (static_cast<long>(T) * k > (1L << 24)) {
    set_error("moe_route_permute: T*k exceeds 2^24");
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  const bool nested = bits_in || w_bit;
  const size_t need = moe_route_permute_workspace_bytes(T, d, E, k, nested ? 1 : 0);
  if (T > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) {
    set_error("moe_route_permute: workspace %zu < %zu bytes or not 16-byte aligned", workspace_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  if (T == 0) {  // empty batch: the separate calls write the (zero) counts and offsets
    const uint8_t* nested_flag = bits_in ? bits_in : (w_bit ? bits_out : nullptr);  // selects 3E bins
    return launch_permute(topk_idx, nested_flag, nullptr, 0, d, E, k, counts, offsets, perm, inv_perm, nullptr,
                          status, workspace, S(stream));
  }
  if (route_permute_fusable(T, d, E, k, w_bit != nullptr))
    return launch_front_tiny(x, w_router, bias, forced_idx, bits_in, w_bit, bias_bit, T, d, E, k, topk_idx, topk_w,
                             bits_out, counts, offsets, perm, inv_perm, x_perm, status, S(stream));
  const size_t rbytes = (route_workspace_bytes(T, d, E) + 255) / 256 * 256;
  st = launch_route(x, w_router, bias, forced_idx, T, d, E, k, topk_idx, topk_w, workspace, rbytes, S(stream));
  if (st != MOE_OK) return st;
  const uint8_t* bits = bits_in;
  if (w_bit) {
    st = launch_bit_gate(x, w_bit, bias_bit, topk_idx, T, d, E, k, bits_out, status, S(stream));
    if (st != MOE_OK) return st;
    bits = bits_out;
  }
  return launch_permute(topk_idx, bits, x_perm ? x : nullptr, T, d, E, k, counts, offsets, perm, inv_perm, x_perm,
                        status, static_cast<uint8_t*>(workspace) + rbytes, S(stream));
}

size_t moe_ffn_workspace_bytes(int total_rows, int E, int d, int F, int layout) {
  (void)E;
  (void)d;
  (void)layout;
  if (total_rows < 0 || F <= 0) return 0;
  return workspace_for(total_rows, F);
}

moe_status_t moe_grouped_ffn_wq(const void* x_perm, const int32_t* offsets, const void* blobs,
                                const int32_t* slot_of, int total_rows, int T, int E, int d,
                                int F, int group, int layout, void* workspace,
                                size_t workspace_bytes, void* y_perm, int32_t* status,
                                moe_stream_t stream) {
  if (total_rows < 0 || T < 0 || E <= 0) {
    set_error("moe_grouped_ffn_wq: bad sizes");
    return MOE_ERR_INVALID_ARG;
  }
  const BlobLayout L = blob_layout(d, F, group, layout);
  if (!L.valid) {
    set_error("moe_grouped_ffn_wq: unsupported shape d=%d F=%d group=%d layout=%d", d, F, group,
              layout);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (total_rows == 0) return MOE_OK;
  if (!x_perm || !offsets || !blobs || !workspace || !y_perm) {
    set_error("moe_grouped_ffn_wq: null pointer");
    return MOE_ERR_INVALID_ARG;
  }
  if (!aligned16(x_perm) || !aligned16(blobs) || !aligned16(workspace) || !aligned16(y_perm)) {
    set_error("moe_grouped_ffn_wq: buffers must be 16-byte aligned");
    return MOE_ERR_INVALID_ARG;
  }
  if (workspace_bytes < workspace_for(total_rows, F)) {
    set_error("moe_grouped_ffn_wq: workspace %zu < %zu bytes", workspace_bytes,
              workspace_for(total_rows, F));
    return MOE_ERR_WORKSPACE;
  }
  if (E * (layout == MOE_LAYOUT_PLANES ? 3 : 1) > 768) {
    set_error("moe_grouped_ffn_wq: too many bins");
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  FfnArgs a{};
  a.x_perm = static_cast<const __half*>(x_perm);
  a.offsets = offsets;
  a.blobs = static_cast<const uint8_t*>(blobs);
  a.slot_of = slot_of;
  a.total_rows = total_rows;
  a.T = T;
  a.E = E;
  a.d = d;
  a.F = F;
  a.group = group;
  a.layout = layout;
  a.blob_bytes = L.bytes;
  a.lay = L;
  a.h = static_cast<__half*>(workspace);
  a.y_perm = static_cast<__half*>(y_perm);
  a.status = status;
  const bool tc_ok = total_rows >= 16 && tc_supported(a);
  int regime = g_force_regime;
  if (regime == 0) {
    const int k = std::max(1, total_rows / std::max(1, T)), mult = layout == MOE_LAYOUT_PLANES ? 3 : 1;
    regime = decode_fits(T, k, E, mult, d) || !tc_ok ? decode_regime(T, k, E, mult) : 2;
  }
  if (regime == 2 && !tc_ok) regime = 3;
  if (regime == 2) return launch_ffn_tc(a, S(stream));
  if (regime == 4) return launch_ffn_gemv(a, S(stream));
  if (regime == 5) return launch_ffn_gemv_mma(a, S(stream));
  return launch_ffn_decode(a, regime == 1 ? 1 : 2, S(stream));
}

size_t moe_ffn_combine_workspace_bytes(int T, int k, int E, int d, int F, int layout) {
  (void)E;
  (void)d;
  (void)layout;
  if (T <= 0 || k <= 0 || F <= 0) return 256;
  return workspace_for(T * k, F);
}

// The FFN call, then the combine launch.  Summing the combine inside the
// decode kernel's second GEMM (the unit that completes a token's k rows of
// an output block adds them, after a fence and a count) was built and
// measured slower at every size (layer step, fused against separate:
// OLMoE-shaped 1 token 29.5 / 27.9 us, 16 tokens 79.4 / 72.7; nested 64
// tokens 220.1 / 199.2; Mixtral-shaped 32 tokens 312.6 / 300.6): the fence
// and barriers each unit pays outweigh the launch.
moe_status_t moe_grouped_ffn_combine(const void* x_perm, const int32_t* offsets, const void* blobs, int T, int k,
                                     int E, int d, int F, int group, int layout, const int32_t* perm,
                                     const int32_t* inv_perm, const float* topk_w, const void* residual, void* y,
                                     void* y_perm, void* workspace, size_t workspace_bytes, int32_t* status,
                                     moe_stream_t stream) {
  if (T < 0 || k <= 0 || k > 16 || E <= 0 || d <= 0 || d % 16) {
    set_error("moe_grouped_ffn_combine: bad sizes T=%d k=%d E=%d d=%d", T, k, E, d);
    return MOE_ERR_INVALID_ARG;
  }
  if (T == 0) return MOE_OK;
  if (!perm || !inv_perm || !topk_w || !y) {
    set_error("moe_grouped_ffn_combine: null pointer");
    return MOE_ERR_INVALID_ARG;
  }
  if (!aligned16(y) || (residual && !aligned16(residual))) {  // the combine's 16-byte loads and stores
    set_error("moe_grouped_ffn_combine: y and residual must be 16-byte aligned");
    return MOE_ERR_INVALID_ARG;
  }
  if (static_cast<long>(T) * k > (1L << 24)) {
    set_error("moe_grouped_ffn_combine: T*k exceeds 2^24");
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  const size_t need = moe_ffn_combine_workspace_bytes(T, k, E, d, F, layout);
  if (!workspace || workspace_bytes < need) {
    set_error("moe_grouped_ffn_combine: workspace %zu < %zu bytes", workspace_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  moe_status_t st = moe_grouped_ffn_wq(x_perm, offsets, blobs, nullptr, T * k, T, E, d, F, group, layout,
                                       workspace, workspace_bytes, y_perm, status, stream);
  if (st != MOE_OK) return st;
  if (!aligned16(y_perm)) {
    set_error("moe_grouped_ffn_combine: y_perm must be 16-byte aligned");
    return MOE_ERR_INVALID_ARG;
  }
  // the FFN's second GEMM, the launch just before, writes only y_perm: the
  // combine may read gates, inv_perm and the residual before its wait
  return launch_combine(y_perm, inv_perm, topk_w, residual, T, k, d, y, S(stream), true);
}

moe_status_t moe_bit_gate(const void* x, const float* w_bit, const float* bias_bit, const int32_t* topk_idx,
                          int T, int d, int E, int k, uint8_t* bits, int32_t* status, moe_stream_t stream) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) {
    set_error("moe_bit_gate: bad sizes T=%d d=%d E=%d k=%d", T, d, E, k);
    return MOE_ERR_INVALID_ARG;
  }
  if (d % 8) {
    set_error("moe_bit_gate: d=%d must be a multiple of 8", d);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (static_cast<long>(T) * k > (1L << 24)) {
    set_error("moe_bit_gate: T*k exceeds 2^24");
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (T == 0) return MOE_OK;
  if (!x || !w_bit || !topk_idx || !bits) {
    set_error("moe_bit_gate: null pointer");
    return MOE_ERR_INVALID_ARG;
  }
  if (!aligned16(x) || !aligned16(w_bit)) {
    set_error("moe_bit_gate: x and w_bit must be 16-byte aligned");
    return MOE_ERR_INVALID_ARG;
  }
  return launch_bit_gate(x, w_bit, bias_bit, topk_idx, T, d, E, k, bits, status, S(stream));
}

moe_status_t moe_static_bits(const int32_t* topk_idx, const uint8_t* width_of, int T, int k, int E,
                             uint8_t* bits, int32_t* status, moe_stream_t stream) {
  if (T < 0 || k <= 0 || E <= 0) {
    set_error("moe_static_bits: bad sizes T=%d k=%d E=%d", T, k, E);
    return MOE_ERR_INVALID_ARG;
  }
  if (static_cast<long>(T) * k > (1L << 24)) {
    set_error("moe_static_bits: T*k exceeds 2^24");
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (T == 0) return MOE_OK;
  if (!topk_idx || !width_of || !bits) {
    set_error("moe_static_bits: null pointer");
    return MOE_ERR_INVALID_ARG;
  }
  return launch_static_bits(topk_idx, width_of, T * k, E, bits, status, S(stream));
}

moe_status_t moe_unpermute_combine(const void* y_perm, const int32_t* inv_perm,
                                   const float* topk_w, const void* residual, int T, int k, int d,
                                   void* y, moe_stream_t stream) {
  if (T < 0 || k <= 0 || d <= 0 || d % 8) {
    set_error("moe_unpermute_combine: bad sizes T=%d k=%d d=%d", T, k, d);
    return MOE_ERR_INVALID_ARG;
  }
  if (T > 0 && (!y_perm || !inv_perm || !topk_w || !y)) {
    set_error("moe_unpermute_combine: null pointer");
    return MOE_ERR_INVALID_ARG;
  }
  if (!aligned16(y_perm) || !aligned16(y) || (residual && !aligned16(residual))) {  // 16-byte loads and stores
    set_error("moe_unpermute_combine: y_perm, y and residual must be 16-byte aligned");
    return MOE_ERR_INVALID_ARG;
  }
  return launch_combine(y_perm, inv_perm, topk_w, residual, T, k, d, y, S(stream));
}

}  // extern "C"
