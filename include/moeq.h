/*
 * moeq.h -- C ABI of a B200 (sm_100a) library for one token-routed
 * mixture-of-experts FFN layer whose expert weights are stored low-bit.
 *
 * The layer, in the order the calls below run it:
 *   route (softmax top-k)  ->  per-expert histogram, prefix sum and
 *   permutation  ->  per-expert SwiGLU FFN with the dequantisation fused in
 *   (gate/up, then down)  ->  weighted unpermute-combine,
 * plus an offline packer and an offload mode with a GPU slot cache.
 *
 * Sources (page title, section):
 *   [ExactMoE] "Every Expert Counts: ExactMoE for Memory-Efficient W4A16
 *              Inference": four-bit expert weights with 16-bit activations;
 *              the router's decisions are executed exactly and every chosen
 *              expert runs; compressed experts live in host memory and are
 *              moved into a GPU-resident slot cache; grouped execution.
 *   [D2MoE]    "D2MoE: Dual Routing and Dynamic Scheduling for Efficient
 *              On-Device MoE-based LLM Serving": Dual Routing (expert gate,
 *              bit gate), MWQ nested weights W(2)=Q2, W(3)=Q2+D3,
 *              W(4)=Q2+D3+D4, quantisation done offline, the pipeline
 *              "I/O -> dequant -> FP16 -> GEMM" and "Load E2 || Compute E1".
 *   [EdgeMoE]  "EdgeMoE" article: expert weights kept outside device memory
 *              and loaded on activation into an expert buffer.
 *   [Read-ME]  "Innovativer Ansatz zur Optimierung der Inferenz von
 *              Mixture-of-Experts-Modellen": expert-aware batching.
 *
 * Conventions for every call:
 *   - Plain C.  Every pointer is a DEVICE pointer unless its name ends in
 *     _host.  The caller allocates and owns every buffer; the library keeps
 *     no pointer after a call returns (except the slot cache object).
 *   - Streams are passed as `moe_stream_t` (a cudaStream_t; NULL = legacy
 *     default stream).  Every call is asynchronous on its stream and
 *     returns after launch-time validation; nothing here synchronises the
 *     device except where a call says so.
 *   - Errors: a call returns a moe_status_t; MOE_OK means the work was
 *     queued.  moe_last_error() gives a message for the calling thread.
 *     Problems that can only be seen on the device (an expert id out of
 *     range, an activation outside fp16 range, a bounded wait that ran
 *     out) are OR-ed into the caller's device word `status` as MOE_DEV_*
 *     bits; the caller reads it after synchronising.  No call aborts,
 *     traps or prints.
 *   - Outputs are fully overwritten and must not alias inputs.
 *   - bf16 / fp16 buffers are passed as void* and hold IEEE binary16 /
 *     bfloat16 bit patterns.
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef void* moe_stream_t; /* cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null pointer, negative size, k > E ... */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* a size the kernels do not handle      */
  MOE_ERR_CUDA = 3,              /* a CUDA runtime call failed            */
  MOE_ERR_OOM = 4,               /* host or device allocation failed      */
  MOE_ERR_TIMEOUT = 5,           /* reserved for host-side waits          */
  MOE_ERR_WORKSPACE = 6,         /* workspace smaller than required       */
  MOE_ERR_FAULT_INJECTED = 7     /* host-side fault injection fired       */
} moe_status_t;

/* Bits OR-ed into the caller's device status word. */
#define MOE_DEV_BAD_INDEX 1u   /* expert id or bit-width out of range (clamped) */
#define MOE_DEV_RANGE 2u       /* activation or expert output outside fp16 range */
#define MOE_DEV_TIMEOUT 4u     /* a bounded on-device wait gave up          */

typedef enum {
  MOE_LAYOUT_INT4 = 0,   /* 4-bit codes, 8 per uint32                      */
  MOE_LAYOUT_PLANES = 1  /* MWQ bit planes Q2 (2 bit) + D3 + D4 (1 bit)    */
} moe_layout_t;

/* Thread-local message describing the last failure (never NULL). */
MOE_API const char* moe_last_error(void);

/* ---------------------------------------------------------------------
 * Weight format ("blob"): one contiguous byte block per expert, so one
 * copy moves one expert ([ExactMoE] slot cache; [EdgeMoE] expert buffer).
 * For hidden size d, expert width F (d_ff) and group size g:
 *   INT4  : gate codes [F][d/8] u32 | up codes [F][d/8] | down codes
 *           [d][F/8] | gate sz | up sz | down sz
 *   PLANES: gate Q2 [F][d/16] | up Q2 | down Q2 [d][F/16] | gate sz |
 *           up sz | down sz | gate D3 [F][d/32] | up D3 | down D3 [d][F/32]
 *           | gate D4 | up D4 | down D4 -- width by width, so that what a
 *           b-bit read needs (Q2 and the scales; D3 from b = 3; D4 at 4)
 *           is the blob's first bytes
 * Code words are stored in tiles of 16 rows x 128 K: a region of N rows
 * holds, for each block of 16 rows and each run of 128 K in order, the 16
 * rows' words of that run one row after another (16 words a row for INT4
 * codes, 8 for Q2, 4 for D3 and D4); word w of row n is at index
 * ((n / 16) * (K / 128) + w / per) * 16 per + (n % 16) per + w % per.  A
 * 16-row stage of 128 K is thus one contiguous 1 KB (INT4), 512 B (Q2) or
 * 256 B (D3, D4).
 * Code word packing: nibble i of an INT4 codes word = element 8w+i (low
 * nibble first).  Planes use the plane order, n(i) = (i >> 1) + 4 (i & 1)
 * for element i of a run of 8 (even elements in nibbles 0..3, odd ones in
 * 4..7): Q2 word w holds element 16w + 8h + i in bits 2h + 4 n(i) .. +1;
 * D3/D4 word w holds element 32w + 8g + i in bit g + 4 n(i), so a 4-bit
 * code word of 8 elements is (Q2 parts) << 2 | D3 part << 1 | D4 part
 * with one shift and mask per plane.  sz of an N x K matrix is N*K/g uint32 words, word =
 * bf16(scale) | bf16(zero) << 16, ordered [N/128][K/g][128] (row tile of
 * 128, then group, then row inside the tile).  Dequantised weight of a
 * b-bit read: w = ((code >> (4-b) << (4-b)) - zero) * scale.
 * Supported: d, F multiples of 128; g in {64, 128}; d % g == F % g == 0.
 * Returns the blob size in bytes, or 0 for an unsupported shape.
 * ------------------------------------------------------------------ */
MOE_API size_t moe_blob_bytes(int d, int F, int group, int layout);

/* moe_quant_pack -- offline quantisation ([D2MoE] quantisation is done
 * offline; [ExactMoE] W4A16).  w_gate, w_up: fp32 [E][F][d]; w_down: fp32
 * [E][d][F] (row-major, K contiguous).  Per (row, group of g consecutive
 * K): mn = min(min w, 0), mx = max(max w, 0), s = bf16((mx-mn)/15) (1 if
 * 0), z = clamp(rint(-mn/s), 0, 15), code = clamp(rint(w/s)+z, 0, 15), all
 * IEEE fp32 with round-half-even.  Writes E blobs of moe_blob_bytes()
 * each into `blobs` (16-byte aligned).  Not on the timed path. */
MOE_API moe_status_t moe_quant_pack(const float* w_gate, const float* w_up, const float* w_down, int E,
                            int d, int F, int group, int layout, void* blobs,
                            moe_stream_t stream);

/* moe_route_topk -- softmax top-k router ([D2MoE] Dual Routing, expert
 * gate; [ExactMoE] the router decides, nothing is pruned).
 *   x        bf16 [T][d];  w_router fp32 [E][d];  bias fp32 [E] or NULL
 *   logits   l[t][e] = sum_i x[t][i] * w_router[e][i] + bias[e]
 *   topk_idx int32 [T][k]: the k largest logits, ordered by descending
 *            logit; equal logits go to the lower expert index.  The choice
 *            is that of the exact logits: they are evaluated in fp32 with
 *            a proven error bound, and a token whose choice the bound does
 *            not settle (near ties, non-finite values) is re-evaluated and
 *            selected in fp64, where every bf16 x fp32 product is exact.
 *   topk_w   fp32 [T][k]: softmax over the k selected logits (the full
 *            softmax renormalised over the selection), from the fp32
 *            logits (fp64 ones for re-evaluated tokens)
 *            The smallest batches (T <= 8, T*E <= 512, d % 256 == 0) run both
 *            steps as one launch of a thread-block cluster (one d slice per
 *            CTA, a tighter per-logit bound from the sums of the products'
 *            magnitudes, fp64 only for the contenders of unsettled tokens).
 *   forced_idx int32 [T][k] or NULL: when given, the selection is taken
 *            from it as is (an external trace) and only topk_w is
 *            computed for it; topk_idx receives a copy.
 *   workspace >= moe_route_workspace_bytes(T, d, E) bytes of device
 *            scratch, 16-byte aligned (x and w_router too).
 * Requires 1 <= k <= E <= 256, k <= 16, d % 32 == 0. */
MOE_API moe_status_t moe_route_topk(const void* x, const float* w_router, const float* bias,
                            const int32_t* forced_idx, int T, int d, int E, int k,
                            int32_t* topk_idx, float* topk_w, void* workspace,
                            size_t workspace_bytes, moe_stream_t stream);

/* Device scratch moe_route_topk needs (per-slice fp32 partial logits and
 * squared norms). */
MOE_API size_t moe_route_workspace_bytes(int T, int d, int E);

/* moe_route_topk_noalloc -- the same router with no workspace argument.
 * (Library plumbing: the pages describe no counterpart.)  For callers that
 * cannot allocate device memory where they route: plugins and runtimes that
 * receive only a stream and no allocator, and serving paths that must not
 * risk an allocation failure or its implicit synchronisation.  The scratch lives in
 * a fixed 8 MiB device array inside the library, which every GPU that loads
 * the library holds until the process exits; the call allocates nothing.
 *   - Arguments and results are those of moe_route_topk (expert ids equal
 *     bit for bit; gates may differ in the last bits where this call sums
 *     the logits over fewer slices of d).
 *   - The number of d slices is lowered until the scratch fits the array;
 *     sizes whose one-slice scratch, (T*E + T + E) fp32 words, exceeds
 *     8 MiB are rejected with MOE_ERR_UNSUPPORTED_SHAPE.
 *   - The first call on a device resolves the array's device address for
 *     that device (cudaGetSymbolAddress, with that device current); make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array: calls that may overlap on
 *     the GPU (different streams without ordering) race and must not be
 *     issued.  Nothing in the array needs clearing between calls. */
MOE_API moe_status_t moe_route_topk_noalloc(const void* x, const float* w_router, const float* bias,
                                            const int32_t* forced_idx, int T, int d, int E, int k,
                                            int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* moe_permute -- per-expert histogram, exclusive prefix sum and stable
 * permutation of the T*k assignments a = t*k + j ([Read-ME] expert-aware
 * batching; [ExactMoE] grouped execution).  No atomics: per-block
 * histograms of 1024 assignments, one scan over (bin, block), and a
 * rank-by-warp-match scatter that also gathers the rows.
 *   workspace >= moe_permute_workspace_bytes(T, E, k, bits != NULL) bytes.
 *   bits uint8 [T][k] or NULL.  NULL: bin of a = topk_idx[a] (nbins = E).
 *        Given ([D2MoE] bit gate): bin = 3*topk_idx[a] + (bits[a]-2),
 *        nbins = 3E, bits in {2,3,4}.
 *   counts  int32 [nbins]; offsets int32 [nbins+1] (offsets[nbins] = T*k)
 *   perm    int32 [T*k]: perm[p] = a, bins contiguous, ascending a inside
 *   inv_perm int32 [T*k]: inv_perm[perm[p]] = p
 *   x (bf16 [T][d]) and x_perm (fp16 [T*k][d]) may both be NULL; when
 *   given, x_perm[p] = fp16(x[perm[p]/k]) (the activation rows in expert
 *   order, converted for the fp16 tensor-core operands).
 * Out-of-range ids/bits are clamped into range and flag MOE_DEV_BAD_INDEX;
 * |x| > 65504 flags MOE_DEV_RANGE.  Requires T*k <= 2^24, nbins <= 768. */
MOE_API moe_status_t moe_permute(const int32_t* topk_idx, const uint8_t* bits, const void* x, int T,
                         int d, int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv_perm, void* x_perm, int32_t* status, void* workspace,
                         size_t workspace_bytes, moe_stream_t stream);

/* Device scratch moe_permute needs (per-block histograms); nested != 0 for
 * the (expert, width) bins. */
MOE_API size_t moe_permute_workspace_bytes(int T, int E, int k, int nested);

/* moe_route_permute -- the front of the layer in one call: moe_route_topk,
 * then (with a bit gate) moe_bit_gate, then moe_permute, with their results
 * bit for bit ([ExactMoE] the router decides, every routed expert runs;
 * [D2MoE] Dual Routing: expert gate and bit gate side by side; [Read-ME]
 * expert-aware batching).  The smallest batches -- T <= 8, T*E <= 512
 * (with a bit gate T*E <= 128), T*k <= 64, d % 256 == 0 -- run as one
 * launch of a thread-block cluster (the cluster router of moe_route_topk,
 * the width scores of every expert computed with the logits and decided
 * the same way, then the permutation and the gather); other sizes issue
 * the separate launches on `stream`.
 *   forced_idx int32 [T][k] or NULL, as in moe_route_topk.
 *   bits_in    uint8 [T][k] widths given by the caller (nested bins), or NULL.
 *   w_bit, bias_bit  the bit gate as in moe_bit_gate, or NULL; with w_bit,
 *              bits_in must be NULL and bits_out (uint8 [T][k]) receives
 *              the widths, which key the nested bins.
 *   topk_idx, topk_w, counts, offsets, perm, inv_perm, x_perm: as in
 *              moe_route_topk and moe_permute (x_perm may be NULL: no gather).
 *   workspace >= moe_route_permute_workspace_bytes(T, d, E, k, nested)
 *              bytes, 16-byte aligned (nested != 0 with bits_in or w_bit).
 * Errors and device flags as in the three calls it stands for. */
MOE_API moe_status_t moe_route_permute(const void* x, const float* w_router, const float* bias,
                                       const int32_t* forced_idx, const uint8_t* bits_in, const float* w_bit,
                                       const float* bias_bit, int T, int d, int E, int k, int32_t* topk_idx,
                                       float* topk_w, uint8_t* bits_out, int32_t* counts, int32_t* offsets,
                                       int32_t* perm, int32_t* inv_perm, void* x_perm, int32_t* status,
                                       void* workspace, size_t workspace_bytes, moe_stream_t stream);
MOE_API size_t moe_route_permute_workspace_bytes(int T, int d, int E, int k, int nested);

/* Workspace bytes moe_grouped_ffn_wq needs for `total_rows` = T*k rows. */
MOE_API size_t moe_ffn_workspace_bytes(int total_rows, int E, int d, int F, int layout);

/* moe_grouped_ffn_wq -- the grouped expert FFN with dequantisation fused
 * into both GEMMs ([D2MoE] pipeline I/O -> dequant -> FP16 -> GEMM;
 * [ExactMoE] W4A16, grouped execution).  For every bin (expert e, width b)
 * and each of its rows p in [offsets[bin], offsets[bin+1]):
 *     h[p]      = silu(Wg_e,b . x_perm[p]) * (Wu_e,b . x_perm[p])
 *     y_perm[p] = Wd_e,b . h[p]
 * with W_e,b the b-bit dequantised weights of the blob format above (b = 4
 * for MOE_LAYOUT_INT4, b = 2 + bin % 3 for MOE_LAYOUT_PLANES).
 *   x_perm   fp16 [total_rows][d] (from moe_permute)
 *   offsets  int32 [nbins+1] (device; never read by the host)
 *   blobs    device pool of expert blobs, blob i at blobs + i*blob_bytes
 *   slot_of  int32 [E] or NULL.  NULL: expert e is blob e.  Given: expert
 *            e is blob slot_of[e]; experts with slot_of[e] < 0 are skipped
 *            (their y_perm rows are left untouched).
 *   T        token count (no bin holds more than T rows; selects the
 *            kernel: up to 16 tokens -- and up to 64 when d >= 4096 and
 *            bins average at most 12 rows (total_rows <= 12 nbins) -- the
 *            decode kernel, which streams the weights once per 8 or 16
 *            rows of a bin with mma.sync dot products split over warps
 *            along K; otherwise the tensor-core grouped GEMM with 128-row
 *            tiles)
 *   workspace >= moe_ffn_workspace_bytes() bytes of device scratch
 *   y_perm   fp16 [total_rows][d]
 * Accumulation is fp32; the SwiGLU intermediate h is stored as fp16 and
 * y_perm rounded once to fp16; an output beyond the fp16 range (|y| >
 * 65504, or NaN) flags MOE_DEV_RANGE in `status`. */
MOE_API moe_status_t moe_grouped_ffn_wq(const void* x_perm, const int32_t* offsets, const void* blobs,
                                const int32_t* slot_of, int total_rows, int T, int E, int d,
                                int F, int group, int layout, void* workspace,
                                size_t workspace_bytes, void* y_perm, int32_t* status,
                                moe_stream_t stream);

/* moe_grouped_ffn_combine -- moe_grouped_ffn_wq (every expert resident,
 * blob e = expert e) followed by moe_unpermute_combine on `stream`, with
 * their results (y_perm and y; [ExactMoE] every routed expert runs exactly,
 * weighted by its gate): one entry point for the second half of a layer
 * step.  (Summing the combine inside the decode kernel's second GEMM was
 * measured slower than the separate launch at every batch size.)
 *   perm, inv_perm  int32 [T*k] from moe_permute; topk_w fp32 [T][k];
 *   residual        bf16 [T][d] or NULL; y bf16 [T][d]; y_perm fp16 [T*k][d],
 *                   all 16-byte aligned
 *   workspace >= moe_ffn_combine_workspace_bytes(T, k, E, d, F, layout),
 *   16-byte aligned (the FFN's scratch).
 * Requires k <= 16, d % 16 == 0; errors and flags as in the two calls. */
MOE_API moe_status_t moe_grouped_ffn_combine(const void* x_perm, const int32_t* offsets, const void* blobs, int T,
                                             int k, int E, int d, int F, int group, int layout,
                                             const int32_t* perm, const int32_t* inv_perm, const float* topk_w,
                                             const void* residual, void* y, void* y_perm, void* workspace,
                                             size_t workspace_bytes, int32_t* status, moe_stream_t stream);
MOE_API size_t moe_ffn_combine_workspace_bytes(int T, int k, int E, int d, int F, int layout);

/* moe_bit_gate -- bit-width router ([D2MoE] Dual Routing: x -> Bit Gate ->
 * b beside x -> Expert Gate -> E; Token-Adaptive Bit-Width Selection): the
 * width at which each selected expert runs for each token.  For the j-th
 * selected expert e = topk_idx[t][j] of token t:
 *   score[c]   = x[t] . w_bit[e][c] + bias_bit[e][c],   c = 0, 1, 2
 *   bits[t][j] = 2 + the c of the largest score (equal scores -> the lower
 *                c, i.e. the narrower width)
 * The decision is that of the exact scores: they are evaluated in fp32 with
 * a proven error bound, and an assignment whose winner the bound does not
 * settle is re-evaluated in fp64, where every bf16 x fp32 product is exact.
 *   x bf16 [T][d]; w_bit fp32 [E][3][d]; bias_bit fp32 [E][3] or NULL;
 *   topk_idx int32 [T][k] (from moe_route_topk); bits uint8 [T][k], the
 *   input moe_permute takes for the (expert, width) bins.
 * Ids outside [0, E) are clamped and flag MOE_DEV_BAD_INDEX in `status`
 * (may be NULL).  Requires d % 8 == 0 and 16-byte aligned x and w_bit. */
MOE_API moe_status_t moe_bit_gate(const void* x, const float* w_bit, const float* bias_bit,
                                  const int32_t* topk_idx, int T, int d, int E, int k, uint8_t* bits,
                                  int32_t* status, moe_stream_t stream);

/* moe_static_bits -- per-expert static bit widths ([EdgeMoE] expert-wise
 * bit-width adaptation, the fixed-width case of [D2MoE] nested weights):
 *   bits[t][j] = width_of[topk_idx[t][j]]
 *   topk_idx int32 [T][k]; width_of uint8 [E] (device), each in {2, 3, 4};
 *   bits uint8 [T][k] (device), the input moe_permute takes for the (expert,
 *   width) bins of the nested-plane layout.
 * Ids outside [0, E) or widths outside {2, 3, 4} are clamped and flag
 * MOE_DEV_BAD_INDEX in `status` (may be NULL). */
MOE_API moe_status_t moe_static_bits(const int32_t* topk_idx, const uint8_t* width_of, int T, int k, int E,
                                     uint8_t* bits, int32_t* status, moe_stream_t stream);

/* moe_unpermute_combine -- weighted combine ([ExactMoE]: every chosen
 * expert's output is used as the router weighted it).
 *   y[t] = bf16( residual[t] + sum_{j<k} topk_w[t][j] * y_perm[inv_perm[t*k+j]] )
 * summed in fp32 in ascending j; y_perm fp16 [T*k][d]; residual bf16 [T][d]
 * or NULL (0).  y bf16 [T][d]; requires d % 8 == 0, and y_perm, y and the
 * residual 16-byte aligned (MOE_ERR_INVALID_ARG otherwise). */
MOE_API moe_status_t moe_unpermute_combine(const void* y_perm, const int32_t* inv_perm,
                                   const float* topk_w, const void* residual, int T, int k, int d,
                                   void* y, moe_stream_t stream);

/* ---------------------------------------------------------------------
 * Offload mode ([ExactMoE] compressed experts in host memory, GPU slot
 * cache; [EdgeMoE] expert buffer; [D2MoE] "Load E2 || Compute E1").
 * One cache object per layer: `slots` device slots of one blob each.
 * ------------------------------------------------------------------ */
typedef struct moe_slot_cache moe_slot_cache;

/* Create a cache for one layer.  host_blobs: E blobs in PINNED host memory
 * (cudaHostAlloc / registered), blob e at host_blobs + e*blob_bytes.
 * device_pool: caller-allocated device memory of slots*blob_bytes bytes.
 * The cache allocates host bookkeeping, CUDA events and a small device
 * table; it starts empty.  Requires 2 <= slots and E <= 256. */
MOE_API moe_status_t moe_slot_cache_create(int E, int slots, size_t blob_bytes, const void* host_blobs,
                                   void* device_pool, moe_slot_cache** out);

/* The same for nested-plane blobs (MOE_LAYOUT_PLANES of shape d, F, group;
 * blob_bytes = moe_blob_bytes(d, F, group, MOE_LAYOUT_PLANES)), in plane
 * mode ([D2MoE] MWQ: W(2) needs only Q2, W(3) adds D3, W(4) adds D4): a
 * slot holds an expert's planes up to some width, a step copies an expert
 * only up to the widest width its assignments use (the Q2 planes and the
 * scales for width 2, plus D3 for 3, plus D4 for 4), and a resident expert
 * that is later needed wider receives only its missing planes.  The blob
 * is laid out width by width, so each of these is one contiguous copy
 * (the blob's first bytes, or the range between two widths); experts are
 * staged hottest first and each expert's base planes come first ([D2MoE]
 * Hottest-Expert-Bit-First). */
MOE_API moe_status_t moe_slot_cache_create_planes(int E, int slots, int d, int F, int group,
                                                  const void* host_blobs, void* device_pool,
                                                  moe_slot_cache** out);

/* Plan one layer-step: ids_host (n_ids expert ids, host memory, repeats
 * allowed) are the experts the router chose; bits_host (n_ids widths in
 * {2, 3, 4}, host memory) their widths in plane mode, or NULL (every expert
 * at width 4; ignored outside plane mode).  Resident experts holding every
 * plane the step needs are hits; the others need copies (a fresh load into
 * the least-recently-used free slot, or the missing planes of a resident
 * expert).  The distinct experts are split into waves of at most slots/2
 * (hits first, then the experts with copies by descending row count) so
 * that copies of wave w+1 run on copy_stream while wave w computes on
 * compute_stream.  Issues the copies of the first two waves.  *n_waves
 * receives the wave count; stats_host (may be NULL) receives {hits,
 * experts copied, bytes copied}. */
MOE_API moe_status_t moe_slot_stage(moe_slot_cache* cache, const int32_t* ids_host, const uint8_t* bits_host,
                                    int n_ids, moe_stream_t copy_stream, moe_stream_t compute_stream,
                                    int32_t* n_waves, int64_t* stats_host);

/* Run the staged layer-step: for each wave, compute_stream waits for the
 * wave's copies, the grouped FFN (same arguments as moe_grouped_ffn_wq)
 * runs on the wave's experts through the device slot table, and the next
 * copies that reuse the wave's slots are issued after it.  Every routed
 * expert is executed; results equal the all-resident call bit for bit. */
MOE_API moe_status_t moe_slot_ffn(moe_slot_cache* cache, const void* x_perm, const int32_t* offsets,
                          int total_rows, int T, int d, int F, int group, int layout,
                          void* workspace, size_t workspace_bytes, void* y_perm,
                          int32_t* status, moe_stream_t copy_stream, moe_stream_t compute_stream);

/* Stage experts ahead of their layer-step ([EdgeMoE] expert preloading;
 * [D2MoE] load the next experts while the current ones compute): copies up
 * to `max_copies` of the listed experts that are not resident into the
 * least recently used slots, in list order, on copy_stream.  Each copy waits
 * for the compute that last read its slot; the next moe_slot_ffn of this
 * cache waits for these copies, and the next moe_slot_stage counts them as
 * hits.  Use the copy stream of this cache's moe_slot_stage calls: a later
 * stage may reuse a prefetched slot, and stream order keeps the two copies
 * apart.  n_copied (may be NULL) receives the number of copies issued.
 * Allowed order per cache: ... moe_slot_ffn -> moe_slot_prefetch ->
 * moe_slot_stage -> moe_slot_ffn ...; a call between moe_slot_stage and
 * its moe_slot_ffn is rejected with MOE_ERR_INVALID_ARG (it could evict an
 * expert the staged plan relies on).  Prefetching changes only where
 * experts are when they are needed, never the result. */
MOE_API moe_status_t moe_slot_prefetch(moe_slot_cache* cache, const int32_t* ids_host, int n_ids, int max_copies,
                                       moe_stream_t copy_stream, int32_t* n_copied);

/* Busy-time measurement of the offload pipeline (the load/compute overlap
 * figure): with enable != 0 the cache records CUDA timing events around each
 * wave's copies (after the copy stream's waits for free slots) and around
 * each wave's FFN (after the compute stream's wait for those copies), so the
 * sums count only the time each stream works, not the time it waits for the
 * other.  moe_slot_timing_read waits for the recorded events (a host
 * synchronisation), returns the copy and FFN milliseconds since the last
 * read or enable, and starts new sums.  Off by default. */
MOE_API moe_status_t moe_slot_timing(moe_slot_cache* cache, int enable);
MOE_API moe_status_t moe_slot_timing_read(moe_slot_cache* cache, double* copy_ms, double* ffn_ms);

/* Next-layer expert predictor (host-only; [EdgeMoE] expert preloading: a
 * statistical profile keyed by the experts activated at the two preceding
 * layers, experts preloaded in order of their estimated probability).
 * Learned online with moe_predictor_observe from the routed ids of earlier
 * steps, per token and choice position j: counts of (expert at layer-1 ->
 * expert at layer) and, when prev2_ids is given and E <= 64, of
 * ((expert at layer-2, expert at layer-1) -> expert at layer).
 * moe_predictor_predict scores the experts of `layer` by the summed
 * conditional frequencies (the expected number of assignments to each
 * expert), using the pair key for a pair seen at least twice and the
 * one-layer key otherwise, and writes up to max_out ids, best first (ties:
 * lower id), only experts whose score is nonzero and at least min_score.
 * ids are host int32 [T][k]; prev2_ids may be NULL (one-layer key only) and
 * needs layer >= 2. */
typedef struct moe_route_predictor moe_route_predictor;
MOE_API moe_status_t moe_predictor_create(int layers, int E, moe_route_predictor** out);
MOE_API void moe_predictor_destroy(moe_route_predictor* p);
MOE_API moe_status_t moe_predictor_observe(moe_route_predictor* p, int layer, const int32_t* prev2_ids,
                                           const int32_t* prev_ids, const int32_t* cur_ids, int T, int k);
MOE_API moe_status_t moe_predictor_predict(const moe_route_predictor* p, int layer, const int32_t* prev2_ids,
                                           const int32_t* prev_ids, int T, int k, int max_out, double min_score,
                                           int32_t* out_ids, int32_t* n_out);

/* Free the cache's host bookkeeping, events and device table (not the
 * caller's pool or host blobs).  Synchronises the events it owns. */
MOE_API void moe_slot_cache_destroy(moe_slot_cache* cache);

/* Host-side fault injection for tests: the next `count` calls of
 * moe_slot_stage fail with MOE_ERR_FAULT_INJECTED before queuing any work
 * (what = 1), or the cache's next copy reports a failed copy (what = 2).
 * what = 0 clears it. */
MOE_API void moe_debug_inject_fault(int what, int count);

/* Test hook: 0 = the default choice of FFN kernel (the rule stated at
 * moe_grouped_ffn_wq: the decode kernel for small batches, with one
 * 8-token block per pass, or two where T > 8 and bins average more than
 * 6 rows, and the tensor-core grouped GEMM above); 1 = the decode kernel
 * with one 8-token block per pass; 2 = the tensor-core kernel whenever
 * the shape allows it; 3 = the decode kernel with two blocks; 4, 5 = the
 * earlier CUDA-core GEMV and small-batch kernels (comparison only).
 * Process-wide. */
MOE_API void moe_debug_force_regime(int regime);

/* Test hook: when non-NULL, the tensor-core FFN kernels record each warp
 * role's progress into this pinned, device-mapped host buffer of
 * 2 * gridDim * 16 ints (slot = (wait site << 24) | (tile << 12) | k-block),
 * so that a stalled launch can be read from the host while it runs.
 * NULL (the default) disables it. */
MOE_API void moe_debug_set_trace(void* host_mapped_ints);

/* Test hook (process-wide), selecting among paths with the same results:
 * 1 (the default): moe_route_topk takes the smallest batches (T <= 8,
 * T*E <= 512, d % 256 == 0) in one thread-block-cluster launch,
 * moe_bit_gate up to 32 assignments (d % 64 == 0) in one cluster launch,
 * and moe_route_permute fuses all three steps (see there).  0: the
 * two-launch router and the one-kernel bit gate, and separate launches in
 * moe_route_permute, at every size. */
MOE_API void moe_debug_route_fused(int mode);

/* Test hook of the on-device failure path: while enabled, the tensor-core
 * FFN kernels give every bounded wait a 20 ms limit (instead of 2 s), and in
 * the gate/up kernel the epilogue of CTA 0 withholds the release of its
 * first tile's accumulators -- an arrive with no copy behind it -- so that
 * the MMA warp's wait for its next tile runs out whenever CTA 0 has more than
 * one tile.  The CTA then sets MOE_DEV_TIMEOUT in `status`, drains its
 * copies and MMAs, frees its tensor memory and returns; that call's outputs
 * are undefined.  0 (the default) disables it.  Process-wide. */
MOE_API void moe_debug_ffn_timeout(int enable);

#ifdef __cplusplus
}
#endif

#endif /* MOEQ_H */
