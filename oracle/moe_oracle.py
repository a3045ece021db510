"""CPU oracle for the token-routed, weight-quantised MoE FFN layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this module.  It shares no code,
header, table or constant with the CUDA library and never imports it.

Every function is a plain, slow restatement of one step of the method, in
the order the sources give it, with a library primitive (a matmul, a sort)
allowed as a step.  Sources (page title, then section):

* "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference" --
  four-bit weights, 16-bit activations; the router's choices are executed
  exactly as made and every chosen expert runs; experts are only stored
  and moved differently; grouped execution of the experts.
* "D2MoE: Dual Routing and Dynamic Scheduling for Efficient On-Device
  MoE-based LLM Serving" -- Design / Token-Adaptive Bit-Width Selection
  (expert gate and bit gate per token), MWQ (W(2)=Q2, W(3)=Q2+D3,
  W(4)=Q2+D3+D4, INT2 within INT3 within INT4), quantisation done offline.
* "Innovativer Ansatz zur Optimierung der Inferenz von Mixture-of-Experts-
  Modellen" (Read-ME) -- expert-aware batching: requests for one expert
  are processed together (the per-expert grouping / permutation).

Precision: integer decisions of the quantiser are taken in IEEE fp32 (the
same operations the GPU performs); router logits, dequantised weights, the
FFN and the combine are evaluated in fp64.  The SwiGLU intermediate h is
kept exact (fp64); the method allows rounding it to bf16, the oracle does
not round it.

Readings where the sources are silent (each also listed in the design
notes): the group range is widened to include 0; the zero-point is an
integer 0..15 stored as bf16; an all-zero group has s=1, z=0; the nested
b-bit weight keeps the top b bits of the 4-bit code with the same s and z;
top-k ties go to the lower expert index and the k outputs are ordered by
descending logit; nested permutation bins are ordered key = 3*e + (b-2);
the bit gate is a linear score per width, ties to the narrower width.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(closed forms, brute force on tiny inputs, invariants, textbook routines).
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# bf16 helpers (bit-level, round-to-nearest-even)
# ---------------------------------------------------------------------------


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 values (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits with round-to-nearest-even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_round(a: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(f32_to_bf16_bits(a))


# ---------------------------------------------------------------------------
# Offline quantisation (ExactMoE: W4A16; D2MoE: quantisation is offline)
# ---------------------------------------------------------------------------


def quantize_groups(w: np.ndarray, group: int):
    """Asymmetric 4-bit group quantisation along K.

    ``w`` float32 [N, K]; each row is cut into K/group groups of ``group``
    consecutive elements.  Per group (fp32 IEEE arithmetic):
      mn = min(min(w), 0), mx = max(max(w), 0)
      s  = bf16((mx - mn) / 15); s = 1 if s == 0
      z  = clamp(rint(-mn / s), 0, 15)
      q  = clamp(rint(w / s) + z, 0, 15)      (rint = round half to even)
    Returns q uint8 [N,K], s float32 [N,K/g] (bf16 values), z float32
    [N,K/g] (integers).
    """
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % group == 0
    G = K // group
    wg = w.reshape(N, G, group)
    mn = np.minimum(wg.min(axis=2), np.float32(0))
    mx = np.maximum(wg.max(axis=2), np.float32(0))
    s = bf16_round((mx - mn) / np.float32(15.0))
    s = np.where(s == 0, np.float32(1.0), s).astype(np.float32)
    # + 0 turns a -0 zero-point (from mn = -0) into +0: an integer has no sign
    z = np.clip(np.rint(-mn / s), 0, 15).astype(np.float32) + np.float32(0.0)
    q = np.rint(wg / s[:, :, None]) + z[:, :, None]
    q = np.clip(q, 0, 15).astype(np.uint8).reshape(N, K)
    return q, s, z


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Codes uint8 [N,K] -> uint32 [N,K/8]; nibble i of word w holds
    element 8w+i (low nibble first)."""
    N, K = q.shape
    qq = q.reshape(N, K // 8, 8).astype(np.uint32)
    out = np.zeros((N, K // 8), dtype=np.uint32)
    for i in range(8):
        out |= qq[:, :, i] << np.uint32(4 * i)
    return out


def unpack_int4(words: np.ndarray, K: int) -> np.ndarray:
    N = words.shape[0]
    out = np.empty((N, K // 8, 8), dtype=np.uint8)
    for i in range(8):
        out[:, :, i] = (words >> np.uint32(4 * i)) & np.uint32(0xF)
    return out.reshape(N, K)


def plane_nibble(i: int) -> int:
    """Nibble that element i (0..7) of an 8-element run occupies in the
    planes' storage order: even elements in nibbles 0..3, odd ones in 4..7
    (element 2j -> nibble j, element 2j+1 -> nibble 4+j)."""
    return (i >> 1) + 4 * (i & 1)


def split_planes(q: np.ndarray):
    """MWQ bit planes of a 4-bit code (D2MoE, MWQ): base = q >> 2 (2 bits),
    D3 = (q >> 1) & 1, D4 = q & 1, stored in the library's plane order:
      Q2 word v (elements 16v..16v+15): element 16v + 8h + i in bits
         2h + 4*plane_nibble(i) .. +1;
      D3, D4 word u (elements 32u..32u+31): element 32u + 8g + i in bit
         g + 4*plane_nibble(i).
    (The method fixes the planes, not their bit order in a storage word.)
    """
    N, K = q.shape
    q = q.astype(np.uint32)
    base = (q >> 2).reshape(N, K // 16, 16)
    d3 = ((q >> 1) & 1).reshape(N, K // 32, 32)
    d4 = (q & 1).reshape(N, K // 32, 32)
    Q2 = np.zeros((N, K // 16), dtype=np.uint32)
    for o in range(16):
        h, i = o // 8, o % 8
        Q2 |= base[:, :, o] << np.uint32(2 * h + 4 * plane_nibble(i))
    D3 = np.zeros((N, K // 32), dtype=np.uint32)
    D4 = np.zeros((N, K // 32), dtype=np.uint32)
    for o in range(32):
        g, i = o // 8, o % 8
        D3 |= d3[:, :, o] << np.uint32(g + 4 * plane_nibble(i))
        D4 |= d4[:, :, o] << np.uint32(g + 4 * plane_nibble(i))
    return Q2, D3, D4


def join_planes(Q2, D3, D4, K: int, b: int = 4) -> np.ndarray:
    """Nested code of width b: W(2) = Q2, W(3) = Q2 + D3, W(4) = Q2 + D3 + D4,
    written as the top b bits of the 4-bit code with the low 4-b bits zero
    (plane order as in split_planes)."""
    N = Q2.shape[0]
    base = np.empty((N, K // 16, 16), dtype=np.uint32)
    for o in range(16):
        h, i = o // 8, o % 8
        base[:, :, o] = (Q2 >> np.uint32(2 * h + 4 * plane_nibble(i))) & np.uint32(3)
    r3 = np.empty((N, K // 32, 32), dtype=np.uint32)
    r4 = np.empty((N, K // 32, 32), dtype=np.uint32)
    for o in range(32):
        g, i = o // 8, o % 8
        r3[:, :, o] = (D3 >> np.uint32(g + 4 * plane_nibble(i))) & np.uint32(1)
        r4[:, :, o] = (D4 >> np.uint32(g + 4 * plane_nibble(i))) & np.uint32(1)
    code = base.reshape(N, K) << np.uint32(2)
    if b >= 3:
        code = code + (r3.reshape(N, K) << np.uint32(1))
    if b >= 4:
        code = code + r4.reshape(N, K)
    return code.astype(np.uint8)


def dequant(q: np.ndarray, s: np.ndarray, z: np.ndarray, group: int, b: int = 4) -> np.ndarray:
    """w' = (q_b - z) * s in fp64, q_b = q with its low 4-b bits cleared."""
    N, K = q.shape
    qb = (q.astype(np.int64) >> (4 - b)) << (4 - b)
    qg = qb.reshape(N, K // group, group).astype(np.float64)
    w = (qg - z.astype(np.float64)[:, :, None]) * s.astype(np.float64)[:, :, None]
    return w.reshape(N, K)


# ---------------------------------------------------------------------------
# Weight blob format (the byte layout the library consumes)
# ---------------------------------------------------------------------------

ROW_TILE = 128  # rows per scale/zero tile in the blob format


def blob_layout(d: int, F: int, group: int, layout: str) -> dict:
    """Byte offsets of every section of one expert's blob.

    INT4: [gate codes F x d/8 u32 | up codes F x d/8 | down codes d x F/8 |
           gate sz | up sz | down sz]
    Code words (INT4 codes, Q2, D3, D4) are stored in tiles of 16 rows x 128
    elements: a tile's rows one after another (16, 8 or 4 words a row), the
    tiles of 16-row block r in K order, then block r + 1 (tile_words).
    planes: [gate Q2 F x d/16 u32 | up Q2 | down Q2 d x F/16 | gate sz | up sz
             | down sz | gate D3 F x d/32 | up D3 | down D3 | gate D4 | up D4
             | down D4]  (bit order inside the words: split_planes).  Width by
             width: the planes a b-bit read needs (Q2 and the scales for b = 2,
             plus D3 for 3, plus D4 for 4) are the blob's first bytes, up to
             the start of D3 (b = 2), of D4 (b = 3) or the end (b = 4).
    sz of an N x K matrix: (scale, zero) bf16 pairs ordered
      [N/128][K/group][128], i.e. pair index ((n//128)*(K/group) + c)*128 + n%128.
    """
    off = {}
    pos = 0
    mats = (("gate", F, d), ("up", F, d), ("down", d, F))
    if layout == "int4":
        for m, N, K in mats:
            off[m + ".codes"] = pos
            pos += N * K // 2
    else:
        for m, N, K in mats:
            off[m + ".q2"] = pos
            pos += N * K // 4
    for m, N, K in mats:
        off[m + ".sz"] = pos
        pos += N * (K // group) * 4
    if layout != "int4":
        for plane in ("d3", "d4"):
            for m, N, K in mats:
                off[m + "." + plane] = pos
                pos += N * K // 8
    off["bytes"] = pos
    return off


def tile_words(words: np.ndarray, per: int) -> np.ndarray:
    """uint32 [N, W] (N rows of W words, `per` words per 128 elements) ->
    the blob's order: for each block of 16 rows, for each run of 128
    elements, the 16 rows' `per` words one row after another."""
    N, W = words.shape
    return np.ascontiguousarray(words.reshape(N // 16, 16, W // per, per).transpose(0, 2, 1, 3)).reshape(-1)


def untile_words(flat: np.ndarray, N: int, W: int, per: int) -> np.ndarray:
    """Inverse of tile_words: the blob's words -> uint32 [N, W]."""
    t = np.asarray(flat, dtype=np.uint32).reshape(N // 16, W // per, 16, per)
    return np.ascontiguousarray(t.transpose(0, 2, 1, 3)).reshape(N, W)


def sz_tiled(s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """(scale, zero) [N, G] -> uint32 words in [N/128][G][128] order, each word
    = bf16(s) | bf16(z) << 16."""
    N, G = s.shape
    word = f32_to_bf16_bits(s).astype(np.uint32) | (f32_to_bf16_bits(z).astype(np.uint32) << np.uint32(16))
    return word.reshape(N // ROW_TILE, ROW_TILE, G).transpose(0, 2, 1).reshape(-1).copy()


def build_blob(w_gate, w_up, w_down, group: int, layout: str) -> np.ndarray:
    """One expert's blob bytes (uint8) from its fp32 matrices."""
    F, d = w_gate.shape
    off = blob_layout(d, F, group, layout)
    blob = np.zeros(off["bytes"], dtype=np.uint8)
    for m, w in (("gate", w_gate), ("up", w_up), ("down", w_down)):
        q, s, z = quantize_groups(w, group)
        if layout == "int4":
            parts = {"codes": tile_words(pack_int4(q), 16)}
        else:
            Q2, D3, D4 = split_planes(q)
            parts = {"q2": tile_words(Q2, 8), "d3": tile_words(D3, 4), "d4": tile_words(D4, 4)}
        parts["sz"] = sz_tiled(s, z)
        for name, arr in parts.items():
            raw = np.ascontiguousarray(arr, dtype=np.uint32).view(np.uint8).reshape(-1)
            o = off[m + "." + name]
            blob[o:o + raw.size] = raw
    return blob


# ---------------------------------------------------------------------------
# Router (ExactMoE: the router decides, every chosen expert runs;
# D2MoE, Dual Routing: x -> Expert Gate -> E_i)
# ---------------------------------------------------------------------------


def router_logits(x: np.ndarray, w_router: np.ndarray, bias=None) -> np.ndarray:
    """l[t,e] = sum_i x[t,i] * W_r[e,i] (+ bias[e]) in fp64.

    Each logit is the same summation of its d exact fp64 products (numpy's
    reduction along a contiguous row), so experts with identical router rows
    get identical logits and the tie rule (lower index) applies; a blocked
    matrix product may round two identical rows differently."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_router, dtype=np.float64)
    l = np.empty((x.shape[0], w.shape[0]), dtype=np.float64)
    for t0 in range(0, x.shape[0], 64):
        l[t0:t0 + 64] = (x[t0:t0 + 64, None, :] * w[None, :, :]).sum(axis=-1)
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def topk_select(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per token, ordered by descending
    logit; equal logits are ordered by ascending expert index."""
    T, E = logits.shape
    out = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        order = np.lexsort((idx, -logits[t]))  # primary -logit, secondary index
        out[t] = order[:k]
    return out


def gates_for(logits: np.ndarray, sel: np.ndarray) -> np.ndarray:
    """Softmax over the selected logits only (= full softmax renormalised
    over the selection), fp64 -> fp32."""
    l = np.take_along_axis(logits, sel.astype(np.int64), axis=1)
    m = l.max(axis=1, keepdims=True)
    e = np.exp(l - m)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def route(x, w_router, bias, k):
    l = router_logits(x, w_router, bias)
    sel = topk_select(l, k)
    return sel, gates_for(l, sel), l


# ---------------------------------------------------------------------------
# Bit-width router (D2MoE, Design / Dual Routing: x -> Bit Gate -> b_i next
# to x -> Expert Gate -> E_i; Token-Adaptive Bit-Width Selection)
# ---------------------------------------------------------------------------

BIT_WIDTHS = (2, 3, 4)


def bit_gate(x: np.ndarray, w_bit: np.ndarray, bias_bit, sel: np.ndarray) -> np.ndarray:
    """Width b[t,j] in {2, 3, 4} of the j-th selected expert e = sel[t,j] of
    token t: the width whose score  x[t] . W_bit[e,c] (+ bias_bit[e,c])  is
    the largest, c = 0, 1, 2 for b = 2, 3, 4, scores in fp64; equal scores
    go to the narrower width.  W_bit fp32 [E, 3, d], bias_bit fp32 [E, 3]
    or None.  (The page places the bit gate per token next to the expert
    gate and ties the width to the expert's importance for the token, but
    gives no form; a linear score per width, read like the expert gate's
    logits, is the plain reading.)"""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_bit, dtype=np.float64)
    b = None if bias_bit is None else np.asarray(bias_bit, dtype=np.float64)
    T, k = sel.shape
    out = np.empty((T, k), dtype=np.uint8)
    for t in range(T):
        for j in range(k):
            e = int(sel[t, j])
            # each score the correctly rounded sum of its exact fp64 products
            # (bf16 x fp32 fits fp64), so equal scores are equal here and the
            # tie rule decides them
            scores = np.array([math.fsum(w[e, c] * x[t]) for c in range(3)])
            if b is not None:
                scores = scores + b[e]
            out[t, j] = BIT_WIDTHS[int(np.argmax(scores))]  # first maximum: the narrower width
    return out


# ---------------------------------------------------------------------------
# Histogram, prefix sum, permutation (expert-aware batching / grouped
# execution)
# ---------------------------------------------------------------------------


def permute(keys: np.ndarray, nbins: int):
    """Stable counting sort of assignments a = 0..n-1 by key.

    counts[b] = #{a: key[a] = b}; offsets = exclusive scan of counts with
    offsets[nbins] = n; perm[p] = a (rows of one bin contiguous, ascending
    a inside a bin); inv_perm[perm[p]] = p.
    """
    keys = np.asarray(keys, dtype=np.int64).reshape(-1)
    n = keys.size
    counts = np.zeros(nbins, dtype=np.int64)
    for a in range(n):
        counts[keys[a]] += 1
    offsets = np.zeros(nbins + 1, dtype=np.int64)
    for b in range(nbins):
        offsets[b + 1] = offsets[b] + counts[b]
    cursor = offsets[:-1].copy()
    perm = np.empty(n, dtype=np.int64)
    for a in range(n):
        p = cursor[keys[a]]
        perm[p] = a
        cursor[keys[a]] += 1
    inv = np.empty(n, dtype=np.int64)
    inv[perm] = np.arange(n)
    return (counts.astype(np.int32), offsets.astype(np.int32), perm.astype(np.int32),
            inv.astype(np.int32))


def assignment_keys(sel: np.ndarray, bits=None) -> tuple:
    """Bin key per assignment a = t*k + j and the number of bins."""
    E_keys = sel.reshape(-1).astype(np.int64)
    if bits is None:
        return E_keys, None
    return E_keys * 3 + (np.asarray(bits).reshape(-1).astype(np.int64) - 2), 3


# ---------------------------------------------------------------------------
# Expert FFN (SwiGLU) and combine
# ---------------------------------------------------------------------------


def silu(v: np.ndarray) -> np.ndarray:
    return v / (1.0 + np.exp(-v))


def expert_ffn(xr: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """y = W_d (silu(W_g x) * (W_u x)) for each row of xr, fp64."""
    a = xr @ wg.T
    u = xr @ wu.T
    h = silu(a) * u
    return h @ wd.T


def combine(y_assign: np.ndarray, gates: np.ndarray) -> np.ndarray:
    """y[t] = sum_j g[t,j] * y_{t*k+j}, j ascending, fp64."""
    T, k = gates.shape
    ya = y_assign.reshape(T, k, -1)
    y = np.zeros((T, ya.shape[2]), dtype=np.float64)
    for j in range(k):
        y += gates[:, j:j + 1].astype(np.float64) * ya[:, j, :]
    return y


class QuantExperts:
    """Quantised experts of one layer, dequantised lazily per (expert, b)."""

    def __init__(self, w_gate, w_up, w_down, group: int):
        self.w = (np.asarray(w_gate, np.float32), np.asarray(w_up, np.float32),
                  np.asarray(w_down, np.float32))
        self.group = group
        self._q = {}

    def quant(self, e: int):
        if e not in self._q:
            self._q[e] = tuple(quantize_groups(m[e], self.group) for m in self.w)
        return self._q[e]

    def weights(self, e: int, b: int = 4):
        return tuple(dequant(q, s, z, self.group, b) for (q, s, z) in self.quant(e))


def moe_layer(x, w_router, bias, k, experts: QuantExperts, bits=None, sel=None,
              token_subset=None) -> dict:
    """Whole layer in the method's order: route, histogram/scan/permute,
    grouped expert FFN, weighted combine.

    ``sel`` (int [T,k]) forces the expert choice (offload trace); gates are
    then the softmax over those logits.  ``token_subset`` limits the FFN and
    combine to some tokens (routing and permutation still cover all).
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    E = np.asarray(w_router).shape[0]
    logits = router_logits(x, w_router, bias)
    if sel is None:
        sel = topk_select(logits, k)
    gates = gates_for(logits, sel)
    keys, mult = assignment_keys(sel, bits)
    nbins = E * (mult or 1)
    counts, offsets, perm, inv = permute(keys, nbins)
    toks = np.arange(T) if token_subset is None else np.asarray(token_subset)
    d = x.shape[1]
    y_assign = np.zeros((T * k, d), dtype=np.float64)
    need = np.zeros(T * k, dtype=bool)
    for t in toks:
        need[t * k:(t + 1) * k] = True
    for key in range(nbins):
        rows = perm[offsets[key]:offsets[key + 1]]
        rows = rows[need[rows]]
        if rows.size == 0:
            continue
        e = key if mult is None else key // 3
        b = 4 if mult is None else key % 3 + 2
        wg, wu, wd = experts.weights(e, b)
        y_assign[rows] = expert_ffn(x[rows // k], wg, wu, wd)
    y = combine(y_assign, gates)
    return dict(logits=logits, sel=sel, gates=gates, counts=counts, offsets=offsets, perm=perm,
                inv_perm=inv, y_assign=y_assign, y=y, tokens=toks)
