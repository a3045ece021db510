"""Pins for the oracle's offline quantisation, bit planes, dequant and blob
format.  Sources: ExactMoE (W4A16 weights), D2MoE (MWQ nested planes,
offline quantisation).  Every expected value here is either worked out by
hand (see tests/golden/quant_worked_examples.txt), a closed form, or an
invariant that a wrong sign, index or dropped term would break."""
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_groups():
    cases = []
    with open(os.path.join(GOLDEN, "quant_worked_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w, s, z, q = line.split("|")
            cases.append((np.array([float(v) for v in w.split()], np.float32), float(s), float(z),
                          np.array([int(v) for v in q.split()], np.uint8)))
    return cases


@pytest.mark.parametrize("case", range(len(_golden_groups())))
def test_worked_examples(case):
    w, s, z, q = _golden_groups()[case]
    qq, ss, zz = O.quantize_groups(w[None, :], w.size)
    assert ss[0, 0] == np.float32(s)
    assert zz[0, 0] == np.float32(z)
    np.testing.assert_array_equal(qq[0], q)


def test_closed_form_uniform_grid():
    # w_i = (i - z) * s with s a power of two: the codes must be exactly i.
    rng = np.random.default_rng(1)
    for z in range(16):
        for e in (-9, -6, -3):
            s = 2.0 ** e
            w = ((np.arange(16) - z) * s).astype(np.float32)
            perm = rng.permutation(16)
            q, ss, zz = O.quantize_groups(w[perm][None, :], 16)
            lo, hi = min(w.min(), 0), max(w.max(), 0)
            if hi - lo != 15 * s:  # range extended by 0 only when z is 0 or 15
                continue
            assert ss[0, 0] == s and zz[0, 0] == z
            np.testing.assert_array_equal(q[0], np.arange(16)[perm])


def test_zero_group_and_zero_point_range():
    q, s, z = O.quantize_groups(np.zeros((2, 64), np.float32), 64)
    assert (s == 1).all() and (z == 0).all() and (q == 0).all()
    rng = np.random.default_rng(2)
    w = rng.normal(0, 0.02, (64, 256)).astype(np.float32)
    q, s, z = O.quantize_groups(w, 64)
    assert q.max() <= 15 and z.min() >= 0 and z.max() <= 15
    # scale is a bf16 value
    np.testing.assert_array_equal(O.bf16_round(s), s)


def test_error_bound():
    rng = np.random.default_rng(3)
    for dist in ("normal", "uniform", "skewed"):
        if dist == "normal":
            w = rng.normal(0, 0.02, (128, 512))
        elif dist == "uniform":
            w = rng.uniform(-1, 1, (128, 512))
        else:
            w = rng.exponential(0.05, (128, 512))
        w = w.astype(np.float32)
        for g in (64, 128):
            q, s, z = O.quantize_groups(w, g)
            wd = O.dequant(q, s, z, g)
            sE = np.repeat(s, g, axis=1).astype(np.float64)
            zE = np.repeat(z, g, axis=1).astype(np.float64)
            err = np.abs(w.astype(np.float64) - wd)
            assert (err <= 1.1 * sE).all()
            raw = np.rint(w / np.repeat(s, g, axis=1)) + zE
            interior = (raw >= 0) & (raw <= 15)
            assert interior.mean() > 0.99
            bound = 0.5 * sE + 2.0 ** -23 * np.abs(w)
            assert (err[interior] <= bound[interior]).all()


def test_pack_int4_hand_values():
    q = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 15, 0, 0, 0, 0, 0, 0, 10]], np.uint8)
    words = O.pack_int4(q)
    assert words.tolist() == [[0x87654321, 0xA000000F]]
    np.testing.assert_array_equal(O.unpack_int4(words, 16), q)


def test_planes_hand_values():
    q = np.zeros((1, 32), np.uint8)
    Q2, D3, D4 = O.split_planes(q + 15)
    assert Q2.tolist() == [[0xFFFFFFFF, 0xFFFFFFFF]] and D3.tolist() == [[0xFFFFFFFF]]
    assert D4.tolist() == [[0xFFFFFFFF]]
    # plane order: in a run of 8 elements, element 2j sits in nibble j and
    # element 2j+1 in nibble 4+j; Q2 puts the second run of its 16 at +2
    # bits, D3/D4 put run g of their 32 at +g bits
    q[0, 0] = 1      # D4 of element 0 (run 0, nibble 0)        -> D4 bit 0
    q[0, 8] = 1      # D4 of element 8 (run 1, nibble 0)        -> D4 bit 1
    q[0, 1] = 4      # base 1 of element 1 (run 0, nibble 4)    -> Q2 word 0 bits 16..17
    q[0, 10] = 12    # base 3 of element 10 (run 1, nibble 1)   -> Q2 word 0 bits 6..7
    q[0, 31] = 8     # base 2 of element 31 (run 1, nibble 7)   -> Q2 word 1 bits 30..31
    q[0, 5] = 2      # D3 of element 5 (run 0, nibble 6)        -> D3 bit 24
    q[0, 9] = 2      # D3 of element 9 (run 1, nibble 4)        -> D3 bit 17
    q[0, 30] = 2     # D3 of element 30 (run 3, nibble 3)       -> D3 bit 15
    Q2, D3, D4 = O.split_planes(q)
    assert Q2.tolist() == [[0x000100C0, 0x80000000]]
    assert D3.tolist() == [[0x01028000]]
    assert D4.tolist() == [[0x00000003]]
    np.testing.assert_array_equal(O.join_planes(Q2, D3, D4, 32), q)
    assert [O.plane_nibble(i) for i in range(8)] == [0, 4, 1, 5, 2, 6, 3, 7]


def test_planes_nesting():
    rng = np.random.default_rng(4)
    q = rng.integers(0, 16, (8, 256)).astype(np.uint8)
    Q2, D3, D4 = O.split_planes(q)
    # W(4) = Q2 + D3 + D4 reproduces the 4-bit code (D2MoE, MWQ)
    np.testing.assert_array_equal(O.join_planes(Q2, D3, D4, 256, 4), q)
    # INT2 within INT3 within INT4: the b-bit code is the top b bits
    np.testing.assert_array_equal(O.join_planes(Q2, D3, D4, 256, 3), q & 0b1110)
    np.testing.assert_array_equal(O.join_planes(Q2, D3, D4, 256, 2), q & 0b1100)
    # 4 * Q2 + 2 * D3 + D4 == q element-wise
    b2 = O.join_planes(Q2, D3, D4, 256, 2).astype(int)
    b3 = O.join_planes(Q2, D3, D4, 256, 3).astype(int)
    assert ((b3 - b2) // 2 <= 1).all() and ((q.astype(int) - b3) <= 1).all()


def test_nested_dequant_hand_values():
    # q = 13 = 0b1101, z = 3, s = 0.5: b=2 keeps 12 -> 4.5, b=3 keeps 12 -> 4.5,
    # b=4 keeps 13 -> 5.0
    q = np.full((1, 64), 13, np.uint8)
    s = np.array([[0.5]], np.float32)
    z = np.array([[3.0]], np.float32)
    assert O.dequant(q, s, z, 64, 2)[0, 0] == 4.5
    assert O.dequant(q, s, z, 64, 3)[0, 0] == 4.5
    assert O.dequant(q, s, z, 64, 4)[0, 0] == 5.0


def test_bf16_rounding_hand_values():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 1.0 + 2 ** -7 + 2 ** -8], np.float32)
    # ties go to even: 1+2^-8 -> 1.0 ; 1+3*2^-9 -> 1+2^-7 ; 1+2^-7+2^-8 -> 1+2^-6
    exp = [0x3F80, 0x3F80, 0x3F81, 0xC020, 0x3F82]
    assert O.f32_to_bf16_bits(vals).tolist() == exp


def test_blob_layout_sizes_and_roundtrip():
    # olmoe-shaped expert, INT4 g128: 3*F*d/2 code bytes + 3 * F*d/128 * 4 sz bytes
    assert O.blob_layout(2048, 1024, 128, "int4")["bytes"] == 3342336
    # nested shape at b=4 reads the same bytes as INT4
    assert O.blob_layout(4096, 1024, 128, "planes")["bytes"] == O.blob_layout(4096, 1024, 128, "int4")["bytes"]
    rng = np.random.default_rng(5)
    d, F, g = 256, 384, 64
    wg, wu = rng.normal(0, .02, (2, F, d)).astype(np.float32)
    wd = rng.normal(0, .02, (d, F)).astype(np.float32)
    for layout in ("int4", "planes"):
        off = O.blob_layout(d, F, g, layout)
        blob = O.build_blob(wg, wu, wd, g, layout)
        assert blob.size == off["bytes"]
        for m, w in (("gate", wg), ("up", wu), ("down", wd)):
            N, K = w.shape
            q, s, z = O.quantize_groups(w, g)
            if layout == "int4":
                o = off[m + ".codes"]
                words = O.untile_words(blob[o:o + N * K // 2].view(np.uint32), N, K // 8, 16)
                np.testing.assert_array_equal(O.unpack_int4(words, K), q)
            else:
                Q2 = O.untile_words(blob[off[m + ".q2"]:off[m + ".q2"] + N * K // 4].view(np.uint32), N, K // 16, 8)
                D3 = O.untile_words(blob[off[m + ".d3"]:off[m + ".d3"] + N * K // 8].view(np.uint32), N, K // 32, 4)
                D4 = O.untile_words(blob[off[m + ".d4"]:off[m + ".d4"] + N * K // 8].view(np.uint32), N, K // 32, 4)
                np.testing.assert_array_equal(O.join_planes(Q2, D3, D4, K), q)
            o = off[m + ".sz"]
            sz = blob[o:o + N * (K // g) * 4].view(np.uint32)
            G = K // g
            for n in (0, 1, 127, 128, N - 1):
                for c in range(G):
                    word = int(sz[((n // 128) * G + c) * 128 + n % 128])
                    assert O.bf16_bits_to_f32(np.array([word & 0xFFFF]))[0] == s[n, c]
                    assert O.bf16_bits_to_f32(np.array([word >> 16]))[0] == z[n, c]


def test_planes_blob_is_laid_out_width_by_width():
    """Nested-plane blobs: what a b-bit read needs -- Q2 and the scales for
    b = 2, D3 from b = 3, D4 at b = 4 (MWQ: W(2) = Q2, W(3) = Q2 + D3,
    W(4) = Q2 + D3 + D4) -- is the blob's first bytes: keeping only the
    prefix up to the end of width b and zeroing the rest still decodes every
    matrix's codes truncated to b bits and its scales exactly, for every b."""
    rng = np.random.default_rng(6)
    d, F, g = 256, 384, 64
    wg, wu = rng.normal(0, .02, (2, F, d)).astype(np.float32)
    wd = rng.normal(0, .02, (d, F)).astype(np.float32)
    off = O.blob_layout(d, F, g, "planes")
    blob = O.build_blob(wg, wu, wd, g, "planes")
    q2_bytes = (2 * F * d + d * F) // 4
    sz_bytes = (2 * F * (d // g) + d * (F // g)) * 4
    ends = {2: off["gate.d3"], 3: off["gate.d4"], 4: off["bytes"]}
    assert ends[2] == q2_bytes + sz_bytes
    assert ends[3] - ends[2] == ends[4] - ends[3] == (2 * F * d + d * F) // 8
    for b, end in ends.items():
        part = blob.copy()
        part[end:] = 0
        for m, w in (("gate", wg), ("up", wu), ("down", wd)):
            N, K = w.shape
            q, s, z = O.quantize_groups(w, g)
            Q2 = O.untile_words(part[off[m + ".q2"]:off[m + ".q2"] + N * K // 4].view(np.uint32), N, K // 16, 8)
            D3 = O.untile_words(part[off[m + ".d3"]:off[m + ".d3"] + N * K // 8].view(np.uint32), N, K // 32, 4)
            D4 = O.untile_words(part[off[m + ".d4"]:off[m + ".d4"] + N * K // 8].view(np.uint32), N, K // 32, 4)
            np.testing.assert_array_equal(O.join_planes(Q2, D3, D4, K), (q >> (4 - b)) << (4 - b))
            o = off[m + ".sz"]
            np.testing.assert_array_equal(part[o:o + N * (K // g) * 4], blob[o:o + N * (K // g) * 4])


def test_code_tiles_hand_positions():
    """The blob's code words come in tiles of 16 rows x 128 elements: word w
    of row n (K/8 words a row for INT4, 16 per tile row) sits at
    ((n // 16) * (K / 128) + w // 16) * 256 + (n % 16) * 16 + w % 16.  Hand
    positions for N = 32, K = 256 (two row blocks, two tiles each), and the
    round trip."""
    N, K = 32, 256
    words = np.arange(N * K // 8, dtype=np.uint32).reshape(N, K // 8)  # value = n * 32 + w
    flat = O.tile_words(words, 16)
    assert flat[0] == 0                      # row 0, word 0
    assert flat[15] == 15                    # row 0, word 15 (end of its first tile row)
    assert flat[16] == 32                    # row 1, word 0
    assert flat[255] == 15 * 32 + 15         # row 15, word 15: end of tile (block 0, run 0)
    assert flat[256] == 16                   # row 0, word 16: tile (block 0, run 1)
    assert flat[512] == 16 * 32              # row 16, word 0: tile (block 1, run 0)
    assert flat[788] == 17 * 32 + 20         # row 17, word 20: ((1 * 2 + 1) * 256) + 1 * 16 + 4
    np.testing.assert_array_equal(O.untile_words(flat, N, K // 8, 16), words)
    q2 = np.arange(N * K // 16, dtype=np.uint32).reshape(N, K // 16)  # 8 words a tile row
    f2 = O.tile_words(q2, 8)
    assert f2[8] == 16 and f2[128] == 8 and f2[256] == 16 * 16
    np.testing.assert_array_equal(O.untile_words(f2, N, K // 16, 8), q2)

