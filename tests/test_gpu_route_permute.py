"""The front of the layer in one call (moe_route_permute): router, optional
bit-width gate (D2MoE, Dual Routing) or given widths, and the permutation
(Read-ME, expert-aware batching).  The smallest batches run as one cluster
launch; every output must equal the separate calls' (moe_route_topk,
moe_bit_gate, moe_permute) bit for bit and the oracle's where it defines
them: ids, widths, counts, offsets, perm, inv_perm and x_perm exactly,
gates within the gate tolerance."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq

from gpu_helpers import GATE_ATOL, GATE_RTOL

pytestmark = pytest.mark.gpu

KEYS = ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm", "x_perm")


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()
    moeq.moe_debug_route_fused(1)


def _separate(x, wr, bias, k, forced=None, bits=None, w_bit=None, bias_bit=None):
    idx, w = moeq.moe_route_topk(x, wr, bias, k, forced_idx=forced)
    if w_bit is not None:
        bits = moeq.moe_bit_gate(x, w_bit, bias_bit, idx)
    out = moeq.moe_permute(idx, wr.shape[0], bits=bits, x=x)
    out.update(topk_idx=idx, topk_w=w, bits=bits)
    return out


# one cluster launch: olmoe 1-8, mixtral 1-8, tiny 8, nested 1-8 (with the gate 1-8);
# separate launches: olmoe 256, nested 16
CASES = [("olmoe", 1, "int4"), ("olmoe", 2, "int4"), ("mixtral", 1, "int4"), ("mixtral", 8, "int4"),
         ("tiny", 8, "int4"), ("nested", 1, "bits"), ("nested", 8, "bits"), ("nested", 1, "gate"),
         ("nested", 8, "gate"), ("nested", 16, "gate"), ("olmoe", 8, "int4"), ("olmoe", 256, "int4")]


@pytest.mark.parametrize("name,T,mode", CASES)
def test_route_permute_equals_separate_calls_and_oracle(name, T, mode):
    shape = I.SHAPES[name]
    L = I.make_layer(shape, T, seed=41, weights=False)
    x, wr = L["x"].cuda(), L["w_router"].cuda()
    bias = L["bias"].cuda() if L["bias"] is not None else None
    bits = G = None
    if mode == "bits":
        gen = torch.Generator().manual_seed(42)
        bits = I.draw_bits(T, shape.k, gen, "cpu").cuda()
    if mode == "gate":
        G = I.make_bit_gate(shape, seed=43, bias=True)
    w_bit = None if G is None else G["w_bit"].cuda()
    bias_bit = None if G is None else G["bias_bit"].cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fused = moeq.moe_route_permute(x, wr, bias, shape.k, bits=bits, w_bit=w_bit, bias_bit=bias_bit, status=status)
    sep = _separate(x, wr, bias, shape.k, bits=bits, w_bit=w_bit, bias_bit=bias_bit)
    torch.cuda.synchronize()
    for key in KEYS:
        assert torch.equal(fused[key], sep[key]), key
    if mode == "gate":
        assert torch.equal(fused["bits"], sep["bits"])
    assert int(status.item()) == 0
    # against the oracle
    sel, gates, _ = O.route(L["x"].float().numpy(), L["w_router"].numpy(),
                            None if L["bias"] is None else L["bias"].numpy(), shape.k)
    np.testing.assert_array_equal(fused["topk_idx"].cpu().numpy(), sel)
    np.testing.assert_allclose(fused["topk_w"].cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)
    b_ref = None
    if mode == "bits":
        b_ref = bits.cpu().numpy()
    if mode == "gate":
        b_ref = O.bit_gate(L["x"].float().numpy(), G["w_bit"].numpy(), G["bias_bit"].numpy(), sel)
        np.testing.assert_array_equal(fused["bits"].cpu().numpy(), b_ref)
    keys, mult = O.assignment_keys(sel, b_ref)
    counts, offsets, perm, inv = O.permute(keys, shape.E * (mult or 1))
    np.testing.assert_array_equal(fused["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(fused["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(fused["perm"].cpu().numpy(), perm)
    np.testing.assert_array_equal(fused["inv_perm"].cpu().numpy(), inv)
    np.testing.assert_array_equal(fused["x_perm"].cpu().numpy(),
                                  L["x"][torch.from_numpy(perm // shape.k).long()].to(torch.float16).numpy())


def test_route_permute_forced_ids_and_exact_ties():
    """Forced ids (offload traces) and duplicated router rows (exact ties to
    the lower index) through the one-launch path."""
    shape = I.SHAPES["olmoe"]
    T = 2
    L = I.make_layer(shape, T, seed=44, weights=False)
    wr = L["w_router"].clone()
    wr[5] = wr[2]
    wr[7] = wr[0]
    x, wr_d = L["x"].cuda(), wr.cuda()
    bias = L["bias"].cuda()
    fused = moeq.moe_route_permute(x, wr_d, bias, shape.k)
    sep = _separate(x, wr_d, bias, shape.k)
    torch.cuda.synchronize()
    for key in KEYS:
        assert torch.equal(fused[key], sep[key]), key
    sel, _, _ = O.route(L["x"].float().numpy(), wr.numpy(), L["bias"].numpy(), shape.k)
    np.testing.assert_array_equal(fused["topk_idx"].cpu().numpy(), sel)
    forced = torch.from_numpy(np.stack([np.random.default_rng(t).permutation(shape.E)[:shape.k]
                                        for t in range(T)]).astype(np.int32)).cuda()
    f2 = moeq.moe_route_permute(x, wr_d, bias, shape.k, forced_idx=forced)
    s2 = _separate(x, wr_d, bias, shape.k, forced=forced)
    torch.cuda.synchronize()
    for key in KEYS:
        assert torch.equal(f2[key], s2[key]), key
    assert torch.equal(f2["topk_idx"], forced)


def test_route_permute_flags_and_argument_errors():
    """Widths out of {2,3,4} are clamped and flagged, activations beyond the
    fp16 range flagged, on the one-launch path; widths and a bit gate
    together are refused."""
    shape = I.SHAPES["tiny"]
    T = 4
    L = I.make_layer(shape, T, seed=45, weights=False)
    x = L["x"].clone()
    x[1, 3] = 1e5
    bits = torch.tensor([[2, 5], [3, 1], [4, 4], [2, 3]], dtype=torch.uint8).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moeq.moe_route_permute(x.cuda(), L["w_router"].cuda(), None, shape.k, bits=bits, status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st & moeq.DEV_BAD_INDEX and st & moeq.DEV_RANGE
    clamped = bits.cpu().numpy().clip(2, 4)
    sel = out["topk_idx"].cpu().numpy()
    keys, mult = O.assignment_keys(sel, clamped)
    _, _, perm, _ = O.permute(keys, shape.E * mult)
    np.testing.assert_array_equal(out["perm"].cpu().numpy(), perm)
    G = I.make_bit_gate(shape, seed=46)
    with pytest.raises(moeq.MoeError) as ei:
        moeq.moe_route_permute(x.cuda(), L["w_router"].cuda(), None, shape.k, bits=bits, w_bit=G["w_bit"].cuda())
    assert ei.value.code == 1


@pytest.mark.parametrize("T", [1, 2, 8])
def test_route_permute_gate_ties_on_open_tokens(T):
    """Exact ties everywhere the one-launch path has a fallback: router rows
    of experts 2 and 5 (and 0 and 7) identical, so tokens whose picks or
    cut involve them are decided on fp64 logits; bit-gate rows of widths 3
    and 4 identical for every expert (width 2 far below), so every width is
    a tie that must go to the narrower width, including for the assignments
    of those tokens.  Ids, widths and the permutation equal the oracle's."""
    shape = I.SHAPES["nested"]
    L = I.make_layer(shape, T, seed=47, weights=False)
    wr = L["w_router"].clone()
    wr[5] = wr[2]
    wr[7] = wr[0]
    G = I.make_bit_gate(shape, seed=48, bias=True)
    wb, bb = G["w_bit"].clone(), G["bias_bit"].clone()
    wb[:, 2] = wb[:, 1]
    bb[:, 2] = bb[:, 1]
    bb[:, 0] = -10.0
    x = L["x"].cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moeq.moe_route_permute(x, wr.cuda(), None, shape.k, w_bit=wb.cuda(), bias_bit=bb.cuda(), status=status)
    sep = _separate(x, wr.cuda(), None, shape.k, w_bit=wb.cuda(), bias_bit=bb.cuda())
    torch.cuda.synchronize()
    sel, _, _ = O.route(L["x"].float().numpy(), wr.numpy(), None, shape.k)
    np.testing.assert_array_equal(out["topk_idx"].cpu().numpy(), sel)
    b_ref = O.bit_gate(L["x"].float().numpy(), wb.numpy(), bb.numpy(), sel)
    assert (b_ref == 3).all()
    np.testing.assert_array_equal(out["bits"].cpu().numpy(), b_ref)
    for key in KEYS:
        assert torch.equal(out[key], sep[key]), key
    assert int(status.item()) == 0


# (E, T, gate): weight rows (E, or 4 E with the gate) against the 64 lane groups
# of the one-launch kernel's dot products -- one token per group (item by item),
# several tokens per group in one or more token chunks (row by row), rows that
# do not divide the groups, more rows than groups
ROW_CASES = [(32, 8, False), (24, 8, False), (40, 8, False), (64, 5, False), (100, 5, False), (16, 8, False),
             (8, 8, True), (16, 8, True), (4, 8, True), (12, 6, True)]


@pytest.mark.parametrize("E,T,gate", ROW_CASES)
def test_route_permute_dot_product_forms(E, T, gate):
    """Every shape of the one-launch kernel's fp32 dot products (item by item,
    or row by row with token chunks): ids, widths and the permutation equal
    the separate calls' and the oracle's, gates within the gate tolerance."""
    shape = I.custom_shape(d=256, E=E, k=2, F=256, group=64, layout="planes" if gate else "int4")
    L = I.make_layer(shape, T, seed=60 + E + T, weights=False)
    x, wr = L["x"].cuda(), L["w_router"].cuda()
    bias = torch.randn(E, generator=torch.Generator().manual_seed(E)).cuda() * 0.5
    G = I.make_bit_gate(shape, seed=61 + E, bias=True) if gate else None
    w_bit = None if G is None else G["w_bit"].cuda()
    bias_bit = None if G is None else G["bias_bit"].cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fused = moeq.moe_route_permute(x, wr, bias, shape.k, w_bit=w_bit, bias_bit=bias_bit, status=status)
    sep = _separate(x, wr, bias, shape.k, w_bit=w_bit, bias_bit=bias_bit)
    torch.cuda.synchronize()
    for key in KEYS:
        assert torch.equal(fused[key], sep[key]), key
    assert int(status.item()) == 0
    sel, gates, _ = O.route(L["x"].float().numpy(), L["w_router"].numpy(), bias.cpu().numpy(), shape.k)
    np.testing.assert_array_equal(fused["topk_idx"].cpu().numpy(), sel)
    np.testing.assert_allclose(fused["topk_w"].cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)
    b_ref = None
    if gate:
        assert torch.equal(fused["bits"], sep["bits"])
        b_ref = O.bit_gate(L["x"].float().numpy(), G["w_bit"].numpy(), G["bias_bit"].numpy(), sel)
        np.testing.assert_array_equal(fused["bits"].cpu().numpy(), b_ref)
    keys, mult = O.assignment_keys(sel, b_ref)
    _, offsets, perm, _ = O.permute(keys, shape.E * (mult or 1))
    np.testing.assert_array_equal(fused["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(fused["perm"].cpu().numpy(), perm)
