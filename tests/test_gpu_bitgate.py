"""GPU parity of the bit-width router (moe_bit_gate; D2MoE, Dual Routing:
the bit gate beside the expert gate) against the oracle's bit_gate: widths
bit for bit, including near-tied and exactly tied width scores, and the
nested-plane layer run end to end on gate-chosen widths."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq
from quantized_moe_expert_histogram_b200.layer import QuantMoELayer

from gpu_helpers import oracle_layer, within_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()
    moeq.moe_debug_force_regime(0)


def _oracle_sel(L, shape):
    bias = L["bias"].numpy() if L["bias"] is not None else None
    sel, _, _ = O.route(L["x"].float().numpy(), L["w_router"].numpy(), bias, shape.k)
    return sel


@pytest.mark.parametrize("name,T,with_bias", [("nested", 300, False), ("nested", 1, True),
                                               ("nested", 16, False), ("olmoe", 8, True),
                                               ("mixtral", 1, False), ("olmoe", 256, True),
                                               ("tiny", 64, False), ("mixtral", 33, True)])
def test_bit_gate_bitexact(name, T, with_bias):
    """Widths bit for bit against the oracle: up to 32 assignments through the
    fp64 cluster kernel, beyond through the fp32-with-bound kernel."""
    shape = I.SHAPES[name]
    L = I.make_layer(shape, T, seed=21, weights=False)
    G = I.make_bit_gate(shape, seed=22, bias=with_bias)
    sel = _oracle_sel(L, shape)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bits = moeq.moe_bit_gate(L["x"].cuda(), G["w_bit"].cuda(),
                             None if G["bias_bit"] is None else G["bias_bit"].cuda(),
                             torch.from_numpy(sel).cuda(), status=status)
    torch.cuda.synchronize()
    ref = O.bit_gate(L["x"].float().numpy(), G["w_bit"].numpy(),
                     None if G["bias_bit"] is None else G["bias_bit"].numpy(), sel)
    np.testing.assert_array_equal(bits.cpu().numpy(), ref)
    assert int(status.item()) == 0
    if T >= 64:
        assert set(np.unique(ref).tolist()) == {2, 3, 4}


@pytest.mark.parametrize("T", [200, 8])
@pytest.mark.parametrize("scale", [0.0, 1e-9, 1e-7, 1e-5])
def test_bit_gate_near_ties_resolved_exactly(scale, T):
    """Width rows that are copies of each other plus a perturbation of the
    given size: the scores of the pair differ by about scale * |x| (exact ties
    at 0, which go to the narrower width), below what fp32 scores can order,
    so these assignments take the fp64 re-evaluation (200 tokens) or the fp64
    cluster kernel (8 tokens, 32 assignments) and must still match the
    oracle."""
    shape = I.SHAPES["nested"]
    L = I.make_layer(shape, T, seed=23, weights=False)
    G = I.make_bit_gate(shape, seed=24, bias=True)
    w = G["w_bit"].clone()
    b = G["bias_bit"].clone()
    rng = np.random.default_rng(3)
    for e in range(shape.E):
        src, dst = (0, 1) if e % 2 else (1, 2)
        w[e, dst] = w[e, src] + torch.from_numpy((rng.standard_normal(shape.d) * scale).astype(np.float32))
        b[e, dst] = b[e, src]
        b[e, 3 - src - dst] = -10.0  # the third width never wins
    sel = _oracle_sel(L, shape)
    bits = moeq.moe_bit_gate(L["x"].cuda(), w.cuda(), b.cuda(), torch.from_numpy(sel).cuda())
    torch.cuda.synchronize()
    ref = O.bit_gate(L["x"].float().numpy(), w.numpy(), b.numpy(), sel)
    np.testing.assert_array_equal(bits.cpu().numpy(), ref)
    if scale == 0.0:  # exact ties everywhere: always the narrower of the pair
        narrower = np.where(sel % 2 == 1, 2, 3)
        np.testing.assert_array_equal(ref, narrower)


@pytest.mark.parametrize("mode", [1, 0])
def test_bit_gate_flags_bad_ids(mode):
    """Out-of-range ids are flagged and clamped, by the fp64 cluster kernel
    (mode 1, the default at this size) and the fp32 kernel (mode 0)."""
    moeq.moe_debug_route_fused(mode)
    try:
        _bad_ids_case()
    finally:
        moeq.moe_debug_route_fused(1)


@pytest.mark.parametrize("name,T", [("nested", 1), ("nested", 16), ("mixtral", 8), ("olmoe", 8)])
def test_bit_gate_small_paths_agree(name, T):
    """The fp64 cluster kernel (default up to 32 assignments) and the
    fp32-with-bound kernel (test hook mode 0) give the same widths, which are
    the oracle's."""
    shape = I.SHAPES[name]
    L = I.make_layer(shape, T, seed=27, weights=False)
    G = I.make_bit_gate(shape, seed=28, bias=True)
    sel = _oracle_sel(L, shape)
    args = (L["x"].cuda(), G["w_bit"].cuda(), G["bias_bit"].cuda(), torch.from_numpy(sel).cuda())
    b1 = moeq.moe_bit_gate(*args)
    moeq.moe_debug_route_fused(0)
    try:
        b2 = moeq.moe_bit_gate(*args)
    finally:
        moeq.moe_debug_route_fused(1)
    torch.cuda.synchronize()
    ref = O.bit_gate(L["x"].float().numpy(), G["w_bit"].numpy(), G["bias_bit"].numpy(), sel)
    np.testing.assert_array_equal(b1.cpu().numpy(), ref)
    np.testing.assert_array_equal(b2.cpu().numpy(), ref)


def _bad_ids_case():
    shape = I.SHAPES["tiny"]
    L = I.make_layer(shape, 4, seed=1, weights=False)
    G = I.make_bit_gate(shape, seed=2)
    idx = torch.tensor([[0, 9], [3, -1], [1, 2], [7, 6]], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bits = moeq.moe_bit_gate(L["x"].cuda(), G["w_bit"].cuda(), None, idx, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & moeq.DEV_BAD_INDEX
    clamped = np.array([[0, 7], [3, 0], [1, 2], [7, 6]], dtype=np.int32)
    np.testing.assert_array_equal(bits.cpu().numpy(),
                                  O.bit_gate(L["x"].float().numpy(), G["w_bit"].numpy(), None, clamped))


@pytest.mark.parametrize("T", [1, 8, 64])
def test_nested_layer_with_gate_chosen_widths(T):
    """The whole nested-plane layer with the widths taken from the bit gate on
    the device: ids, widths, (expert, width) bins and permutation bit for
    bit; outputs within the layer's bar against the oracle at those widths."""
    shape = I.SHAPES["nested"]
    L = I.make_layer(shape, T, seed=25)
    G = I.make_bit_gate(shape, seed=26, bias=True)
    layer = QuantMoELayer.from_weights(shape, L["w_router"].cuda(), None, L["w_gate"].cuda(), L["w_up"].cuda(),
                                       L["w_down"].cuda(), max_tokens=T)
    layer.w_bit, layer.bias_bit = G["w_bit"].cuda(), G["bias_bit"].cuda()
    layer.buf["status"].zero_()
    y = layer.forward(L["x"].cuda()).float().cpu().numpy()
    torch.cuda.synchronize()
    v = layer.views(T)
    sel = _oracle_sel(L, shape)
    bits_ref = O.bit_gate(L["x"].float().numpy(), G["w_bit"].numpy(), G["bias_bit"].numpy(), sel)
    np.testing.assert_array_equal(v["topk_idx"].cpu().numpy(), sel)
    np.testing.assert_array_equal(v["bits"].cpu().numpy(), bits_ref)
    ref, _ = oracle_layer(shape, L, bits=torch.from_numpy(bits_ref))
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(v["perm"].cpu().numpy(), ref["perm"])
    ok, worst = within_tol(y, ref["y"])
    assert ok, f"worst err/tol = {worst:.3f}"
    assert int(v["status"].item()) == 0
