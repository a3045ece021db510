"""Pins for the oracle's router, permutation, expert FFN and combine.

Sources: ExactMoE (the router's choices are executed exactly; every chosen
expert runs; experts are executed grouped), D2MoE (Dual Routing: x -> Expert
Gate -> E_i; per-token bit width), Read-ME (expert-aware batching).  Pins:
brute force over all k-subsets, a library softmax, numpy's stable argsort
(a textbook routine the oracle does not use), a dense all-experts
evaluation, a torch float64 SwiGLU for E = k = 1, and zero special cases.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from quantized_moe_expert_histogram_b200 import inputs as I


def _brute_topk(l, k):
    E = l.size
    best, best_sum = None, None
    for sub in itertools.combinations(range(E), k):  # lexicographic order
        s = math.fsum(l[i] for i in sub)  # correctly rounded: equal multisets tie exactly
        if best_sum is None or s > best_sum:
            best, best_sum = sub, s
    return sorted(best, key=lambda e: (-l[e], e))


@pytest.mark.parametrize("E,k", [(4, 1), (6, 2), (8, 2), (8, 3), (8, 8), (5, 4)])
def test_topk_brute_force(E, k):
    rng = np.random.default_rng(E * 10 + k)
    l = rng.normal(0, 1, (200, E))
    # inject exact ties: duplicate columns and repeated values
    l[:50, E - 1] = l[:50, 0]
    l[50:80, 1] = l[50:80, E // 2]
    sel = O.topk_select(l, k)
    for t in range(l.shape[0]):
        assert list(sel[t]) == _brute_topk(l[t], k), t


def test_topk_ties_lowest_index():
    l = np.array([[1.0, 3.0, 3.0, 0.5, 3.0]])
    assert O.topk_select(l, 1).tolist() == [[1]]
    assert O.topk_select(l, 2).tolist() == [[1, 2]]
    assert O.topk_select(l, 4).tolist() == [[1, 2, 4, 0]]
    assert O.topk_select(l, 5).tolist() == [[1, 2, 4, 0, 3]]


def test_gates_library_softmax_and_sum():
    rng = np.random.default_rng(7)
    l = rng.normal(0, 2, (300, 16))
    sel = O.topk_select(l, 4)
    g = O.gates_for(l, sel)
    full = torch.softmax(torch.from_numpy(l), dim=1).numpy()
    picked = np.take_along_axis(full, sel.astype(np.int64), 1)
    ref = picked / picked.sum(1, keepdims=True)
    np.testing.assert_allclose(g, ref, rtol=1e-6, atol=1e-7)
    assert np.abs(g.sum(1) - 1).max() < 1e-6
    # hand value: logits (0, ln 3) -> gates (1/4, 3/4)
    g2 = O.gates_for(np.array([[0.0, math.log(3.0), -5.0]]), np.array([[1, 0]]))
    np.testing.assert_allclose(g2, [[0.75, 0.25]], rtol=1e-7)


def test_router_logits_exact_products():
    # bf16 x times fp32 W_r is exact in fp64; check one hand case
    x = np.array([[1.5, -2.0, 0.25]], np.float32)
    w = np.array([[0.5, 0.25, 4.0], [1.0, 1.0, 1.0]], np.float32)
    l = O.router_logits(x, w, np.array([0.125, -1.0], np.float32))
    assert l.tolist() == [[0.75 - 0.5 + 1.0 + 0.125, 1.5 - 2.0 + 0.25 - 1.0]]


def test_permute_matches_stable_argsort():
    rng = np.random.default_rng(8)
    for n, nb in ((1, 1), (17, 4), (1000, 64), (4096, 24), (333, 3)):
        keys = rng.integers(0, nb, n)
        if n > 10:
            keys[: n // 3] = nb - 1  # one heavy bin
        counts, offsets, perm, inv = O.permute(keys, nb)
        np.testing.assert_array_equal(counts, np.bincount(keys, minlength=nb))
        np.testing.assert_array_equal(perm, np.argsort(keys, kind="stable"))
        assert offsets[0] == 0 and offsets[-1] == n
        np.testing.assert_array_equal(np.diff(offsets), counts)
        np.testing.assert_array_equal(inv[perm], np.arange(n))
        assert sorted(perm.tolist()) == list(range(n))


def test_permute_hand_example():
    keys = np.array([2, 0, 2, 1, 0, 2])
    counts, offsets, perm, inv = O.permute(keys, 4)
    assert counts.tolist() == [2, 1, 3, 0]
    assert offsets.tolist() == [0, 2, 3, 6, 6]
    assert perm.tolist() == [1, 4, 3, 0, 2, 5]
    assert inv.tolist() == [3, 0, 4, 2, 1, 5]


def test_nested_keys():
    sel = np.array([[3, 0], [1, 3]])
    bits = np.array([[2, 4], [3, 2]])
    keys, mult = O.assignment_keys(sel, bits)
    assert mult == 3 and keys.tolist() == [9, 2, 4, 9]


def _small_layer(E=6, k=2, d=64, F=128, g=64, T=40, layout="int4", seed=0):
    shape = I.custom_shape(d=d, E=E, k=k, F=F, group=g, layout=layout)
    L = I.make_layer(shape, T, seed=seed)
    x = L["x"].float().numpy()
    ex = O.QuantExperts(L["w_gate"].numpy(), L["w_up"].numpy(), L["w_down"].numpy(), g)
    return shape, L, x, ex


def test_layer_equals_dense_masked_evaluation():
    shape, L, x, ex = _small_layer()
    out = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, ex)
    T = x.shape[0]
    dense = np.zeros((T, shape.d))
    for e in range(shape.E):
        wg, wu, wd = ex.weights(e)
        ye = O.expert_ffn(x.astype(np.float64), wg, wu, wd)
        gate = np.zeros(T)
        for t in range(T):
            for j in range(shape.k):
                if out["sel"][t, j] == e:
                    gate[t] = out["gates"][t, j]
        dense += gate[:, None] * ye
    np.testing.assert_allclose(out["y"], dense, rtol=1e-9, atol=1e-12)
    # every token appears exactly k times in the permutation
    np.testing.assert_array_equal(np.bincount(out["perm"] // shape.k, minlength=T), shape.k)


def test_single_expert_is_dense_swiglu_torch():
    shape, L, x, ex = _small_layer(E=1, k=1, T=16)
    out = O.moe_layer(x, L["w_router"].numpy(), None, 1, ex)
    wg, wu, wd = (torch.from_numpy(w) for w in ex.weights(0))
    xt = torch.from_numpy(x.astype(np.float64))
    ref = torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(xt, wg)) * torch.nn.functional.linear(xt, wu), wd)
    assert (out["gates"] == 1).all()
    np.testing.assert_allclose(out["y"], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_zero_special_cases():
    shape, L, x, ex = _small_layer(T=8)
    zero_x = np.zeros_like(x)
    out = O.moe_layer(zero_x, L["w_router"].numpy(), None, shape.k, ex)
    assert (out["y"] == 0).all()
    zero_w = O.QuantExperts(np.zeros((shape.E, shape.F, shape.d), np.float32),
                            np.zeros((shape.E, shape.F, shape.d), np.float32),
                            np.zeros((shape.E, shape.d, shape.F), np.float32), shape.group)
    out = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, zero_w)
    assert (out["y"] == 0).all()


def test_nested_layer_bits_select_planes():
    shape, L, x, ex = _small_layer(E=4, k=2, T=24, layout="planes")
    bits = L["bits"].numpy()
    out = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, ex, bits=bits)
    # recompute each assignment directly with its own width
    for a in range(x.shape[0] * shape.k):
        t, e, b = a // shape.k, out["sel"].reshape(-1)[a], bits.reshape(-1)[a]
        wg, wu, wd = ex.weights(int(e), int(b))
        ya = O.expert_ffn(x[t:t + 1].astype(np.float64), wg, wu, wd)[0]
        np.testing.assert_allclose(out["y_assign"][a], ya, rtol=1e-12, atol=1e-14)
    # bins are ordered key = 3e + (b - 2)
    keys = out["sel"].reshape(-1) * 3 + bits.reshape(-1) - 2
    np.testing.assert_array_equal(out["perm"], np.argsort(keys, kind="stable"))
    # b = 4 everywhere reduces to the INT4 layer
    out4 = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, ex, bits=np.full_like(bits, 4))
    outi = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, ex)
    np.testing.assert_allclose(out4["y"], outi["y"], rtol=0, atol=0)


def test_forced_selection_and_subset():
    shape, L, x, ex = _small_layer(T=12)
    sel = np.array([[t % shape.E, (t + 1) % shape.E] for t in range(12)])
    out = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, ex, sel=sel)
    assert (out["sel"] == sel).all()
    full = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, ex)
    sub = O.moe_layer(x, L["w_router"].numpy(), None, shape.k, ex, token_subset=[0, 5, 11])
    np.testing.assert_allclose(sub["y"][[0, 5, 11]], full["y"][[0, 5, 11]], rtol=1e-12, atol=1e-15)


def test_identical_router_rows_give_identical_logits():
    # duplicated router rows at full length: equal logits, so every token that
    # picks one of the pair and not the other picks the lower index
    rng = np.random.default_rng(6)
    T, E, d, k = 512, 16, 2048, 3
    w = rng.normal(0, 0.02, (E, d)).astype(np.float32)
    w[9] = w[4]
    x = rng.normal(size=(T, d)).astype(np.float32)
    l = O.router_logits(x, w)
    assert np.array_equal(l[:, 9], l[:, 4])
    sel = O.topk_select(l, k)
    one = [s for s in sel if (4 in s) != (9 in s)]
    assert one and all(4 in s for s in one)
