"""GPU parity: every call of the C ABI against the oracle on the same seeded
inputs.  Integer and index outputs (codes, expert ids, counts, offsets,
permutations) must match bit for bit; floating outputs must satisfy
|y - y_ref| <= 1e-2 + 1e-2 |y_ref| against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq

from gpu_helpers import gpu_layer, layer_inputs, oracle_layer, run_gpu_layer, within_tol, GATE_RTOL, GATE_ATOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()


# ---------------------------------------------------------------- pack ----

@pytest.mark.parametrize("d,F,g,layout,E", [(256, 512, 64, "int4", 3), (256, 384, 64, "planes", 2),
                                            (2048, 1024, 128, "int4", 2), (4096, 1024, 128, "planes", 1)])
def test_pack_bitexact(d, F, g, layout, E):
    shape = I.custom_shape(d=d, E=E, k=1, F=F, group=g, layout=layout)
    L = I.make_layer(shape, 1, seed=11)
    # a few special groups: all zero, all positive, all negative, constant
    L["w_gate"][0, 0, :g] = 0
    L["w_gate"][0, 1, :g] = L["w_gate"][0, 1, :g].abs()
    L["w_up"][0, 2, :g] = -L["w_up"][0, 2, :g].abs()
    L["w_down"][0, 3, :g] = 0.37
    lay = moeq.LAYOUT_PLANES if layout == "planes" else moeq.LAYOUT_INT4
    blobs = moeq.moe_quant_pack(L["w_gate"].cuda(), L["w_up"].cuda(), L["w_down"].cuda(), g, lay)
    torch.cuda.synchronize()
    got = blobs.cpu().numpy()
    for e in range(E):
        ref = O.build_blob(L["w_gate"][e].numpy(), L["w_up"][e].numpy(), L["w_down"][e].numpy(), g, layout)
        assert got[e].size == ref.size
        diff = np.nonzero(got[e] != ref)[0]
        assert diff.size == 0, f"expert {e}: {diff.size} bytes differ, first at {diff[:5]}"


# --------------------------------------------------------------- route ----

@pytest.mark.parametrize("name,T,dup", [("tiny", 64, False), ("olmoe", 256, False), ("olmoe", 1, False),
                                        ("mixtral", 32, False), ("tiny", 100, True),
                                        ("nested", 77, False)])
def test_route_bitexact(name, T, dup):
    shape = I.SHAPES[name]
    L = I.make_layer(shape, T, seed=3, weights=False)
    if dup:  # exact ties: identical router rows must resolve to the lower index
        L["w_router"][5] = L["w_router"][2]
        L["w_router"][7] = L["w_router"][0]
    bias = L["bias"].cuda() if L["bias"] is not None else None
    idx, w = moeq.moe_route_topk(L["x"].cuda(), L["w_router"].cuda(), bias, shape.k)
    torch.cuda.synchronize()
    sel, gates, logits = O.route(L["x"].float().numpy(), L["w_router"].numpy(),
                                 None if L["bias"] is None else L["bias"].numpy(), shape.k)
    np.testing.assert_array_equal(idx.cpu().numpy(), sel)
    np.testing.assert_allclose(w.cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)


@pytest.mark.parametrize("E,k", [(1, 1), (5, 5), (31, 4), (32, 16), (33, 8), (64, 8), (65, 2), (100, 16),
                                 (128, 7), (129, 8), (200, 1), (256, 16)])
def test_route_every_expert_count_per_lane(E, k):
    """The two-launch router's select kernel is built for 1, 2, 4 and 8
    experts per lane (E up to 32, 64, 128, 256): ids bit-exact and gates
    within the bar against the oracle at each, across the boundaries, with
    k = E, k = 16 (the largest), exact ties (duplicated router rows) and
    forced ids."""
    shape = I.custom_shape(d=256, E=E, k=k, F=256, group=64)
    T = 40  # above the one-launch sizes
    L = I.make_layer(shape, T, seed=E + 100 * k, weights=False)
    w = L["w_router"].clone()
    if E >= 8:
        w[E - 1] = w[1]
        w[E // 2] = w[0]
    b = None  # a bias on every other count (the duplicated rows keep equal biases)
    if E % 2 == 0:
        b = torch.randn(E, generator=torch.Generator().manual_seed(E)) * 0.5
        if E >= 8:
            b[E - 1] = b[1]
            b[E // 2] = b[0]
    bias = b.cuda() if b is not None else None
    idx, gw = moeq.moe_route_topk(L["x"].cuda(), w.cuda(), bias, k)
    torch.cuda.synchronize()
    sel, gates, _ = O.route(L["x"].float().numpy(), w.numpy(), None if b is None else b.numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), sel)
    np.testing.assert_allclose(gw.cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)
    rng = np.random.default_rng(E)
    forced = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx2, gw2 = moeq.moe_route_topk(L["x"].cuda(), w.cuda(), bias, k, forced_idx=torch.from_numpy(forced).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx2.cpu().numpy(), forced)
    logits = L["x"].double().numpy() @ w.double().numpy().T + (0 if b is None else b.double().numpy())
    lf = np.take_along_axis(logits, forced.astype(np.int64), axis=1)
    ref = np.exp(lf - lf.max(axis=1, keepdims=True))
    ref /= ref.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(gw2.cpu().numpy(), ref, rtol=GATE_RTOL, atol=GATE_ATOL)


@pytest.mark.parametrize("name,T", [("olmoe", 1), ("olmoe", 2), ("olmoe", 8), ("olmoe", 33), ("nested", 1),
                                    ("nested", 8), ("nested", 17), ("mixtral", 1), ("mixtral", 8), ("tiny", 16),
                                    ("tiny", 64)])
def test_route_fused_small_batches(name, T):
    """The smallest batches run the router as one cluster launch on fp64
    logits; at every size its expert ids equal the fp32-with-bound two-launch
    router's and the oracle's bit for bit, and the gates match the
    oracle's."""
    shape = I.SHAPES[name]
    L = I.make_layer(shape, T, seed=17, weights=False)
    bias = L["bias"].cuda() if L["bias"] is not None else None
    x, wr = L["x"].cuda(), L["w_router"].cuda()
    idx_f, w_f = moeq.moe_route_topk(x, wr, bias, shape.k)
    others = []
    for mode in (0,):  # the fp32-with-bound two-launch router
        moeq.moe_debug_route_fused(mode)
        try:
            others.append(moeq.moe_route_topk(x, wr, bias, shape.k))
        finally:
            moeq.moe_debug_route_fused(1)
    torch.cuda.synchronize()
    sel, gates, _ = O.route(L["x"].float().numpy(), L["w_router"].numpy(),
                            None if L["bias"] is None else L["bias"].numpy(), shape.k)
    np.testing.assert_array_equal(idx_f.cpu().numpy(), sel)
    np.testing.assert_allclose(w_f.cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)
    for idx_o, w_o in others:
        np.testing.assert_array_equal(idx_o.cpu().numpy(), sel)
        np.testing.assert_allclose(w_o.cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)


@pytest.mark.parametrize("T", [300, 2])
@pytest.mark.parametrize("scale", [0.0, 1e-9, 1e-7, 1e-5])
def test_route_near_ties_resolved_exactly(scale, T):
    """Router rows that are copies of others plus a perturbation of the given
    size: the logits of the pairs differ by about scale * |x| (exact ties at
    0), below what fp32 logits can order, so these tokens must take the fp64
    re-evaluation (300 tokens) or be decided on fp64 logits (2 tokens, the
    cluster path) and still match the oracle's choice and order exactly."""
    shape = I.SHAPES["olmoe"]
    L = I.make_layer(shape, T, seed=9, weights=False)
    w = L["w_router"].clone()
    b = L["bias"].clone()
    rng = np.random.default_rng(1)
    for a, src in ((1, 0), (9, 4), (33, 17), (63, 62), (2, 0)):
        w[a] = w[src] + torch.from_numpy((rng.standard_normal(shape.d) * scale).astype(np.float32))
        b[a] = b[src]
    idx, gw = moeq.moe_route_topk(L["x"].cuda(), w.cuda(), b.cuda(), shape.k)
    torch.cuda.synchronize()
    sel, gates, _ = O.route(L["x"].float().numpy(), w.numpy(), b.numpy(), shape.k)
    np.testing.assert_array_equal(idx.cpu().numpy(), sel)
    np.testing.assert_allclose(gw.cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)
    # the pairs really are near-tied inside many tokens' picks
    both = sum(int((s == 0).any() and (s == 1).any()) for s in sel)
    assert both > 10 or T < 100


def test_route_k_equals_E_and_forced():
    shape = I.custom_shape(d=256, E=8, k=8, F=512, group=64)
    L = I.make_layer(shape, 40, seed=4, weights=False)
    idx, w = moeq.moe_route_topk(L["x"].cuda(), L["w_router"].cuda(), None, 8)
    sel, gates, logits = O.route(L["x"].float().numpy(), L["w_router"].numpy(), None, 8)
    np.testing.assert_array_equal(idx.cpu().numpy(), sel)
    forced = torch.tensor(np.stack([np.random.default_rng(t).permutation(8)[:3] for t in range(40)]),
                          dtype=torch.int32)
    idx3, w3 = moeq.moe_route_topk(L["x"].cuda(), L["w_router"].cuda(), None, 3, forced_idx=forced.cuda())
    np.testing.assert_array_equal(idx3.cpu().numpy(), forced.numpy())
    np.testing.assert_allclose(w3.cpu().numpy(), O.gates_for(logits, forced.numpy()), rtol=GATE_RTOL, atol=GATE_ATOL)
    # a decode-sized batch (fp64 cluster path): forced ids and their gates
    idx4, w4 = moeq.moe_route_topk(L["x"][:4].cuda(), L["w_router"].cuda(), None, 3, forced_idx=forced[:4].cuda())
    np.testing.assert_array_equal(idx4.cpu().numpy(), forced[:4].numpy())
    np.testing.assert_allclose(w4.cpu().numpy(), O.gates_for(logits[:4], forced[:4].numpy()), rtol=GATE_RTOL,
                               atol=GATE_ATOL)


# ------------------------------------------------------------- permute ----

@pytest.mark.parametrize("T,k,E,nested,skew,d", [(1, 2, 8, False, False, 64), (33, 2, 8, False, True, 64),
                                                  (4096, 8, 64, False, True, 64), (777, 4, 16, True, False, 64),
                                                  (100, 3, 256, True, True, 64), (5, 8, 8, False, False, 64),
                                                  # many 1024-assignment blocks, ragged last block, wide rows
                                                  (2049, 8, 64, False, True, 2056),
                                                  # the largest bin count (3 * 256) over several blocks
                                                  (3001, 4, 256, True, True, 8),
                                                  # exactly one full block (single-launch path), one past it
                                                  (128, 8, 64, False, True, 64), (129, 8, 64, False, True, 64)])
def test_permute_bitexact(T, k, E, nested, skew, d):
    rng = np.random.default_rng(T * 7 + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    if skew:
        idx[: T // 2, 0] = 0
    bits = rng.choice([2, 3, 4], size=(T, k), p=[.3, .4, .3]).astype(np.uint8) if nested else None
    x = torch.randn(T, d).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moeq.moe_permute(torch.from_numpy(idx).cuda(), E,
                           bits=None if bits is None else torch.from_numpy(bits).cuda(), x=x.cuda(),
                           status=status)
    torch.cuda.synchronize()
    keys, mult = O.assignment_keys(idx, bits)
    counts, offsets, perm, inv = O.permute(keys, E * (mult or 1))
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(out["perm"].cpu().numpy(), perm)
    np.testing.assert_array_equal(out["inv_perm"].cpu().numpy(), inv)
    xp = out["x_perm"].cpu()
    np.testing.assert_array_equal(xp.numpy(), x[torch.from_numpy(perm // k).long()].to(torch.float16).numpy())
    assert int(status.item()) == 0


def test_permute_flags_bad_ids_and_range():
    idx = torch.tensor([[0, 9], [3, -1]], dtype=torch.int32).cuda()
    x = torch.tensor([[1.0] * 8, [1e5] * 8]).to(torch.bfloat16).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moeq.moe_permute(idx, 4, x=x, status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st & moeq.DEV_BAD_INDEX and st & moeq.DEV_RANGE
    # clamped ids still give a valid permutation
    assert sorted(out["perm"].cpu().tolist()) == [0, 1, 2, 3]


# --------------------------------------------------------------- layer ----

def _check_layer(shape, T, seed=0, token_subset=None):
    L = layer_inputs(shape, T, seed=seed)
    layer = gpu_layer(shape, L, T)
    bits = L.get("bits")
    v, y = run_gpu_layer(layer, L, T, bits=bits)
    ref, _ = oracle_layer(shape, L, bits=bits, token_subset=token_subset)
    np.testing.assert_array_equal(v["topk_idx"].cpu().numpy(), ref["sel"])
    np.testing.assert_array_equal(v["perm"].cpu().numpy(), ref["perm"])
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), ref["offsets"])
    toks = ref["tokens"]
    ok, worst = within_tol(y[toks], ref["y"][toks])
    assert ok, f"worst err/tol = {worst:.3f}"
    # per-assignment expert outputs (before the combine)
    yp = v["y_perm"].float().cpu().numpy()
    rows = np.array([a for t in toks for a in range(t * shape.k, (t + 1) * shape.k)])
    ok2, worst2 = within_tol(yp[ref["inv_perm"][rows]], ref["y_assign"][rows])
    assert ok2, f"y_perm worst err/tol = {worst2:.3f}"
    assert int(v["status"].item()) == 0
    return worst, worst2


@pytest.mark.parametrize("name,T", [("tiny", 64), ("olmoe", 1), ("olmoe", 16), ("nested", 1),
                                    ("nested", 64)])
def test_layer_parity(name, T):
    _check_layer(I.SHAPES[name], T)


@pytest.mark.parametrize("d,E,k,F,g,layout,T", [(384, 5, 3, 640, 64, "int4", 7),
                                                (128, 4, 4, 128, 64, "int4", 3),
                                                (256, 6, 2, 384, 128, "planes", 13),
                                                (1152, 12, 2, 256, 128, "int4", 2)])
def test_layer_ragged_shapes(d, E, k, F, g, layout, T):
    _check_layer(I.custom_shape(d=d, E=E, k=k, F=F, group=g, layout=layout), T, seed=5)


@pytest.mark.parametrize("layout", ["int4", "planes"])
def test_small_batch_kernel_multi_pass(layout):
    # bins of ~27 rows: the small-batch kernel runs two 16-row passes per bin
    shape = I.custom_shape(d=384, E=3, k=2, F=256, group=64, layout=layout)
    moeq.moe_debug_force_regime(3)
    try:
        _check_layer(shape, 40, seed=7)
    finally:
        moeq.moe_debug_force_regime(0)


@pytest.mark.parametrize("regime", [1, 3])
@pytest.mark.parametrize("d,E,k,F,g,layout,T", [
    (4096, 4, 2, 512, 128, "int4", 8),     # gate/up rows of K = 4096: more stages than one ring
    (4096, 4, 2, 512, 128, "planes", 8),
    (256, 2, 1, 14336, 128, "int4", 6),    # down rows of K = 14336
    (256, 3, 2, 14336, 64, "planes", 5),
    (4096, 3, 2, 256, 64, "int4", 40),     # bins above 16 rows: several passes per bin
])
def test_decode_kernels_long_rows(regime, d, E, k, F, g, layout, T):
    """The decode-regime kernels forced on (1: the one-token kernel, 3: the
    small-batch kernel) at the row lengths of the d = 4096 and d_ff = 14336
    workloads, where a row spans many shared-memory stages."""
    moeq.moe_debug_force_regime(regime)
    try:
        _check_layer(I.custom_shape(d=d, E=E, k=k, F=F, group=g, layout=layout), T, seed=13)
    finally:
        moeq.moe_debug_force_regime(0)


@pytest.mark.parametrize("T", [5, 300])
def test_static_per_expert_widths(T):
    """Static per-expert widths: bits come from moe_static_bits (width_of[e]
    for every assignment of expert e), the layer then runs the nested-plane
    path; bits bit-exact, outputs against the oracle at those widths."""
    shape = I.custom_shape(d=512, E=12, k=3, F=256, group=128, layout="planes")
    L = layer_inputs(shape, T, seed=8)
    layer = gpu_layer(shape, L, T)
    width_of = torch.tensor(np.random.default_rng(8).choice([2, 3, 4], size=shape.E).astype(np.uint8))
    x = L["x"].cuda()
    v = layer.views(T)
    moeq.moe_route_topk(x, layer.w_router, layer.bias, shape.k, topk_idx=v["topk_idx"], topk_w=v["topk_w"],
                        workspace=v["route_ws"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bits = moeq.moe_static_bits(v["topk_idx"], width_of.cuda(), shape.E, status=status)
    torch.cuda.synchronize()
    sel = v["topk_idx"].cpu().numpy()
    np.testing.assert_array_equal(bits.cpu().numpy(), width_of.numpy()[sel])
    assert int(status.item()) == 0
    _, y = run_gpu_layer(layer, L, T, bits=bits.cpu())
    ref, _ = oracle_layer(shape, L, bits=bits.cpu())
    np.testing.assert_array_equal(ref["sel"], sel)
    ok, worst = within_tol(y, ref["y"])
    assert ok, f"worst err/tol = {worst:.3f}"
    # each expert occupies exactly one (expert, width) bin: its own width
    counts = layer.views(T)["counts"].cpu().numpy().reshape(shape.E, 3)
    for e in range(shape.E):
        assert (counts[e][np.arange(3) != width_of[e].item() - 2] == 0).all()


def test_static_bits_flags_bad_widths():
    idx = torch.tensor([[0, 1], [2, 7]], dtype=torch.int32, device="cuda")
    width_of = torch.tensor([2, 5, 4, 3], dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bits = moeq.moe_static_bits(idx, width_of, 4, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & moeq.DEV_BAD_INDEX
    assert bits.cpu().tolist() == [[2, 4], [4, 3]]  # width 5 clamped to 4; id 7 clamped to 3


def test_layer_deterministic():
    shape = I.SHAPES["tiny"]
    L = layer_inputs(shape, 64)
    layer = gpu_layer(shape, L, 64)
    _, y1 = run_gpu_layer(layer, L, 64)
    _, y2 = run_gpu_layer(layer, L, 64)
    np.testing.assert_array_equal(y1, y2)


# ---------------------------------------------------------- api errors ----

def test_api_rejects_bad_arguments():
    x = torch.randn(4, 256).to(torch.bfloat16).cuda()
    wr = torch.randn(8, 256).cuda()
    with pytest.raises(moeq.MoeError) as ei:
        moeq.moe_route_topk(x, wr, None, 9)
    assert ei.value.code in (1, 2)
    xp = torch.zeros(8, 256, dtype=torch.float16, device="cuda")
    off = torch.zeros(9, dtype=torch.int32, device="cuda")
    blobs = torch.zeros(8, moeq.moe_blob_bytes(256, 512, 64, 0), dtype=torch.uint8, device="cuda")
    with pytest.raises(moeq.MoeError) as ei:
        moeq.moe_grouped_ffn_wq(xp, off, blobs, 4, 8, 256, 512, 64, 0,
                                workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert ei.value.code == 6
    with pytest.raises(moeq.MoeError) as ei:
        moeq.moe_grouped_ffn_wq(xp, off, blobs, 4, 8, 256, 500, 64, 0)
    assert ei.value.code == 2
