"""The grouped FFN and the weighted combine in one call
(moe_grouped_ffn_combine; ExactMoE: every routed expert runs exactly,
weighted by its gate): y and y_perm must equal the separate calls'
(moe_grouped_ffn_wq, then moe_unpermute_combine) bit for bit, for every
batch size and kernel (decode kernel with one or two token blocks, tensor
cores), with and without a residual, with nested widths, and when a token
names one expert twice (a bin holding more rows than there are tokens);
misaligned rows are refused."""
import numpy as np
import pytest
import torch

from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq
from quantized_moe_expert_histogram_b200.layer import QuantMoELayer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()
    moeq.moe_debug_force_regime(0)


def _run(shape, T, seed, residual=True, forced=None, bits=None):
    L = I.make_layer(shape, T, seed=seed)
    layer = QuantMoELayer.from_weights(shape, L["w_router"].cuda(), L["bias"].cuda() if L["bias"] is not None
                                       else None, L["w_gate"].cuda(), L["w_up"].cuda(), L["w_down"].cuda(),
                                       max_tokens=T)
    x = L["x"].cuda()
    if bits is None and shape.layout == "planes":
        bits = L["bits"].cuda()
    v = layer.views(T)
    moeq.moe_route_permute(x, layer.w_router, layer.bias, shape.k, forced_idx=forced, bits=bits, out=v,
                           status=v["status"], workspace=v["rp_ws"])
    res = x if residual else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y_f, yp_f = moeq.moe_grouped_ffn_combine(v["x_perm"], v["offsets"], layer.blobs, T, shape.k, shape.E, shape.d,
                                             shape.F, shape.group, layer.layout, v["perm"], v["inv_perm"],
                                             v["topk_w"], residual=res, status=status)
    yp_s = moeq.moe_grouped_ffn_wq(v["x_perm"], v["offsets"], layer.blobs, T, shape.E, shape.d, shape.F,
                                   shape.group, layer.layout, status=status).clone()
    y_s = torch.empty_like(y_f)
    moeq.moe_unpermute_combine(yp_s, v["inv_perm"], v["topk_w"], residual=res, y=y_s)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y_f, yp_f, y_s, yp_s


@pytest.mark.parametrize("name,T", [("olmoe", 1), ("olmoe", 2), ("olmoe", 8), ("olmoe", 9), ("olmoe", 16),
                                    ("mixtral", 1), ("mixtral", 8), ("nested", 1), ("nested", 4), ("nested", 16),
                                    ("tiny", 3), ("olmoe", 32), ("mixtral", 24), ("mixtral", 48), ("nested", 64)])
def test_ffn_combine_equals_separate_calls(name, T):
    shape = I.SHAPES[name]
    y_f, yp_f, y_s, yp_s = _run(shape, T, seed=61 + T)
    assert torch.equal(yp_f, yp_s)
    assert torch.equal(y_f, y_s)


def test_ffn_combine_without_residual_and_repeated_experts():
    """No residual; and forced ids where every token names its first expert
    twice, so that expert's bin holds up to 2 T rows -- more than the tokens
    in the batch -- and each token's k rows still complete exactly once."""
    shape = I.SHAPES["olmoe"]
    T = 4
    y_f, yp_f, y_s, yp_s = _run(shape, T, seed=71, residual=False)
    assert torch.equal(y_f, y_s) and torch.equal(yp_f, yp_s)
    rng = np.random.default_rng(5)
    ids = np.stack([rng.permutation(shape.E)[:shape.k] for _ in range(T)]).astype(np.int32)
    ids[:, 1] = ids[:, 0]
    ids[:, 0] = 3  # every token: expert 3 twice
    ids[:, 1] = 3
    forced = torch.from_numpy(ids).cuda()
    y_f, yp_f, y_s, yp_s = _run(shape, T, seed=72, forced=forced)
    assert torch.equal(yp_f, yp_s)
    assert torch.equal(y_f, y_s)


@pytest.mark.parametrize("T,layout", [(1, "int4"), (8, "int4"), (12, "int4"), (2, "planes")])
def test_long_rows_against_oracle_and_slot_path(T, layout):
    """Long rows in the second GEMM (d_ff = 8192: 64 stages of 128 per row,
    eight per warp): the layer matches the oracle within the bar, and the
    slot path (the FFN wave by wave over a slot pool) gives the resident
    path's y_perm bit for bit."""
    from gpu_helpers import oracle_layer, within_tol
    shape = I.custom_shape(d=256, E=8, k=2, F=8192, group=128, layout=layout)
    L = I.make_layer(shape, T, seed=81 + T)
    layer = QuantMoELayer.from_weights(shape, L["w_router"].cuda(), L["bias"].cuda() if L["bias"] is not None
                                       else None, L["w_gate"].cuda(), L["w_up"].cuda(), L["w_down"].cuda(),
                                       max_tokens=T)
    bits = L["bits"].cuda() if layout == "planes" else None
    layer.buf["status"].zero_()
    y = layer.forward(L["x"].cuda(), bits=bits, residual=None).float().cpu().numpy()
    torch.cuda.synchronize()
    assert int(layer.buf["status"].item()) == 0
    ref, _ = oracle_layer(shape, L, bits=None if bits is None else bits.cpu())
    ok, worst = within_tol(y, ref["y"])
    assert ok, f"worst err/tol = {worst:.3f}"
    # the slot path: every expert through a pool of 4 slots, in waves
    v = layer.views(T)
    y_res = v["y_perm"].clone()
    blob = layer.blobs.shape[1]
    host = layer.blobs.cpu().pin_memory()
    pool = torch.empty(4, blob, dtype=torch.uint8, device="cuda")
    planes = (shape.d, shape.F, shape.group) if layout == "planes" else None
    cache = moeq.SlotCache(shape.E, 4, blob, host, pool, planes=planes)
    copy, compute = torch.cuda.Stream(), torch.cuda.current_stream()
    cache.stage(v["topk_idx"].cpu().reshape(-1), copy, compute,
                bits_host=None if bits is None else bits.cpu().reshape(-1))
    y_off = torch.empty_like(y_res)
    cache.ffn(v["x_perm"], v["offsets"], T, shape.d, shape.F, shape.group, layer.layout, v["workspace"], y_off,
              v["status"], copy, compute)
    torch.cuda.synchronize()
    assert torch.equal(y_off, y_res)
    cache.close()


def test_ffn_combine_and_combine_reject_misaligned_rows():
    """y, the residual and y_perm are read and written 16 bytes at a time:
    a pointer off a 16-byte boundary is refused on the host (before any
    launch), by both entry points."""
    shape = I.SHAPES["tiny"]
    T = 4
    L = I.make_layer(shape, T, seed=31)
    layer = QuantMoELayer.from_weights(shape, L["w_router"].cuda(), None, L["w_gate"].cuda(), L["w_up"].cuda(),
                                       L["w_down"].cuda(), max_tokens=T)
    x = L["x"].cuda()
    v = layer.views(T)
    moeq.moe_route_permute(x, layer.w_router, None, shape.k, out=v, status=v["status"], workspace=v["rp_ws"])
    torch.cuda.synchronize()
    y_off = torch.empty(T * shape.d + 8, dtype=torch.bfloat16, device="cuda")[1:1 + T * shape.d].view(T, shape.d)
    with pytest.raises(moeq.MoeError) as ei:
        moeq.moe_grouped_ffn_combine(v["x_perm"], v["offsets"], layer.blobs, T, shape.k, shape.E, shape.d,
                                     shape.F, shape.group, layer.layout, v["perm"], v["inv_perm"], v["topk_w"],
                                     residual=x, y=y_off)
    assert ei.value.code == 1
    yp = torch.zeros(T * shape.k, shape.d, dtype=torch.float16, device="cuda")
    with pytest.raises(moeq.MoeError) as ei:
        moeq.moe_unpermute_combine(yp, v["inv_perm"], v["topk_w"], residual=x, y=y_off)
    assert ei.value.code == 1

