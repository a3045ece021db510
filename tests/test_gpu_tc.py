"""GPU parity of the tensor-core grouped FFN (tcgen05, swap-AB, fused
dequant) against the oracle, across shapes that exercise several weight
blocks, ragged token blocks (bins that are not multiples of 16 rows), empty
bins, group sizes 64 and 128, both weight layouts and the nested widths."""
import numpy as np
import pytest
import torch

from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq

from gpu_helpers import gpu_layer, layer_inputs, oracle_layer, run_gpu_layer, within_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _tc_regime():
    build.build()
    moeq.load()
    moeq.moe_debug_force_regime(2)
    yield
    moeq.moe_debug_force_regime(0)


def _check(shape, T, seed=0):
    L = layer_inputs(shape, T, seed=seed)
    layer = gpu_layer(shape, L, T)
    bits = L.get("bits")
    v, y = run_gpu_layer(layer, L, T, bits=bits)
    ref, _ = oracle_layer(shape, L, bits=bits)
    np.testing.assert_array_equal(v["perm"].cpu().numpy(), ref["perm"])
    assert int(v["status"].item()) == 0, f"device status {int(v['status'].item())}"
    yp = v["y_perm"].float().cpu().numpy()
    ok2, worst2 = within_tol(yp[ref["inv_perm"]], ref["y_assign"])
    ok, worst = within_tol(y, ref["y"])
    assert ok2, f"y_perm worst err/tol = {worst2:.3f}"
    assert ok, f"y worst err/tol = {worst:.3f}"
    return layer, L, v


@pytest.mark.parametrize("d,E,k,F,g,layout,T", [
    (256, 4, 2, 128, 64, "int4", 16),      # one weight block per matrix, one token block
    (256, 4, 2, 256, 64, "int4", 40),      # ragged bins
    (384, 6, 3, 640, 128, "int4", 97),     # several weight blocks, odd sizes
    (256, 5, 2, 384, 64, "planes", 70),    # nested widths, (e, b) bins
    (512, 3, 1, 256, 128, "int4", 600),    # bins larger than one 128/256-row token block
])
def test_tc_small_shapes(d, E, k, F, g, layout, T):
    _check(I.custom_shape(d=d, E=E, k=k, F=F, group=g, layout=layout), T, seed=9)


@pytest.mark.parametrize("name,T", [("tiny", 64), ("olmoe", 16), ("olmoe", 256), ("nested", 64)])
def test_tc_named_shapes(name, T):
    _check(I.SHAPES[name], T)


def test_tc_matches_gemv():
    shape = I.custom_shape(d=512, E=6, k=2, F=384, group=128)
    T = 48
    L = layer_inputs(shape, T, seed=2)
    layer = gpu_layer(shape, L, T)
    v_tc, y_tc = run_gpu_layer(layer, L, T)
    moeq.moe_debug_force_regime(1)
    v_gv, y_gv = run_gpu_layer(layer, L, T)
    ok, worst = within_tol(y_tc, y_gv)
    assert ok, worst
    # h of both kernels (fp16) agree to fp16 weight rounding
    h_tc = v_tc["workspace"][: T * shape.k * shape.F * 2].view(torch.float16).float().cpu().numpy()
    h_gv = v_gv["workspace"][: T * shape.k * shape.F * 2].view(torch.float16).float().cpu().numpy()
    ok, worst = within_tol(h_tc, h_gv, atol=1e-3, rtol=1e-2)
    assert ok, worst
