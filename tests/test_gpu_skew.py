"""Degenerate routings through every FFN kernel ([ExactMoE] every routed
expert runs exactly, however the tokens fall): all tokens on the same k
experts (one or two bins hold every row, the others are empty), and a
skewed routing where one expert takes most tokens while most bins hold zero
or one row.  The decode kernel (one or two 8-token blocks per pass), the
tensor-core kernel (a bin spanning several 128-row token blocks) and the
default choice, for INT4 and the nested widths, against the oracle at the
same forced expert ids: permutation exact, y_perm and y within the bar."""
import numpy as np
import pytest
import torch

from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq

from gpu_helpers import gpu_layer, layer_inputs, oracle_layer, within_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()
    yield
    moeq.moe_debug_force_regime(0)


def _ids(pattern, T, E, k, seed):
    rng = np.random.default_rng(seed)
    if pattern == "hot":  # every token: experts 3 and E - 5, in that order
        return np.tile(np.array([3, E - 5][:k], dtype=np.int32), (T, 1))
    # skewed: expert 0 first for 3 tokens in 4, the rest spread at random
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    hot = rng.random(T) < 0.75
    for t in np.nonzero(hot)[0]:
        row = [0] + [e for e in ids[t] if e != 0][:k - 1]
        ids[t] = row
    return ids


@pytest.mark.parametrize("layout", ["int4", "planes"])
@pytest.mark.parametrize("pattern", ["hot", "skew"])
@pytest.mark.parametrize("regime,T", [(1, 9), (1, 64), (3, 40), (2, 64), (2, 300), (0, 300)])
def test_degenerate_routing_every_kernel(layout, pattern, regime, T):
    shape = I.custom_shape(d=512, E=16, k=2, F=256, group=128, layout=layout)
    L = layer_inputs(shape, T, seed=90 + T)
    ids = _ids(pattern, T, shape.E, shape.k, seed=T)
    layer = gpu_layer(shape, L, T)
    bits = L.get("bits")
    moeq.moe_debug_force_regime(regime)
    try:
        layer.buf["status"].zero_()
        y = layer.forward(L["x"].cuda(), bits=None if bits is None else bits.cuda(),
                          forced_idx=torch.from_numpy(ids).cuda())
        torch.cuda.synchronize()
    finally:
        moeq.moe_debug_force_regime(0)
    v = {key: val.clone() for key, val in layer.views(T).items()}
    assert int(v["status"].item()) == 0, f"device status {int(v['status'].item())}"
    ref, _ = oracle_layer(shape, L, bits=bits, sel=ids)
    np.testing.assert_array_equal(v["topk_idx"].cpu().numpy(), ids)
    np.testing.assert_array_equal(v["counts"].cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(v["perm"].cpu().numpy(), ref["perm"])
    if pattern == "hot":  # every row in k bins (k of them per width with nested planes)
        assert int((ref["counts"] > 0).sum()) <= shape.k * (3 if layout == "planes" else 1)
    yp = v["y_perm"].float().cpu().numpy()
    ok2, worst2 = within_tol(yp[ref["inv_perm"]], ref["y_assign"])
    ok, worst = within_tol(y.float().cpu().numpy(), ref["y"])
    assert ok2, f"y_perm worst err/tol = {worst2:.3f}"
    assert ok, f"y worst err/tol = {worst:.3f}"
