"""The allocation-free router entry point (moe_route_topk_noalloc) against
the workspace-taking one (moe_route_topk), through the C ABI.

Callers that cannot allocate device memory where they route (plugins
handed only a stream, latency-critical serving paths) use the noalloc
variant, whose scratch is a fixed array inside the library.  Its
results must equal the regular router's: the same expert ids bit for bit
and the same gates, on two calls in a row (the second reuses the array).
This file is collected last so that a failure here never hides another."""
import numpy as np
import pytest
import torch

from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()


@pytest.mark.parametrize("name,T,seed", [("olmoe", 256, 1), ("tiny", 64, 2)])
def test_noalloc_router_matches_workspace_router(name, T, seed):
    shape = I.SHAPES[name]
    for call in range(2):  # two calls in a row share the fixed scratch
        L = I.make_layer(shape, T, seed=seed + call, weights=False)
        x, wr = L["x"].cuda(), L["w_router"].cuda()
        bias = L["bias"].cuda() if L["bias"] is not None else None
        idx_a, w_a = moeq.moe_route_topk(x, wr, bias, shape.k)
        idx_b, w_b = moeq.moe_route_topk_noalloc(x, wr, bias, shape.k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx_b.cpu().numpy(), idx_a.cpu().numpy())
        np.testing.assert_allclose(w_b.cpu().numpy(), w_a.cpu().numpy(), rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T", [2048, 4096])
def test_noalloc_router_at_large_batches(T):
    """Batches whose preferred d-slicing needs more scratch than the fixed
    array: the call lowers the slice count instead of refusing.  Expert ids
    equal the workspace router's bit for bit; gates (summed over fewer
    slices) agree with the fp64 oracle as the workspace router's do."""
    from oracle import moe_oracle as O
    from gpu_helpers import GATE_RTOL, GATE_ATOL
    shape = I.SHAPES["olmoe"]
    assert moeq.moe_route_workspace_bytes(T, shape.d, shape.E) > (8 << 20)
    for call in range(2):
        L = I.make_layer(shape, T, seed=40 + call, weights=False)
        x, wr, bias = L["x"].cuda(), L["w_router"].cuda(), L["bias"].cuda()
        idx_a, _ = moeq.moe_route_topk(x, wr, bias, shape.k)
        idx_b, w_b = moeq.moe_route_topk_noalloc(x, wr, bias, shape.k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx_b.cpu().numpy(), idx_a.cpu().numpy())
        sel, gates, _ = O.route(L["x"].float().numpy(), L["w_router"].numpy(), L["bias"].numpy(), shape.k)
        np.testing.assert_array_equal(idx_b.cpu().numpy(), sel)
        np.testing.assert_allclose(w_b.cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)


def test_noalloc_router_rejects_oversized_scratch():
    shape = I.SHAPES["olmoe"]
    T = 1 << 16  # needs more than the fixed 8 MiB of partial logits
    assert moeq.moe_route_workspace_bytes(T, shape.d, shape.E) > (8 << 20)
    x = torch.zeros(T, shape.d, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(shape.E, shape.d, dtype=torch.float32, device="cuda")
    with pytest.raises(moeq.MoeError) as ei:
        moeq.moe_route_topk_noalloc(x, wr, None, shape.k)
    assert ei.value.code == 2
