"""Parity at the full sizes of the named workloads, in the launch
configuration the benchmark times (auto regime: tensor cores above 8
tokens).  Routing, histograms and permutations are compared on every token;
layer outputs on a seeded sample of tokens (tokens are independent in an
MoE layer, so a sample is a valid check of the same launch)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq
from quantized_moe_expert_histogram_b200.layer import QuantMoELayer

from gpu_helpers import within_tol, GATE_RTOL, GATE_ATOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()
    moeq.moe_debug_force_regime(0)


@pytest.mark.parametrize("name,T,n_sample", [("olmoe", 4096, 48), ("nested", 2048, 24), ("mixtral", 8192, 6)])
def test_full_size_sampled(name, T, n_sample):
    shape = I.SHAPES[name]
    L = I.make_layer(shape, T, seed=0, device="cuda")
    layer = QuantMoELayer.from_weights(shape, L["w_router"], L["bias"], L["w_gate"], L["w_up"], L["w_down"],
                                       max_tokens=T)
    bits = L.get("bits")
    y = layer.forward(L["x"], bits=bits).float().cpu().numpy()
    torch.cuda.synchronize()
    v = layer.views(T)
    assert int(v["status"].item()) == 0
    x = L["x"].float().cpu().numpy()
    bias = L["bias"].cpu().numpy() if L["bias"] is not None else None
    sel, gates, _ = O.route(x, L["w_router"].cpu().numpy(), bias, shape.k)
    np.testing.assert_array_equal(v["topk_idx"].cpu().numpy(), sel)
    np.testing.assert_allclose(v["topk_w"].cpu().numpy(), gates, rtol=GATE_RTOL, atol=GATE_ATOL)
    keys, mult = O.assignment_keys(sel, None if bits is None else bits.cpu().numpy())
    counts, offsets, perm, inv = O.permute(keys, shape.E * (mult or 1))
    np.testing.assert_array_equal(v["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(v["perm"].cpu().numpy(), perm)
    np.testing.assert_array_equal(v["inv_perm"].cpu().numpy(), inv)
    # outputs of sampled tokens; the oracle quantises only the experts they use
    rng = np.random.default_rng(T)
    toks = np.sort(rng.choice(T, n_sample, replace=False))
    needed = sorted(set(sel[toks].reshape(-1).tolist()))
    wg = {e: L["w_gate"][e].cpu().numpy() for e in needed}
    wu = {e: L["w_up"][e].cpu().numpy() for e in needed}
    wd = {e: L["w_down"][e].cpu().numpy() for e in needed}
    del L["w_gate"], L["w_up"], L["w_down"]
    torch.cuda.empty_cache()

    class Sparse(O.QuantExperts):
        def __init__(self):
            self.group, self._q = shape.group, {}

        def quant(self, e):
            if e not in self._q:
                self._q[e] = tuple(O.quantize_groups(m[e], shape.group) for m in (wg, wu, wd))
            return self._q[e]

    ref = O.moe_layer(x[toks], L["w_router"].cpu().numpy(), bias, shape.k, Sparse(),
                      bits=None if bits is None else bits.cpu().numpy()[toks])
    np.testing.assert_array_equal(ref["sel"], sel[toks])
    ok, worst = within_tol(y[toks], ref["y"])
    assert ok, f"{name} T={T}: worst err/tol {worst:.3f}"
