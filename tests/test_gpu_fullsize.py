"""Parity at the full sizes of the named workloads, in the launch
configuration the benchmark times (the default regime choice by token
count).  One layer instance per workload (weights drawn once, seed 0) serves
every token count: the first T rows of the seeded activations are the batch.
Routing, histograms and permutations are compared on every token; layer
outputs on a seeded sample of tokens (tokens are independent in an MoE
layer, so a sample checks the same launch), all tokens for small T."""
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

T_MAX = {"olmoe": 4096, "nested": 2048, "mixtral": 8192}
_CACHE = {}


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    moeq.load()
    moeq.moe_debug_force_regime(0)
    yield
    _CACHE.clear()
    torch.cuda.empty_cache()


class _Sparse(O.QuantExperts):
    """The oracle's quantised experts, quantising an expert only when a
    sampled token needs it (host fp32 weights kept for that)."""

    def __init__(self, w, group):
        self.w_host, self.group, self._q = w, group, {}

    def quant(self, e):
        if e not in self._q:
            self._q[e] = tuple(O.quantize_groups(m[e], self.group) for m in self.w_host)
        return self._q[e]


def _workload(name):
    if name not in _CACHE:
        for other in list(_CACHE):  # one workload's device buffers at a time
            del _CACHE[other]
        torch.cuda.empty_cache()
        shape = I.SHAPES[name]
        L = I.make_layer(shape, T_MAX[name], seed=0, device="cuda")
        layer = QuantMoELayer.from_weights(shape, L["w_router"], L["bias"], L["w_gate"], L["w_up"], L["w_down"],
                                           max_tokens=T_MAX[name])
        w_host = tuple(L[k].cpu().numpy() for k in ("w_gate", "w_up", "w_down"))
        del L["w_gate"], L["w_up"], L["w_down"]
        torch.cuda.empty_cache()
        _CACHE[name] = (shape, L, layer, _Sparse(w_host, shape.group))
    return _CACHE[name]


@pytest.mark.parametrize("name,T,n_sample", [
    ("olmoe", 4096, 48), ("olmoe", 256, 32), ("olmoe", 16, 16), ("olmoe", 1, 1),
    ("nested", 2048, 24), ("nested", 64, 16), ("nested", 8, 8), ("nested", 4, 4), ("nested", 1, 1),
    ("mixtral", 8192, 6), ("mixtral", 512, 64), ("mixtral", 32, 32), ("mixtral", 1, 1)])
def test_full_size_sampled(name, T, n_sample):
    shape, L, layer, experts = _workload(name)
    x_dev = L["x"][:T].contiguous()
    bits = L["bits"][:T].contiguous() if "bits" in L else None
    layer.buf["status"].zero_()
    y = layer.forward(x_dev, bits=bits).float().cpu().numpy()
    torch.cuda.synchronize()
    v = layer.views(T)
    assert int(v["status"].item()) == 0
    x = x_dev.float().cpu().numpy()
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
    # outputs of sampled tokens (all of them when n_sample == T)
    rng = np.random.default_rng(T)
    toks = np.arange(T) if n_sample >= T else np.sort(rng.choice(T, n_sample, replace=False))
    ref = O.moe_layer(x[toks], L["w_router"].cpu().numpy(), bias, shape.k, experts,
                      bits=None if bits is None else bits.cpu().numpy()[toks])
    np.testing.assert_array_equal(ref["sel"], sel[toks])
    ok, worst = within_tol(y[toks], ref["y"])
    assert ok, f"{name} T={T}: worst err/tol {worst:.3f}"
    # per-assignment expert outputs of the sampled tokens (before the combine)
    yp = v["y_perm"].float().cpu().numpy()
    rows = np.array([t * shape.k + j for t in toks for j in range(shape.k)])
    ok2, worst2 = within_tol(yp[inv[rows]], ref["y_assign"])
    assert ok2, f"{name} T={T}: y_perm worst err/tol {worst2:.3f}"
