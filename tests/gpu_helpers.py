"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI and the oracle on the same seeded inputs."""
import numpy as np
import torch

from oracle import moe_oracle as O
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq
from quantized_moe_expert_histogram_b200.layer import QuantMoELayer

RTOL = 1e-2  # |y - y_ref| <= ATOL + RTOL * |y_ref|  (the layer's stated bar)
ATOL = 1e-2

# Gates come from fp32 logits (fp64 only for tokens whose top-k the fp32
# error bound leaves open).  A logit error dl moves gate j by a relative
# g_j * (dl_j - sum_i g_i dl_i), at most 2 max|dl|; the fp32 logits of these
# workloads (|l| of order 1-10, d <= 4096) err by ~1e-7 typically and a few
# 1e-7 at worst over a full batch, so 1e-5 relative leaves ample room while
# catching any mistake in the softmax itself.
GATE_RTOL = 1e-5
GATE_ATOL = 1e-8


def within_tol(y, y_ref, atol=ATOL, rtol=RTOL):
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    err = np.abs(y - y_ref)
    lim = atol + rtol * np.abs(y_ref)
    worst = float((err / lim).max()) if err.size else 0.0
    return bool((err <= lim).all()), worst


def layer_inputs(shape, T, seed=0, device="cpu"):
    return I.make_layer(shape, T, seed=seed, device=device)


def gpu_layer(shape, L, T):
    """Pack on the GPU and build the layer (weights moved to the device)."""
    dev = "cuda"
    wg, wu, wd = (L[k].to(dev) for k in ("w_gate", "w_up", "w_down"))
    bias = L["bias"].to(dev) if L["bias"] is not None else None
    layer = QuantMoELayer.from_weights(shape, L["w_router"].to(dev), bias, wg, wu, wd, max_tokens=T)
    return layer


def oracle_layer(shape, L, bits=None, sel=None, token_subset=None, experts=None):
    x = L["x"].float().cpu().numpy()
    if experts is None:
        experts = O.QuantExperts(L["w_gate"].cpu().numpy(), L["w_up"].cpu().numpy(),
                                 L["w_down"].cpu().numpy(), shape.group)
    bias = L["bias"].cpu().numpy() if L["bias"] is not None else None
    out = O.moe_layer(x, L["w_router"].cpu().numpy(), bias, shape.k, experts,
                      bits=None if bits is None else bits.cpu().numpy(), sel=sel,
                      token_subset=token_subset)
    return out, experts


def run_gpu_layer(layer, L, T, bits=None):
    x = L["x"].to("cuda")
    b = bits.to("cuda") if bits is not None else None
    layer.buf["status"].zero_()
    y = layer.forward(x, bits=b)
    torch.cuda.synchronize()
    return {k: v.clone() for k, v in layer.views(T).items()}, y.float().cpu().numpy()
