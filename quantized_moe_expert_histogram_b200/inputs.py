"""Seeded synthetic inputs for the quantized MoE layer.

This module only draws random numbers with the shapes and distributions of
the workloads; it holds none of the layer's arithmetic (no quantisation,
routing, permutation or FFN math).  Both the CUDA path and the CPU oracle
are fed from here, so a test hands the same tensors to both sides.

Workloads (shapes of public MoE architectures, random weights):

* ``tiny``    d=256,  E=8,  k=2, d_ff=512,   group 64,  INT4, 64 tokens
* ``olmoe``   d=2048, E=64, k=8, d_ff=1024,  group 128, INT4, router bias
              skewed by a Zipf(1.1) rank order, tokens {1,16,256,4096}
* ``mixtral`` d=4096, E=8,  k=2, d_ff=14336, group 128, INT4, tokens
              {1,32,512,8192}
* ``nested``  d=4096, E=16, k=4, d_ff=1024,  group 128, bit planes 2+1+1,
              per (token, expert) width b in {2,3,4} w.p. {0.3,0.4,0.3},
              tokens {1,64,2048}
* ``slot``    16 stacked ``olmoe`` layers, 16 GPU slots per layer, batch 8
              decode steps, expert ids from a Zipf trace with a 70 %
              layer-to-layer successor table.

Distributions: x ~ N(0,1) rounded to bf16; router W_r ~ N(0, 0.02^2) fp32;
expert weights ~ N(0, 0.02^2) fp32.  Zipf bias: rank = randperm(E),
bias[e] = -1.1 * ln(1 + rank[e]) (the log of a Zipf(1.1) pmf over ranks).
Generation order inside one call: x, W_r, bias ranks, W_gate, W_up, W_down,
bit-widths.  Everything comes from one ``torch.Generator`` seeded with
``seed`` on the requested device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class LayerShape:
    name: str
    d: int
    E: int
    k: int
    F: int
    group: int
    layout: str  # "int4" or "planes"
    zipf: bool
    tokens: tuple = field(default=())


SHAPES = {
    "tiny": LayerShape("tiny", 256, 8, 2, 512, 64, "int4", False, (64,)),
    "olmoe": LayerShape("olmoe", 2048, 64, 8, 1024, 128, "int4", True, (1, 16, 256, 4096)),
    "mixtral": LayerShape("mixtral", 4096, 8, 2, 14336, 128, "int4", False, (1, 32, 512, 8192)),
    "nested": LayerShape("nested", 4096, 16, 4, 1024, 128, "planes", False, (1, 64, 2048)),
}

# Offload workload: stacked olmoe-shaped layers with a slot cache.
SLOT_WORKLOAD = dict(base="olmoe", layers=16, slots=16, steps=512, batch=8, p_successor=0.7)

WEIGHT_STD = 0.02
ROUTER_STD = 0.02
ZIPF_S = 1.1
BIT_PROBS = (0.3, 0.4, 0.3)  # b = 2, 3, 4


def custom_shape(name="custom", d=256, E=8, k=2, F=512, group=64, layout="int4", zipf=False):
    return LayerShape(name, d, E, k, F, group, layout, zipf, ())


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_bias(E: int, gen: torch.Generator, device) -> torch.Tensor:
    rank = torch.randperm(E, generator=gen, device=device)
    return (-ZIPF_S * torch.log1p(rank.to(torch.float64))).to(torch.float32)


def draw_bits(T: int, k: int, gen: torch.Generator, device) -> torch.Tensor:
    u = torch.rand(T, k, generator=gen, device=device)
    b = torch.full((T, k), 4, dtype=torch.uint8, device=device)
    b[u < BIT_PROBS[0] + BIT_PROBS[1]] = 3
    b[u < BIT_PROBS[0]] = 2
    return b


def make_layer(shape: LayerShape, T: int, seed: int = 0, device="cpu", weights=True) -> dict:
    """Draw one layer's inputs.

    Returns a dict with ``x`` bf16 [T,d], ``w_router`` fp32 [E,d], ``bias``
    fp32 [E] or None, ``w_gate``/``w_up`` fp32 [E,F,d], ``w_down`` fp32
    [E,d,F] (absent when ``weights`` is False) and ``bits`` uint8 [T,k]
    (nested layout only).
    """
    gen = _gen(seed, device)
    d, E, F = shape.d, shape.E, shape.F
    out = {}
    out["x"] = torch.randn(T, d, generator=gen, device=device).to(torch.bfloat16)
    out["w_router"] = torch.randn(E, d, generator=gen, device=device) * ROUTER_STD
    out["bias"] = zipf_bias(E, gen, device) if shape.zipf else None
    if weights:
        out["w_gate"] = torch.randn(E, F, d, generator=gen, device=device) * WEIGHT_STD
        out["w_up"] = torch.randn(E, F, d, generator=gen, device=device) * WEIGHT_STD
        out["w_down"] = torch.randn(E, d, F, generator=gen, device=device) * WEIGHT_STD
    if shape.layout == "planes":
        out["bits"] = draw_bits(T, shape.k, gen, device)
    return out


def make_bit_gate(shape: LayerShape, seed: int, device="cpu", bias: bool = False) -> dict:
    """Synthetic weights of a bit-width gate (one linear score per width and
    expert): ``w_bit`` fp32 [E,3,d] ~ N(0, 0.02^2) and, when ``bias``,
    ``bias_bit`` fp32 [E,3] ~ N(0, 0.1^2) (else None)."""
    gen = _gen(seed, device)
    out = {"w_bit": torch.randn(shape.E, 3, shape.d, generator=gen, device=device) * ROUTER_STD}
    out["bias_bit"] = torch.randn(shape.E, 3, generator=gen, device=device) * 0.1 if bias else None
    return out


def make_expert_weights(shape: LayerShape, seed: int, device="cpu") -> dict:
    """Expert weights alone (used for the stacked offload layers)."""
    gen = _gen(seed, device)
    d, E, F = shape.d, shape.E, shape.F
    return {
        "w_gate": torch.randn(E, F, d, generator=gen, device=device) * WEIGHT_STD,
        "w_up": torch.randn(E, F, d, generator=gen, device=device) * WEIGHT_STD,
        "w_down": torch.randn(E, d, F, generator=gen, device=device) * WEIGHT_STD,
    }


def make_router(shape: LayerShape, seed: int, device="cpu") -> dict:
    gen = _gen(seed, device)
    return {
        "w_router": torch.randn(shape.E, shape.d, generator=gen, device=device) * ROUTER_STD,
        "bias": zipf_bias(shape.E, gen, device) if shape.zipf else None,
    }


def _zipf_pmf(E: int):
    w = np.array([1.0 / math.pow(r + 1, ZIPF_S) for r in range(E)], dtype=np.float64)
    return w / w.sum()


def make_slot_trace(E: int, k: int, layers: int, steps: int, batch: int, seed: int = 0,
                    p_successor: float = 0.7) -> torch.Tensor:
    """Expert-id trace for the offload workload, int32 [steps, layers, batch, k].

    Layer 0: k distinct ids drawn by Zipf(1.1) over a seeded rank order.
    Layer l>0, choice j: with probability ``p_successor`` the successor
    table's entry for the id chosen at layer l-1 (same j), otherwise a Zipf
    draw; a repeated id inside one token is redrawn from Zipf.
    """
    rng = np.random.default_rng(seed)
    rank_to_expert = rng.permutation(E)
    succ = rng.integers(0, E, size=(layers, E))
    pmf = _zipf_pmf(E)
    u = rng.random((steps, layers, batch, k))
    pool = rank_to_expert[rng.choice(E, size=steps * layers * batch * k * 4, p=pmf)]
    pos = 0
    trace = np.empty((steps, layers, batch, k), dtype=np.int32)
    for s in range(steps):
        for t in range(batch):
            prev = None
            for l in range(layers):
                chosen = []
                for j in range(k):
                    cand = -1
                    if prev is not None and u[s, l, t, j] < p_successor:
                        cand = int(succ[l, prev[j]])
                    while cand < 0 or cand in chosen:
                        if pos == pool.size:
                            pool = rank_to_expert[rng.choice(E, size=pool.size, p=pmf)]
                            pos = 0
                        cand = int(pool[pos])
                        pos += 1
                    chosen.append(cand)
                trace[s, l, t] = chosen
                prev = chosen
    return torch.from_numpy(trace)


def make_slot_x(d: int, steps: int, batch: int, seed: int = 0, device="cpu") -> torch.Tensor:
    gen = _gen(seed + 7919, device)
    return torch.randn(steps, batch, d, generator=gen, device=device).to(torch.bfloat16)
