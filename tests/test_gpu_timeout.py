"""On-device failure detection without a GPU fault: every wait of the
tensor-core FFN is bounded.  A test hook shortens the limit to 20 ms and has
one epilogue withhold an arrive that no copy stands behind (so nothing is in
flight when the waiting CTA gives up); the launch must return, the caller's
status word must carry MOE_DEV_TIMEOUT, and the next normal call must be
exact again."""
import numpy as np
import pytest
import torch

from quantized_moe_expert_histogram_b200 import build
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq

from gpu_helpers import gpu_layer, layer_inputs, oracle_layer, run_gpu_layer, within_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _hooks():
    build.build()
    moeq.load()
    moeq.moe_debug_force_regime(2)
    yield
    moeq.moe_debug_ffn_timeout(0)
    moeq.moe_debug_force_regime(0)


def test_bounded_wait_times_out_and_the_next_call_is_exact():
    # d_ff 8192: 64 weight blocks x 4 bins = 256 gate/up tiles, so CTA 0 has a
    # second tile whose accumulators it waits for
    shape = I.custom_shape(d=256, E=4, k=2, F=8192, group=64)
    T = 24
    L = layer_inputs(shape, T, seed=3)
    layer = gpu_layer(shape, L, T)
    moeq.moe_debug_ffn_timeout(1)
    v, _ = run_gpu_layer(layer, L, T)  # returns (synchronised) instead of hanging
    st = int(v["status"].item())
    assert st & moeq.DEV_TIMEOUT, f"status {st}"
    moeq.moe_debug_ffn_timeout(0)
    v, y = run_gpu_layer(layer, L, T)
    assert int(v["status"].item()) == 0
    ref, _ = oracle_layer(shape, L)
    ok, worst = within_tol(y, ref["y"])
    assert ok, f"worst err/tol = {worst:.3f}"
