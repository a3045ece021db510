"""The benchmark's count of this library's kernels per layer step
(`gpu_launches`) follows the library's own launch choices: router, bit gate
and permutation are one cluster launch for the smallest batches (T <= 8,
T*E <= 512, with a bit gate T*E <= 128, T*k <= 64); otherwise the router is
two launches, the bit gate adds one, the
permutation is one single-CTA launch up to 1024 assignments (gathering the
rows itself up to 64 K elements, else one gather launch after it) and
histogram + scan + scatter + gather above; the FFN two; the combine one.
(No GPU needed.)"""
import bench
from quantized_moe_expert_histogram_b200 import inputs as I


def test_kernel_launches_per_step():
    S = I.SHAPES
    assert bench.kernel_launches(S["olmoe"], 1) == 1 + 2 + 1              # route + permute in one launch, FFN, combine
    assert bench.kernel_launches(S["olmoe"], 2) == 1 + 2 + 1              # T*E = 128
    assert bench.kernel_launches(S["olmoe"], 8) == 1 + 2 + 1              # T*E = 512, T*k = 64
    assert bench.kernel_launches(S["olmoe"], 16) == 2 + 2 + 2 + 1
    assert bench.kernel_launches(S["olmoe"], 17) == 2 + 2 + 2 + 1
    assert bench.kernel_launches(S["olmoe"], 64) == 2 + 2 + 2 + 1
    assert bench.kernel_launches(S["olmoe"], 4096) == 2 + 4 + 2 + 1       # histogram, scan, scatter, gather
    assert bench.kernel_launches(S["mixtral"], 1) == 1 + 2 + 1
    assert bench.kernel_launches(S["mixtral"], 8) == 1 + 2 + 1            # T*E = 64, T*k = 16
    assert bench.kernel_launches(S["mixtral"], 16) == 2 + 2 + 2 + 1       # 32 x 4096 > 64 K: gather launch
    assert bench.kernel_launches(S["mixtral"], 8192) == 2 + 4 + 2 + 1
    assert bench.kernel_launches(S["nested"], 1, bit_gate=True) == 1 + 2 + 1
    assert bench.kernel_launches(S["nested"], 8, bit_gate=True) == 1 + 2 + 1   # T*k = 32
    assert bench.kernel_launches(S["nested"], 32, bit_gate=True) == 2 + 1 + 2 + 2 + 1
    assert bench.kernel_launches(S["nested"], 2048, bit_gate=True) == 2 + 1 + 4 + 2 + 1
