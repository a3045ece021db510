"""The benchmark's count of this library's kernels per layer step
(`gpu_launches`) follows the library's own launch choices: router, bit gate
and permutation are one cluster launch for the smallest batches (T <= 8,
T*k <= 64, T*E <= 512); otherwise the router is one cluster launch up to 64
tokens (E <= 64) and two launches beyond, the bit gate adds one, the
permutation is one single-CTA launch up to 1024 assignments (gathering the
rows itself up to 64 K elements, else one gather launch after it) and
histogram + scan + scatter + gather above; the FFN two; the combine one.
(No GPU needed.)"""
import bench
from quantized_moe_expert_histogram_b200 import inputs as I


def test_kernel_launches_per_step():
    S = I.SHAPES
    assert bench.kernel_launches(S["olmoe"], 1) == 1 + 2 + 1              # route + permute in one launch
    assert bench.kernel_launches(S["olmoe"], 8) == 1 + 2 + 1              # 64 assignments, T*E = 512
    assert bench.kernel_launches(S["olmoe"], 9) == 1 + 2 + 2 + 1          # 72 x 2048 > 64 K: gather launch
    assert bench.kernel_launches(S["olmoe"], 64) == 1 + 2 + 2 + 1         # 64 tokens: 8 slices x 8 tokens
    assert bench.kernel_launches(S["olmoe"], 65) == 2 + 2 + 2 + 1         # beyond the one-launch router
    assert bench.kernel_launches(S["olmoe"], 4096) == 2 + 4 + 2 + 1
    assert bench.kernel_launches(S["mixtral"], 1) == 1 + 2 + 1
    assert bench.kernel_launches(S["mixtral"], 16) == 1 + 2 + 2 + 1       # 32 x 4096 > 64 K: gather launch
    assert bench.kernel_launches(S["mixtral"], 8192) == 2 + 4 + 2 + 1
    assert bench.kernel_launches(S["nested"], 1, bit_gate=True) == 1 + 2 + 1
    assert bench.kernel_launches(S["nested"], 32, bit_gate=True) == 1 + 1 + 2 + 2 + 1
    assert bench.kernel_launches(S["nested"], 2048, bit_gate=True) == 2 + 1 + 4 + 2 + 1
