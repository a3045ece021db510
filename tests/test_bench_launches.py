"""The benchmark's count of this library's kernels per layer step
(`gpu_launches`) follows the library's own launch choices: the router is
one cluster launch for decode-sized batches (up to 8 tokens per d slice of
a cluster of up to 8 CTAs, E <= 64) and two launches otherwise; the bit gate
adds one; the permutation is one single-CTA launch up to 1024 assignments
(gathering the rows itself up to 64 K elements, else one gather launch
after it) and histogram + scan + scatter + gather above; the FFN two; the
combine one.  (No GPU needed.)"""
import bench
from quantized_moe_expert_histogram_b200 import inputs as I


def test_kernel_launches_per_step():
    S = I.SHAPES
    assert bench.kernel_launches(S["olmoe"], 1) == 1 + 1 + 2 + 1          # 8 x 2048 = 16 K gathered
    assert bench.kernel_launches(S["olmoe"], 8) == 1 + 2 + 2 + 1          # 64 x 2048 > 64 K: gather launch
    assert bench.kernel_launches(S["olmoe"], 64) == 1 + 2 + 2 + 1         # 64 tokens: 8 slices x 8 tokens
    assert bench.kernel_launches(S["olmoe"], 65) == 2 + 2 + 2 + 1         # beyond the one-launch router
    assert bench.kernel_launches(S["olmoe"], 4096) == 2 + 4 + 2 + 1
    assert bench.kernel_launches(S["mixtral"], 1) == 1 + 1 + 2 + 1
    assert bench.kernel_launches(S["mixtral"], 8192) == 2 + 4 + 2 + 1
    assert bench.kernel_launches(S["nested"], 1, bit_gate=True) == 1 + 1 + 1 + 2 + 1
    assert bench.kernel_launches(S["nested"], 2048, bit_gate=True) == 2 + 1 + 4 + 2 + 1
