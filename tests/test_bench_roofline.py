"""The roofline's numerators (no GPU needed): the FFN's algorithmic bytes
are the routed experts' blob bytes -- each expert once, whole for INT4, up
to the widest width its assignments use for the nested planes -- plus the
activations in and out; its FLOPs are 6 d F per assignment.  The byte count
is checked against the library's own blob size."""
import torch

import bench
from quantized_moe_expert_histogram_b200 import inputs as I
from quantized_moe_expert_histogram_b200 import moeq


class _Routed:
    """Stands in for a layer whose last step routed `counts` rows per bin."""

    def __init__(self, counts):
        self.counts = torch.tensor(counts, dtype=torch.int32)

    def views(self, T):
        return {"counts": self.counts}


def test_int4_bytes_are_the_routed_blobs_and_flops_6dF():
    lib = moeq.open_library()
    S = I.SHAPES["olmoe"]
    T = 4096
    counts = [0] * S.E
    for e in range(0, S.E, 3):  # 22 experts routed, the rest empty
        counts[e] = 7
    b, fl = bench.algorithmic(S, T, _Routed(counts), bits_present=False)
    blob = lib.moe_blob_bytes(S.d, S.F, S.group, 0)
    assert blob == 3342336
    assert b == 22 * blob + 2 * T * S.d * 2
    assert fl == 6 * S.d * S.F * T * S.k


def test_nested_bytes_read_planes_up_to_the_widest_width():
    lib = moeq.open_library()
    S = I.SHAPES["nested"]
    T = 64
    counts = [0] * (3 * S.E)        # bins 3 e + (b - 2)
    counts[3 * 0 + 0] = 5           # expert 0: width 2 only
    counts[3 * 1 + 0] = 2           # expert 1: widths 2 and 4
    counts[3 * 1 + 2] = 1
    counts[3 * 2 + 1] = 4           # expert 2: width 3
    b, fl = bench.algorithmic(S, T, _Routed(counts), bits_present=True)
    full = lib.moe_blob_bytes(S.d, S.F, S.group, 1)
    sz = 3 * S.d * S.F // S.group * 4
    codes = full - sz
    assert b == (codes * 2 // 4 + sz) + (codes + sz) + (codes * 3 // 4 + sz) + 2 * T * S.d * 2
    assert fl == 6 * S.d * S.F * T * S.k
