"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/moeq.h declares, and its blob-size arithmetic agrees
with the oracle's statement of the blob format."""
import pytest

from oracle import moe_oracle as O
from quantized_moe_expert_histogram_b200 import build, moeq


@pytest.fixture(scope="module")
def hostlib():
    build.build()
    return moeq.open_library()


def test_header_symbols_exported(hostlib):
    names = moeq.header_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(hostlib, n), n
    # the binding exposes every header function under the same name
    for n in names:
        if n not in ("moe_slot_cache_create", "moe_slot_stage", "moe_slot_ffn", "moe_slot_cache_destroy"):
            assert hasattr(moeq, n), n


@pytest.mark.parametrize("d,F,g,layout", [(256, 512, 64, "int4"), (2048, 1024, 128, "int4"),
                                          (4096, 14336, 128, "int4"), (4096, 1024, 128, "planes"),
                                          (256, 384, 64, "planes")])
def test_blob_bytes_match_format(hostlib, d, F, g, layout):
    lay = 1 if layout == "planes" else 0
    assert hostlib.moe_blob_bytes(d, F, g, lay) == O.blob_layout(d, F, g, layout)["bytes"]


@pytest.mark.parametrize("d,F,g,layout", [(100, 512, 64, 0), (256, 512, 32, 0), (256, 500, 64, 0),
                                          (256, 512, 64, 7), (0, 512, 64, 0)])
def test_blob_bytes_rejects_unsupported(hostlib, d, F, g, layout):
    assert hostlib.moe_blob_bytes(d, F, g, layout) == 0


def test_error_string_available(hostlib):
    assert isinstance(hostlib.moe_last_error(), bytes)
