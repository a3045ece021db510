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


# Argument checks and the empty batch are decided before any CUDA call, so
# they can be pinned on a host without a GPU.
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE = 0, 1, 2


def test_zero_tokens_are_no_ops(hostlib):
    n = None
    # route, FFN and combine of an empty batch succeed without touching memory
    assert hostlib.moe_route_topk(n, n, n, n, 0, 256, 8, 2, n, n, n, 0, n) == MOE_OK
    assert hostlib.moe_grouped_ffn_wq(n, n, n, n, 0, 0, 8, 256, 512, 64, 0, n, 0, n, n, n) == MOE_OK
    assert hostlib.moe_unpermute_combine(n, n, n, n, 0, 2, 256, n, n) == MOE_OK


@pytest.mark.parametrize("call,code,words", [
    (lambda L: L.moe_route_topk(None, None, None, None, -1, 256, 8, 2, None, None, None, 0, None),
     MOE_ERR_INVALID_ARG, "bad sizes"),
    (lambda L: L.moe_route_topk(None, None, None, None, 4, 256, 8, 2, None, None, None, 0, None),
     MOE_ERR_INVALID_ARG, "null pointer"),
    (lambda L: L.moe_permute(None, None, None, 4, 64, 8, 9, None, None, None, None, None, None, None, 0, None),
     MOE_ERR_INVALID_ARG, "bad sizes"),
    (lambda L: L.moe_grouped_ffn_wq(None, None, None, None, 4, 4, 8, 256, 500, 64, 0, None, 0, None, None, None),
     MOE_ERR_UNSUPPORTED_SHAPE, "unsupported shape"),
    (lambda L: L.moe_grouped_ffn_wq(None, None, None, None, 4, 4, 8, 256, 512, 64, 0, None, 0, None, None, None),
     MOE_ERR_INVALID_ARG, "null pointer"),
    (lambda L: L.moe_unpermute_combine(None, None, None, None, 4, 2, 250, None, None),
     MOE_ERR_INVALID_ARG, "bad sizes"),
    (lambda L: L.moe_static_bits(None, None, 4, 8, 2, None, None, None), MOE_ERR_INVALID_ARG, "null pointer"),
])
def test_bad_arguments_rejected_with_message(hostlib, call, code, words):
    assert call(hostlib) == code
    assert words in hostlib.moe_last_error().decode()
