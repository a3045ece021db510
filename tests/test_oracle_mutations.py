"""The oracle's pins catch plausible mistakes.  Each case plants one mistake
in the oracle -- on the CPU, in this process only (pytest's monkeypatch
undoes it) -- of the kinds a restatement of the pages could make: a wrong
sign, a dropped term or factor, an off-by-one zero point, a wrong tie rule,
swapped operands or planes, a wrong nibble or bin order, an unstable sort.
At least one of the pins named for it must then fail; with nothing planted
they all pass."""
import numpy as np
import pytest

import test_oracle_bitgate as PB
import test_oracle_quant as PQ
import test_oracle_route_ffn as PR
from oracle import moe_oracle as O

_ORIG = {name: getattr(O, name) for name in (
    "quantize_groups", "dequant", "pack_int4", "join_planes", "router_logits", "topk_select", "gates_for",
    "permute", "assignment_keys", "silu", "expert_ffn", "combine", "bit_gate", "tile_words", "f32_to_bf16_bits",
    "sz_tiled")}


def _calls(fn):
    """The pin with each of its parametrisations."""
    marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
    if not marks:
        return [{}]
    (m,) = marks
    names = [a.strip() for a in m.args[0].split(",")]
    return [dict(zip(names, v if len(names) > 1 else (v,))) for v in m.args[1]]


def _fails(pins):
    """Name of the first listed pin (any parametrisation) whose assertion
    fails, else None (any other error propagates: a mutant that merely
    breaks the call does not count as caught)."""
    for fn in pins:
        for kw in _calls(fn):
            try:
                fn(**kw)
            except AssertionError:
                return fn.__name__
    return None


def _topk_high_ties(logits, k):
    T, E = logits.shape
    out = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        out[t] = np.lexsort((-idx, -logits[t]))[:k]  # equal logits: higher index first
    return out


def _gates_unrenormalised(logits, sel):
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)  # softmax over every expert, not the selection
    return np.take_along_axis(p, sel.astype(np.int64), axis=1).astype(np.float32)


def _permute_unstable(keys, nbins):
    counts, offsets, perm, _ = _ORIG["permute"](keys, nbins)
    perm = perm.copy()
    for b in range(nbins):  # rows of a bin in descending assignment order
        perm[offsets[b]:offsets[b + 1]] = perm[offsets[b]:offsets[b + 1]][::-1]
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=perm.dtype)
    return counts, offsets, perm, inv


def _pack_reversed(q):
    N, K = q.shape
    return _ORIG["pack_int4"](q.reshape(N, K // 8, 8)[:, :, ::-1].reshape(N, K))


def _bit_gate_wide_ties(x, w_bit, bias_bit, sel):
    # the widths in reverse order: the first maximum is then the widest of equals
    b = _ORIG["bit_gate"](x, np.ascontiguousarray(w_bit[:, ::-1]),
                          None if bias_bit is None else np.ascontiguousarray(np.asarray(bias_bit)[:, ::-1]), sel)
    return (6 - b.astype(np.int64)).astype(b.dtype)


def _combine_last_dropped(y_assign, gates):
    g = gates.copy()
    g[:, -1] = 0.0
    return _ORIG["combine"](y_assign, g)


MUTANTS = {
    "zero point one too high": (
        "quantize_groups", lambda w, group: (lambda q, s, z: (q, s, z + 1))(*_ORIG["quantize_groups"](w, group)),
        [PQ.test_worked_examples, PQ.test_closed_form_uniform_grid, PQ.test_error_bound]),
    "dequantisation adds the zero point": (
        "dequant", lambda q, s, z, group, b=4: _ORIG["dequant"](q, s, -z, group, b),
        [PQ.test_nested_dequant_hand_values, PQ.test_error_bound]),
    "dequantisation ignores the width": (
        "dequant", lambda q, s, z, group, b=4: _ORIG["dequant"](q, s, z, group, 4),
        [PQ.test_nested_dequant_hand_values, PR.test_nested_layer_bits_select_planes]),
    "nibbles packed high first": ("pack_int4", _pack_reversed, [PQ.test_pack_int4_hand_values]),
    "residual planes swapped": (
        "join_planes", lambda Q2, D3, D4, K, b=4: _ORIG["join_planes"](Q2, D4, D3, K, b),
        [PQ.test_planes_hand_values, PQ.test_planes_nesting]),
    "router bias dropped": (
        "router_logits", lambda x, w_router, bias=None: _ORIG["router_logits"](x, w_router, None),
        [PR.test_router_logits_exact_products]),
    "ties to the higher index": ("topk_select", _topk_high_ties, [PR.test_topk_ties_lowest_index]),
    "gates not renormalised over the selection": (
        "gates_for", _gates_unrenormalised, [PR.test_gates_library_softmax_and_sum]),
    "unstable permutation": (
        "permute", _permute_unstable, [PR.test_permute_matches_stable_argsort, PR.test_permute_hand_example]),
    "width order of the bins reversed": (
        "assignment_keys",
        lambda sel, bits=None: (lambda k, m: (k if m is None else k - 2 * (k % 3) + 2, m))(
            *_ORIG["assignment_keys"](sel, bits)),
        [PR.test_nested_keys]),
    "SiLU without its factor v": (
        "silu", lambda v: 1.0 / (1.0 + np.exp(-v)), [PR.test_single_expert_is_dense_swiglu_torch]),
    "gate and up projections swapped": (
        "expert_ffn", lambda xr, wg, wu, wd: _ORIG["expert_ffn"](xr, wu, wg, wd),
        [PR.test_single_expert_is_dense_swiglu_torch]),
    "combine drops the last choice": (
        "combine", _combine_last_dropped, [PR.test_layer_equals_dense_masked_evaluation]),
    "combine ignores the gates": (
        "combine", lambda y_assign, gates: _ORIG["combine"](y_assign, np.ones_like(gates)),
        [PR.test_layer_equals_dense_masked_evaluation]),
    "width ties go to the wider width": (
        "bit_gate", _bit_gate_wide_ties, [PB.test_ties_go_to_the_narrower_width]),
    "bf16 by truncation": (
        "f32_to_bf16_bits",
        lambda a: (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16),
        [PQ.test_bf16_rounding_hand_values]),
    "scale and zero halves of a word swapped": (
        "sz_tiled", lambda s, z: _ORIG["sz_tiled"](z, s), [PQ.test_blob_layout_sizes_and_roundtrip]),
    "code tiles of the wrong height": (
        "tile_words", lambda words, per: _ORIG["tile_words"](words, per * 2), [PQ.test_code_tiles_hand_positions]),
}


def test_pins_pass_with_nothing_planted():
    pins = {fn for _, _, listed in MUTANTS.values() for fn in listed}
    assert _fails(sorted(pins, key=lambda f: f.__name__)) is None


@pytest.mark.parametrize("mistake", sorted(MUTANTS))
def test_a_planted_mistake_fails_a_pin(mistake, monkeypatch):
    name, mutant, pins = MUTANTS[mistake]
    monkeypatch.setattr(O, name, mutant)
    assert _fails(pins) is not None, f"no pin caught: {mistake}"
