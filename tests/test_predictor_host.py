"""Host-side checks of the next-layer expert predictor (moe_predictor_*),
which is plain host bookkeeping: counts of (expert at layer l-1, expert at
layer l) pairs at the same token and choice, and a ranking of layer l's
experts by the summed conditional frequencies.  Checked against a direct
numpy statement of that ranking on random observations, and on the
successor-table traces the offload workload uses."""
import ctypes

import numpy as np
import pytest

from quantized_moe_expert_histogram_b200 import build, inputs as I, moeq


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moeq.open_library()


def _create(lib, layers, E):
    h = ctypes.c_void_p()
    assert lib.moe_predictor_create(layers, E, ctypes.byref(h)) == 0
    return h


def _arr(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _predict(lib, h, layer, prev, max_out, min_score=0.0):
    prev, pp = _arr(prev)
    out = np.zeros(max(1, max_out), dtype=np.int32)
    n = ctypes.c_int32(0)
    assert lib.moe_predictor_predict(h, layer, None, pp, prev.shape[0], prev.shape[1], max_out, ctypes.c_double(min_score),
                                     out.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)) == 0
    return out[:n.value].tolist()


def test_predict_matches_direct_ranking(lib):
    rng = np.random.default_rng(0)
    L, E, k = 3, 16, 4
    h = _create(lib, L, E)
    counts = np.zeros((L, E, E), dtype=np.int64)
    for _ in range(40):
        layer = int(rng.integers(1, L))
        prev = rng.integers(0, E, size=(5, k))
        cur = rng.integers(0, E, size=(5, k))
        (p, pp), (c, cp) = _arr(prev), _arr(cur)
        assert lib.moe_predictor_observe(h, layer, None, pp, cp, 5, k) == 0
        np.add.at(counts[layer], (prev.reshape(-1), cur.reshape(-1)), 1)
    for layer in (1, 2):
        prev = rng.integers(0, E, size=(3, k))
        rows = counts[layer][prev.reshape(-1)]
        sums = rows.sum(axis=1, keepdims=True)
        score = np.where(sums > 0, rows / np.maximum(sums, 1), 0.0).sum(axis=0)
        expect = [int(e) for e in sorted(np.nonzero(score > 0)[0], key=lambda e: (-score[e], e))][:6]
        assert _predict(lib, h, layer, prev, 6) == expect
        keep = [int(e) for e in sorted(np.nonzero(score >= 0.75)[0], key=lambda e: (-score[e], e))][:6]
        assert _predict(lib, h, layer, prev, 6, 0.75) == keep
    lib.moe_predictor_destroy(h)


def test_predictor_learns_successor_table(lib):
    """On the offload trace (70% of choices follow a per-layer successor
    table), after a few steps the predicted set covers most of the next
    layer's experts."""
    E, k, L, steps, batch = 64, 8, 4, 40, 8
    trace = I.make_slot_trace(E, k, L, steps, batch, seed=2).numpy()
    h = _create(lib, L, E)
    covered = total = 0
    for s in range(steps):
        for l in range(1, L):
            if s >= steps // 2:
                pred = set(_predict(lib, h, l, trace[s, l - 1], 32))
                need = set(trace[s, l].reshape(-1).tolist())
                covered += len(need & pred)
                total += len(need)
            (p, pp), (c, cp) = _arr(trace[s, l - 1]), _arr(trace[s, l])
            assert lib.moe_predictor_observe(h, l, None, pp, cp, batch, k) == 0
    assert covered / total > 0.6
    lib.moe_predictor_destroy(h)


def test_predictor_rejects_bad_arguments(lib):
    h = _create(lib, 2, 8)
    prev, pp = _arr([[0, 9]])
    cur, cp = _arr([[1, 2]])
    assert lib.moe_predictor_observe(h, 1, None, pp, cp, 1, 2) != 0  # id 9 >= E
    assert lib.moe_predictor_observe(h, 0, None, cp, cp, 1, 2) != 0  # layer 0 has no predecessor
    assert lib.moe_predictor_observe(h, 1, cp, cp, cp, 1, 2) != 0  # layer 1 has no second predecessor
    lib.moe_predictor_destroy(h)


def _predict2(lib, h, layer, prev2, prev, max_out):
    (p2, pp2), (p, pp) = _arr(prev2), _arr(prev)
    out = np.zeros(max(1, max_out), dtype=np.int32)
    n = ctypes.c_int32(0)
    assert lib.moe_predictor_predict(h, layer, pp2, pp, p.shape[0], p.shape[1], max_out, ctypes.c_double(0.0),
                                     out.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)) == 0
    return out[:n.value].tolist()


def test_pair_key_ranking_and_back_off(lib):
    """Two-layer key: the ranking equals a direct numpy statement that uses a
    pair's counts when it was seen at least twice and the one-layer counts
    otherwise."""
    rng = np.random.default_rng(5)
    L, E, k = 4, 8, 2
    h = _create(lib, L, E)
    c1 = np.zeros((L, E, E), np.int64)
    c2 = np.zeros((L, E, E, E), np.int64)
    for _ in range(60):
        layer = int(rng.integers(2, L))
        p2, p1, cur = (rng.integers(0, E, size=(3, k)) for _ in range(3))
        (a2, pa2), (a1, pa1), (c, pc) = _arr(p2), _arr(p1), _arr(cur)
        assert lib.moe_predictor_observe(h, layer, pa2, pa1, pc, 3, k) == 0
        np.add.at(c1[layer], (p1.reshape(-1), cur.reshape(-1)), 1)
        np.add.at(c2[layer], (p2.reshape(-1), p1.reshape(-1), cur.reshape(-1)), 1)
    for layer in (2, 3):
        p2, p1 = rng.integers(0, E, size=(4, k)), rng.integers(0, E, size=(4, k))
        score = np.zeros(E)
        for a2, a1 in zip(p2.reshape(-1), p1.reshape(-1)):
            row = c2[layer, a2, a1] if c2[layer, a2, a1].sum() >= 2 else c1[layer, a1]
            if row.sum():
                score += row / row.sum()
        expect = [int(e) for e in sorted(np.nonzero(score > 0)[0], key=lambda e: (-score[e], e))][:5]
        assert _predict2(lib, h, layer, p2, p1, 5) == expect
    lib.moe_predictor_destroy(h)


def test_pair_key_predicts_a_second_order_path(lib):
    """Paths where the next expert depends on the two previous ones
    (b = (c + 3 a) mod E) and not on the previous one alone: the pair key
    names the right expert; the one-layer key cannot single it out."""
    E, k, L = 16, 1, 3
    h = _create(lib, L, E)
    for rep in range(3):  # every pair three times
        for c, a in ((c, a) for c in range(E) for a in range(E)):
            b = (c + 3 * a) % E
            (x2, p2), (x1, p1), (x0, p0) = _arr([[c]]), _arr([[a]]), _arr([[b]])
            assert lib.moe_predictor_observe(h, 2, p2, p1, p0, 1, k) == 0
    hits2 = hits1 = 0
    for c in range(E):
        for a in range(E):
            b = (c + 3 * a) % E
            hits2 += _predict2(lib, h, 2, [[c]], [[a]], 1) == [b]
            hits1 += _predict(lib, h, 2, [[a]], 1) == [b]
    assert hits2 == E * E
    assert hits1 <= 0.2 * E * E
    lib.moe_predictor_destroy(h)
