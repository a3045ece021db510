"""Pins of the oracle's bit-width router (D2MoE, Dual Routing: the bit
gate next to the expert gate) by construction: cases whose winning width is
known without evaluating the gate, an invariance of the arg-max, the
per-expert lookup and the tie rule."""
import numpy as np

from oracle import moe_oracle as O


def test_width_follows_the_sign_of_a_designed_direction():
    # W_bit[e, c] = (c - 1) * u: scores (-a, 0, a) with a = x . u, so the
    # width is 4 when a > 0, 2 when a < 0, and 2 (tie of all three) at a = 0
    d, E = 7, 5
    u = np.zeros(d)
    u[2] = 1.0
    w = np.stack([np.stack([(c - 1) * u for c in range(3)]) for _ in range(E)]).astype(np.float32)
    x = np.zeros((3, d))
    x[0, 2], x[1, 2], x[2, 2] = 1.5, -0.25, 0.0
    sel = np.array([[0, 4], [1, 3], [2, 0]], dtype=np.int32)
    assert O.bit_gate(x, w, None, sel).tolist() == [[4, 4], [2, 2], [2, 2]]


def test_bias_alone_decides_and_is_looked_up_per_expert():
    # expert e prefers width 2 + (e % 3); which expert sits in which slot j
    # must not matter
    d, E, T, k = 6, 7, 9, 3
    rng = np.random.default_rng(1)
    w = np.zeros((E, 3, d), np.float32)
    bias = np.full((E, 3), -1.0, np.float32)
    for e in range(E):
        bias[e, e % 3] = 1.0
    x = rng.normal(size=(T, d))
    sel = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    assert (O.bit_gate(x, w, bias, sel) == 2 + sel % 3).all()


def test_shift_common_to_all_widths_changes_nothing():
    # adding one vector r to the three rows of an expert adds x . r to all
    # three scores: the arg-max cannot move
    rng = np.random.default_rng(2)
    d, E, T, k = 33, 6, 40, 2
    w = rng.normal(0, 0.02, (E, 3, d)).astype(np.float32)
    r = rng.normal(0, 1.0, (E, 1, d)).astype(np.float32)
    bias = rng.normal(0, 0.01, (E, 3)).astype(np.float32)
    x = rng.normal(size=(T, d)).astype(np.float32)
    sel = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    a = O.bit_gate(x, w, bias, sel)
    b = O.bit_gate(x, (w.astype(np.float64) + r).astype(np.float64), bias, sel)
    assert (a == b).all()
    assert set(np.unique(a).tolist()) == {2, 3, 4}  # the random gate uses every width


def test_ties_go_to_the_narrower_width():
    d, E = 4, 2
    w = np.zeros((E, 3, d), np.float32)
    w[1, 1] = w[1, 2] = np.array([1.0, 0, 0, 0])   # widths 3 and 4 tie for expert 1
    x = np.array([[2.0, 0, 0, 0]])
    assert O.bit_gate(x, w, None, np.array([[1, 0]], np.int32)).tolist() == [[3, 2]]


def test_identical_rows_tie_exactly_at_full_length():
    # two identical width rows of a realistic length (d = 4096, random
    # values): the two scores are the same number, so the narrower width wins
    # every time (a blocked dot product may round identical rows apart)
    rng = np.random.default_rng(4)
    d, E, T = 4096, 4, 64
    w = rng.normal(0, 0.02, (E, 3, d)).astype(np.float32)
    w[:, 2] = w[:, 1]
    bias = np.zeros((E, 3), np.float32)
    bias[:, 0] = -100.0  # width 2 never wins
    x = rng.normal(size=(T, d)).astype(np.float32)
    sel = np.stack([rng.permutation(E)[:2] for _ in range(T)]).astype(np.int32)
    assert (O.bit_gate(x, w, bias, sel) == 3).all()
