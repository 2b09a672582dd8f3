"""Pins of the oracle's MoE steps (route, permute, combine) against what the
definitions fix: brute force on tiny cases, the inverse-permutation property,
counting, and linearity of the combine."""
import itertools

import numpy as np
import pytest

from oracle import moe


def _brute_route(ids, E):
    """Rows by enumeration: for each expert in order, its pairs in ascending p."""
    rows = [p for e in range(E) for p in range(len(ids)) if ids[p] == e]
    dest = [-1] * len(ids)
    for r, p in enumerate(rows):
        dest[p] = r
    return rows, dest


@pytest.mark.parametrize("ids,E", [([2, 0, 2, 1, 0], 3), ([0], 1), ([1, 1, 1], 4),
                                   ([3, 3, 0, 0, 2, 2, 1, 1], 4), ([], 5)])
def test_route_equals_brute_force(ids, E):
    off, dest, src = moe.route(ids, E)
    rows, bdest = _brute_route(ids, E)
    assert list(dest) == bdest
    assert list(src[:len(rows)]) == rows
    assert off[0] == 0 and off[-1] == len(ids)
    for e in range(E):
        assert off[e + 1] - off[e] == sum(1 for i in ids if i == e)


def test_route_every_small_case():
    for P in range(0, 5):
        for ids in itertools.product(range(3), repeat=P):
            off, dest, src = moe.route(list(ids), 3)
            rows, bdest = _brute_route(list(ids), 3)
            assert list(dest) == bdest and list(src) == rows


def test_route_is_a_stable_permutation():
    rng = np.random.default_rng(0)
    ids = rng.integers(0, 16, size=3000)
    off, dest, src = moe.route(ids, 16)
    assert sorted(dest) == list(range(3000))
    assert np.array_equal(src[dest], np.arange(3000))
    for e in range(16):
        seg = src[off[e]:off[e + 1]]
        assert np.all(ids[seg] == e) and np.all(np.diff(seg) > 0)


def test_route_leaves_out_bad_ids():
    off, dest, src = moe.route([0, 5, 1, -1, 0], 2)
    assert list(off) == [0, 2, 3]
    assert list(dest) == [0, -1, 2, -1, 1]


def test_permute_then_gather_back_is_identity():
    rng = np.random.default_rng(1)
    T, k, E = 50, 3, 7
    ids = rng.integers(0, E, size=(T, k))
    x = rng.integers(0, 256, size=(T, 48), dtype=np.uint8)
    off, dest, src = moe.route(ids, E)
    g = moe.permute_rows(x, src, k)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(g[dest[t * k + j]], x[t])


def test_combine_unit_weights_k1_is_the_inverse_permutation():
    rng = np.random.default_rng(2)
    T, E, N = 40, 5, 16
    ids = rng.integers(0, E, size=T)
    off, dest, src = moe.route(ids, E)
    Yg = rng.standard_normal((T, N))
    Y = moe.combine(Yg, dest, None, T, 1)
    assert np.array_equal(Y, Yg[dest])


def test_combine_is_linear_in_the_weights():
    rng = np.random.default_rng(3)
    T, k, E, N = 30, 2, 4, 8
    ids = rng.integers(0, E, size=(T, k))
    off, dest, src = moe.route(ids, E)
    Yg = rng.standard_normal((T * k, N))
    w1, w2 = rng.random((T, k)), rng.random((T, k))
    a = moe.combine(Yg, dest, w1 + 2 * w2, T, k)
    b = moe.combine(Yg, dest, w1, T, k) + 2 * moe.combine(Yg, dest, w2, T, k)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)
    # a token's output is the weighted sum of its own k rows, written out by hand
    t = 7
    ref = sum(w1[t, j] * Yg[dest[t * k + j]] for j in range(k))
    assert np.allclose(moe.combine(Yg, dest, w1, T, k)[t], ref, rtol=0, atol=0)
