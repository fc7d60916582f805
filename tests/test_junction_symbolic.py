"""The junction plan's symbolic phase (host C++, no device) against the
oracle's own elimination: the minimum-degree order and the filled pattern S
must agree bit for bit on lattices, random patterns, trees, given orders and
edge cases."""
import numpy as np
import pytest

import oracle
from sparse_spd_selected_b200 import build, inputs, selinv


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def random_pattern(n, m, seed):
    rng = np.random.default_rng(seed)
    pairs = sorted({(max(a, c), min(a, c)) for a, c in rng.integers(0, n, (m, 2)) if a != c})
    return np.array(pairs, dtype=np.int64).T.reshape(2, -1)


CASES = [
    ("grid_3x3", 9, inputs.grid_edges(3, 3), None),
    ("grid_7x5", 35, inputs.grid_edges(7, 5), None),
    ("grid_12x12", 144, inputs.grid_edges(12, 12), None),
    ("random_40", 40, random_pattern(40, 90, 1), None),
    ("random_100_dense", 100, random_pattern(100, 600, 2), None),
    ("grid_6x6_reversed", 36, inputs.grid_edges(6, 6), np.arange(36)[::-1].copy()),
    ("random_30_shuffled", 30, random_pattern(30, 60, 3), np.random.default_rng(4).permutation(30)),
    ("no_edges", 5, np.zeros((2, 0), dtype=np.int64), None),
    ("single", 1, np.zeros((2, 0), dtype=np.int64), None),
    ("star", 9, np.array([[1, 2, 3, 4, 5, 6, 7, 8], [0] * 8]), None),
]


@pytest.mark.parametrize("name,n,E,order", CASES, ids=[c[0] for c in CASES])
def test_symbolic_matches_oracle(name, n, E, order):
    o, S = selinv.junction_symbolic(n, E, order)
    o_ref, S_ref = oracle.junction_symbolic(n, E, order)
    assert o.tolist() == o_ref.tolist()
    assert np.array_equal(S, S_ref)


def test_tree_pattern_has_no_fill():
    parent = inputs.random_parent(np.random.default_rng(9), 200)
    E = np.array([[max(v, p) for v, p in enumerate(parent) if p >= 0],
                  [min(v, p) for v, p in enumerate(parent) if p >= 0]])
    _, S = selinv.junction_symbolic(200, E)
    assert S.shape[1] == E.shape[1]
