"""The diagonal enumeration, pinned by brute force and a hand-written table.

Source: skill page "Diagonal Batching for Recurrent Memory Transformers", "Implementation"
(the diagonal scheduler) and "Architecture Overview" (dependency preservation): the
(layer, segment) grid is swept along anti-diagonals d = l + s, and cell (l, s) needs
(l-1, s) and (l, s-1) to have run first.
"""
import itertools
import os

import numpy as np
import pytest

from oracle import armt

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_force_diagonals(L, S):
    """Group all L*S cells by l+s, each group in ascending l -- no diagonal-index loop."""
    cells = sorted(itertools.product(range(L), range(S)), key=lambda c: (c[0] + c[1], c[0]))
    groups = {}
    for l, s in cells:
        groups.setdefault(l + s, []).append((l, s))
    return [groups[k] for k in sorted(groups)]


@pytest.mark.parametrize("L,S", [(L, S) for L in range(1, 13) for S in range(1, 13)])
def test_diagonals_brute_force(L, S):
    diags = armt.diagonals(L, S)
    assert diags == brute_force_diagonals(L, S)
    assert len(diags) == L + S - 1
    flat = [c for d in diags for c in d]
    assert len(flat) == L * S and len(set(flat)) == L * S
    where = {c: i for i, d in enumerate(diags) for c in d}
    for (l, s), i in where.items():
        assert l + s == i
        if l > 0:
            assert where[(l - 1, s)] == i - 1
        if s > 0:
            assert where[(l, s - 1)] == i - 1
        # at most one cell per layer on a diagonal (layer state is updated in place)
    for d in diags:
        ls = [l for l, _ in d]
        assert ls == sorted(ls) and len(set(ls)) == len(ls)
    # size of diagonal d (a count of lattice points on the line l + s = d inside the grid)
    sizes = [len(d) for d in diags]
    for i, n in enumerate(sizes):
        assert n == sum(1 for l in range(L) if 0 <= i - l < S)


def test_diagonals_golden_table():
    rows = np.loadtxt(os.path.join(GOLDEN, "schedule_L3_S4.txt"), dtype=np.int32, comments="#")
    np.testing.assert_array_equal(armt.schedule_triples(3, 4, "diagonal"), rows)


def test_sequential_steps():
    t = armt.schedule_triples(3, 2, "sequential")
    np.testing.assert_array_equal(t, [[0, 0, 0], [1, 1, 0], [2, 2, 0], [3, 0, 1], [4, 1, 1], [5, 2, 1]])


def test_bf16_rounding_of_the_input_generator():
    """The fast (torch) rounding used for inputs equals round-to-nearest-even on the bits."""
    from armt_synthetic import bf16_bits, bf16_bits_to_f32, round_to_bf16
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * s for s in (1e-3, 1.0, 1e3)])
    x = np.concatenate([x, np.array([0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], np.float32)])
    np.testing.assert_array_equal(round_to_bf16(x).view(np.uint32), bf16_bits_to_f32(bf16_bits(x)).view(np.uint32))
    # ties go to even: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7
    assert round_to_bf16(np.array([1.0 + 2.0 ** -8], np.float32))[0] == 1.0


def brute_force_batch(L, S):
    """All cells (b, l, s) of a batch grouped by l + s, each group ordered by (l, b)."""
    cells = [(b, l, s) for b, n in enumerate(S) for l in range(L) for s in range(n)]
    cells.sort(key=lambda c: (c[1] + c[2], c[1], c[0]))
    groups = {}
    for b, l, s in cells:
        groups.setdefault(l + s, []).append((b, l, s))
    return [groups[k] for k in sorted(groups)]


@pytest.mark.parametrize("S", [[1], [3, 1], [2, 5, 2], [4, 4], [1, 1, 1, 7]])
@pytest.mark.parametrize("L", [1, 2, 5])
def test_batch_diagonals_brute_force(L, S):
    q = armt.schedule_quads(L, S, "diagonal")
    got = [[tuple(r[1:]) for r in q if r[0] == t] for t in range(q[:, 0].max() + 1)]
    assert got == brute_force_batch(L, S)
    assert len(q) == L * sum(S) and len({tuple(r[1:]) for r in q}) == len(q)
    where = {tuple(r[1:]): r[0] for r in q}
    for (b, l, s), t in where.items():
        if l > 0:
            assert where[(b, l - 1, s)] < t
        if s > 0:
            assert where[(b, l, s - 1)] < t
    # at most one cell per (sequence, layer) in a step: each state is updated in place
    for t in range(q[:, 0].max() + 1):
        bl = [(r[1], r[2]) for r in q if r[0] == t]
        assert len(set(bl)) == len(bl)
    # one sequence: the single-sequence schedule with a zero sequence column
    if len(S) == 1:
        np.testing.assert_array_equal(q[:, [0, 2, 3]], armt.schedule_triples(L, S[0], "diagonal"))


def test_batch_sequential_order():
    q = armt.schedule_quads(2, [2, 1], "sequential")
    np.testing.assert_array_equal(q, [[0, 0, 0, 0], [1, 0, 1, 0], [2, 0, 0, 1], [3, 0, 1, 1], [4, 1, 0, 0], [5, 1, 1, 0]])
