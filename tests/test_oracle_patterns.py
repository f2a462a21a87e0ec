"""Pins of the tile-pattern oracle (oracle/tile_patterns.py).

Each term is checked against a closed form or a differently written brute
force: the diagonal window's row and total counts, a single off-diagonal's
entries, vertical stripes (unsorted, repeated columns), the axial term's
per-row count (n a multiple of the period) and an explicit search over the
period's multiples, the union by inclusion-exclusion, empty and inverted
terms. The seeded generic workload, drawn by vectorised code of its own,
gives the same lists from its descriptors. A planted slip (a truncating
remainder in the axial term) fails the brute-force pin.
"""

import numpy as np
import pytest

import oracle
from workloads import generic_tile_patterns, make_generic_lists


def _rows(rp, ci):
    return [ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)]


@pytest.mark.parametrize("n,w", [(1, 0), (7, 0), (16, 3), (16, 15), (16, 40), (256, 31)])
def test_diagonal_window_counts(n, w):
    rp, ci = oracle.tile_pattern_lists([{"bands": [(-w, w)]}], n)
    rows = _rows(rp, ci)
    for qb, row in enumerate(rows):
        lo, hi = max(qb - w, 0), min(qb + w, n - 1)
        assert len(row) == hi - lo + 1
        assert row == list(range(lo, hi + 1))
    if n > w:
        assert rp[-1] == n * (2 * w + 1) - w * (w + 1)
    else:
        assert rp[-1] == n * n


@pytest.mark.parametrize("o", [-20, -5, -1, 1, 6, 19, 20, 33])
def test_single_off_diagonal(o):
    n = 20
    rp, ci = oracle.tile_pattern_lists([{"bands": [(o, o)]}], n)
    assert rp[-1] == max(n - abs(o), 0)
    for qb, row in enumerate(_rows(rp, ci)):
        assert row == ([qb + o] if 0 <= qb + o < n else [])


def test_vertical_stripes_every_row():
    cols = [9, 2, 2, 30, 0, 31, 9]
    rp, ci = oracle.tile_pattern_lists([{"columns": cols}], 32)
    for row in _rows(rp, ci):
        assert row == sorted(set(cols))


@pytest.mark.parametrize("P,a", [(8, 0), (8, 1), (16, 2), (5, 2), (4, 1), (32, 0)])
def test_axial_row_count(P, a):
    n = 4 * P * 3
    rp, _ = oracle.tile_pattern_lists([{"axial": (P, a)}], n)
    counts = np.diff(rp)
    assert np.all(counts == min(2 * a + 1, P) * n // P)


def _axial_bruteforce(n, P, a):
    """Block kb is on the axial term of row qb when some multiple m*P of the
    period lies within a of kb - qb (searched explicitly, no remainder)."""
    m = np.zeros((n, n), dtype=bool)
    for qb in range(n):
        for kb in range(n):
            rel = kb - qb
            m[qb, kb] = any(abs(rel - t * P) <= a for t in range(-(n // P) - 2, n // P + 3))
    return m


@pytest.mark.parametrize("n,P,a", [(23, 8, 1), (40, 16, 0), (17, 5, 2), (9, 1, 0), (12, 6, 3)])
def test_axial_against_bruteforce(n, P, a):
    got = oracle.tile_pattern_mask({"axial": (P, a)}, n)
    np.testing.assert_array_equal(got, _axial_bruteforce(n, P, a))


def test_planted_remainder_slip_is_caught():
    """A truncating remainder (sign of the dividend) loses the tiles before
    the diagonal; the brute-force pin sees it."""
    n, P, a = 23, 8, 1
    rel = np.arange(n)[None, :] - np.arange(n)[:, None]
    r = np.fmod(rel, P)
    wrong = (r <= a) & (r >= -a) | (r >= P - a)
    assert not np.array_equal(wrong, _axial_bruteforce(n, P, a))


def test_union_inclusion_exclusion():
    n, w = 64, 4
    cols = [0, 3, 17, 40, 41, 63]
    rp, ci = oracle.tile_pattern_lists([{"bands": [(-w, w)], "columns": cols}], n)
    for qb, row in enumerate(_rows(rp, ci)):
        lo, hi = max(qb - w, 0), min(qb + w, n - 1)
        inside = sum(lo <= c <= hi for c in cols)
        assert len(row) == (hi - lo + 1) + len(cols) - inside
        assert row == sorted(row)


def test_empty_and_inverted_terms():
    rp, ci = oracle.tile_pattern_lists([{}, {"bands": [(3, 2)]}, {"columns": []}], 10)
    assert rp.tolist() == [0] * 31 and ci.size == 0


def test_dual_window_local_term_width():
    """A local window of W tiles holds W tiles in every row away from the edges."""
    n = 64
    for W in range(1, 17):
        rp, ci = oracle.tile_pattern_lists([{"bands": [(-(W // 2), W - W // 2 - 1)]}], n)
        rows = _rows(rp, ci)
        for qb in range(W, n - W):
            assert len(rows[qb]) == W and qb in rows[qb]


def test_generic_workload_descriptors_reproduce_its_lists():
    rp, ci, kinds = make_generic_lists(24, 256)
    rq, cq = oracle.tile_pattern_lists(generic_tile_patterns(24, 256), 256)
    np.testing.assert_array_equal(rp, rq)
    np.testing.assert_array_equal(ci, cq)
    assert set(kinds) == {"dual_window", "diagonal", "multi_diagonal", "stripe_diagonal"}


def test_random_descriptors_against_loops():
    """Random unions of every term, including bands outside the row, inverted
    bands and repeated columns, against a per-tile loop (the axial term by the
    explicit search over period multiples)."""
    rng = np.random.default_rng(7)
    for _ in range(30):
        n = int(rng.integers(1, 40))
        pat = {"bands": [], "axial": None, "columns": []}
        for _ in range(int(rng.integers(0, 5))):
            o, h = int(rng.integers(-n - 3, n + 3)), int(rng.integers(-2, 6))
            pat["bands"].append((o - h, o + h))
        if rng.random() < 0.6:
            pat["axial"] = (int(rng.integers(1, 12)), int(rng.integers(0, 4)))
        if rng.random() < 0.6:
            pat["columns"] = rng.integers(0, n, size=int(rng.integers(0, 6))).tolist()
        want = np.zeros((n, n), dtype=bool)
        ax = _axial_bruteforce(n, *pat["axial"]) if pat["axial"] else np.zeros((n, n), bool)
        for qb in range(n):
            for kb in range(n):
                want[qb, kb] = (any(lo <= kb - qb <= hi for lo, hi in pat["bands"])
                                or ax[qb, kb] or kb in pat["columns"])
        np.testing.assert_array_equal(oracle.tile_pattern_mask(pat, n), want)
