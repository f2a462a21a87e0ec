"""Pins for the oracle's radial mask (CPU only).

Each check ties the oracle to something other than itself: hand-derived rows
(tests/golden), the properties the pages state (dense diagonal band, density
halving per doubling of temporal distance, a spatial window that shrinks with
temporal distance, O(n log n) block count), and a second, independent block
construction.
"""

import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_band_index_hand_values():
    # floor(log2(max(d, 1))): band 0 holds d = 0 and d = 1.
    assert [oracle.band_index(d) for d in (0, 1, 2, 3, 4, 7, 8, 15, 16, 1023, 1024)] == \
        [0, 0, 1, 1, 2, 2, 3, 3, 4, 9, 10]
    arr = oracle.band_index(np.array([0, 1, 2, 5, 9, 40]))
    assert arr.tolist() == [0, 0, 1, 2, 3, 5]


def test_r_star_hand_values():
    # The window S >> r shrinks until it would hold fewer than one block.
    assert oracle.r_star(1560, 128) == 3   # 1560>>3 = 195 >= 128, 1560>>4 = 97
    assert oracle.r_star(3600, 128) == 4   # 3600>>4 = 225, 3600>>5 = 112
    assert oracle.r_star(256, 64) == 2
    assert oracle.r_star(255, 64) == 1
    assert oracle.r_star(96, 64) == 0
    assert oracle.r_star(32, 64) == 0      # S < B: no shrinking at all


def _load_golden_rows(path):
    rows = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        q, iv = line.split(":")
        keys = set()
        for tok in iv.split():
            lo, hi = map(int, tok.split("-"))
            keys |= set(range(lo, hi))
        rows[int(q)] = keys
    return rows


def test_golden_rows_hand_derived():
    F, S, B = 20, 8, 4
    mask = oracle.radial_token_mask(F, S, B)
    rows = _load_golden_rows(os.path.join(GOLDEN, "radial_rows_F20_S8_B4.txt"))
    assert len(rows) == 3
    for i, keys in rows.items():
        assert set(np.nonzero(mask[i])[0].tolist()) == keys, f"query token {i}"


GRIDS = [(1, 64, 16), (2, 64, 64), (3, 96, 64), (5, 255, 64), (8, 256, 64),
         (17, 16, 32), (6, 48, 16), (9, 100, 32), (12, 64, 16), (4, 256, 64)]


@pytest.mark.parametrize("F,S,B", GRIDS)
def test_dense_diagonal_band(F, S, B):
    mask = oracle.radial_token_mask(F, S, B)
    f = np.arange(F * S) // S
    near = np.abs(f[:, None] - f[None, :]) <= 1
    assert mask[near].all()


@pytest.mark.parametrize("F,S,B", GRIDS)
def test_window_is_local_contiguous_and_shrinks(F, S, B):
    mask = oracle.radial_token_mask(F, S, B).reshape(F, S, F, S)
    for fi in range(F):
        for si in range(S):
            widths = {}
            for fj in range(F):
                sel = np.nonzero(mask[fi, si, fj])[0]
                if sel.size == 0:
                    continue
                # one contiguous run of keys that contains the query's own position
                assert sel[-1] - sel[0] + 1 == sel.size
                assert sel[0] <= si <= sel[-1]
                widths.setdefault(abs(fi - fj), sel.size)
                assert widths[abs(fi - fj)] == sel.size
            ds = sorted(widths)
            assert all(widths[a] >= widths[b] for a, b in zip(ds, ds[1:]))


@pytest.mark.parametrize("F,S,B", [(40, 64, 16), (33, 96, 16), (24, 64, 8), (34, 32, 8)])
def test_density_halves_per_band(F, S, B):
    """Per query and per side, a band fully inside the video has density exactly 2^-r."""
    rs = oracle.r_star(S, B)
    assert S % (1 << rs) == 0
    mask = oracle.radial_token_mask(F, S, B).reshape(F, S, F, S)
    per_frame = mask.sum(axis=3)          # [F, S, F]: admitted keys per key frame
    checked = 0
    for fi in range(F):
        for side in (-1, 1):
            r = 1
            while True:
                ds = range(1 << r, 1 << (r + 1))
                frames = [fi + side * d for d in ds]
                if not all(0 <= f < F for f in frames):
                    break
                got = per_frame[fi][:, frames].sum(axis=1) / ((1 << r) * S)
                assert np.all(got == 2.0 ** -r), (fi, side, r, got[:4])
                checked += 1
                r += 1
    assert checked > 0


@pytest.mark.parametrize("F,S,B", GRIDS + [(31, 64, 16), (64, 32, 16), (7, 255, 16)])
def test_two_block_constructions_agree(F, S, B):
    rp1, ci1 = oracle.radial_block_lists_bruteforce(F, S, B)
    rp2, ci2 = oracle.radial_block_lists_intervals(F, S, B)
    assert np.array_equal(rp1, rp2) and np.array_equal(ci1, ci2)
    nb = -(-F * S // B)
    assert rp1.size == nb + 1 and rp1[0] == 0
    for r in range(nb):
        row = ci1[rp1[r]:rp1[r + 1]]
        assert np.all(np.diff(row) > 0) and (row.size == 0 or (row[0] >= 0 and row[-1] < nb))


def test_block_lists_are_exact_cover():
    F, S, B = 9, 100, 32
    mask = oracle.radial_token_mask(F, S, B)
    rp, ci = oracle.block_lists_from_token_mask(mask, B)
    n = F * S
    nb = -(-n // B)
    for qb in range(nb):
        row = set(ci[rp[qb]:rp[qb + 1]].tolist())
        blk = mask[qb * B:min(n, (qb + 1) * B)]
        for kb in range(nb):
            has = blk[:, kb * B:min(n, (kb + 1) * B)].any()
            assert has == (kb in row)


def _upper_bound_per_row(S, B, F):
    """Blocks a query-block row can touch, from the rule: O(log F) for fixed S, B."""
    rs = oracle.r_star(S, B)
    qframes = -(-B // S) + 1
    per_window = lambda w: -(-(w + B - 1) // B) + 1
    total = 3 * per_window(S)
    for r in range(1, max(1, int(math.log2(max(F, 2)))) + 1):
        w = max(1, S >> min(r, rs))
        kept = 2 * ((1 << r) if r <= rs else (1 << rs))
        total += kept * per_window(w)
    return qframes * total


def test_block_count_grows_n_log_n():
    S, B = 256, 64
    nnz, dens = {}, {}
    for F in (2, 4, 8, 16, 32, 64, 128, 256, 512):
        rp, _ = oracle.radial_block_lists_intervals(F, S, B)
        nqb = rp.size - 1
        nnz[F] = int(rp[-1])
        dens[F] = nnz[F] / nqb ** 2
        assert nnz[F] <= nqb * _upper_bound_per_row(S, B, F)
    Fs = sorted(nnz)
    assert all(dens[a] >= dens[b] for a, b in zip(Fs, Fs[1:]))
    # Quadratic growth would give 4x per doubling of F; n log n tends to 2x.
    ratios = [nnz[2 * F] / nnz[F] for F in Fs[1:-1]]
    assert all(a > b for a, b in zip(ratios, ratios[1:]))
    assert ratios[-1] < 2.4
    assert dens[512] < 0.08


@pytest.mark.parametrize("F,S,B,nnz,rmin,rmax", [
    (4, 256, 64, 220, 12, 15),
    (21, 1560, 128, 31248, 85, 168),
    (33, 3600, 128, 272376, 200, 458),
    (84, 1560, 128, 230963, 122, 304),
])
def test_independent_block_counts(F, S, B, nnz, rmin, rmax):
    """Counts predicted by a separate brute-force script written from the same rule."""
    rp, _ = oracle.radial_block_lists(F, S, B)
    counts = np.diff(rp)
    assert int(rp[-1]) == nnz
    assert counts.max() == rmax
    assert counts.min() == rmin
