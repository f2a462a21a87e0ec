"""Pins of the joint text + video lists (oracle/radial_mask.py, joint_*):
the composed form equals brute force over the token mask; no text reduces to
the radial lists; text query blocks are dense; every row holds the text key
blocks; the video-video part is the radial rule, pair by pair, for tokens far
from the text boundary; a planted slip (text keys left out of video rows) is
caught."""

import numpy as np
import pytest

import oracle


CASES = [  # (F, S, T, B)
    (4, 64, 16, 16),     # T a whole block
    (3, 40, 21, 16),     # nv and T both ragged, mixed block at the boundary
    (5, 48, 7, 32),      # short text inside one block
    (2, 100, 130, 64),   # text longer than a block
    (6, 33, 1, 8),       # a single text token
]


@pytest.mark.parametrize("F,S,T,B", CASES)
def test_composed_equals_bruteforce(F, S, T, B):
    rb, cb = oracle.joint_block_lists_bruteforce(F, S, T, B)
    rc, cc = oracle.joint_block_lists(F, S, T, B, method="compose")
    np.testing.assert_array_equal(rb, rc)
    np.testing.assert_array_equal(cb, cc)


@pytest.mark.parametrize("F,S,B", [(4, 64, 16), (3, 40, 16), (8, 256, 64)])
def test_no_text_is_the_radial_lists(F, S, B):
    r0, c0 = oracle.joint_block_lists(F, S, 0, B)
    r1, c1 = oracle.radial_block_lists(F, S, B)
    np.testing.assert_array_equal(r0, r1)
    np.testing.assert_array_equal(c0, c1)


@pytest.mark.parametrize("F,S,T,B", CASES)
def test_text_rows_dense_and_text_columns_everywhere(F, S, T, B):
    nv, n = F * S, F * S + T
    nb = -(-n // B)
    rp, ci = oracle.joint_block_lists(F, S, T, B)
    for qb in range(nb):
        row = set(ci[rp[qb]:rp[qb + 1]].tolist())
        if min(n, (qb + 1) * B) > nv:
            assert row == set(range(nb)), qb
        assert set(range(nv // B, nb)) <= row, qb


def test_video_part_matches_the_token_rule():
    F, S, T, B = 4, 64, 20, 16
    m = oracle.joint_token_mask(F, S, T, B)
    nv = F * S
    i = np.arange(nv)
    fi, si = i // S, i % S
    for a in range(0, nv, 7):
        for b in range(0, nv, 5):
            d = abs(fi[a] - fi[b])
            r = oracle.band_index(d)
            w = oracle.window_width(S, B, r)
            st = oracle.window_start(si[a], w, S)
            want = bool(oracle.keep_frame(d, S, B)) and st <= si[b] < st + w
            assert m[a, b] == want
    assert m[nv:].all() and m[:, nv:].all()


def test_planted_slip_is_caught():
    """Forgetting the text key blocks in video rows changes the lists."""
    F, S, T, B = 3, 40, 21, 16
    rp, ci = oracle.joint_block_lists(F, S, T, B)
    nv, n = F * S, F * S + T
    nb = -(-n // B)
    rv, cv = oracle.radial_block_lists(F, S, B)
    wrong = np.zeros((nb, nb), dtype=bool)
    for qb in range(nb):
        if min(n, (qb + 1) * B) > nv:
            wrong[qb] = True
        else:
            wrong[qb, cv[rv[qb]:rv[qb + 1]]] = True
    good = np.zeros((nb, nb), dtype=bool)
    for qb in range(nb):
        good[qb, ci[rp[qb]:rp[qb + 1]]] = True
    assert (good != wrong).any()
