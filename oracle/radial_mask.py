"""Oracle: the radial attention mask, token level and block level.

TEST INFRASTRUCTURE ONLY (see the package docstring). Plain NumPy; written
to be checked by eye against the rule below, not to be fast.

The rule (page tags are defined in ``oracle/__init__.py``):

1. Tokens are frame-major: token ``i`` sits in frame ``i // S`` at in-frame
   position ``i % S`` ([RA-skill] Step 1, frame/spatial index of each token).
2. The temporal distance ``d = |f_i - f_j|`` falls in band
   ``r = floor(log2(max(d, 1)))`` ([RA-skill] Step 1, ``should_attend_radial``;
   the ``max(., 1)`` guard is garbled on the page and read as written here, so
   band 0 holds d = 0 and d = 1).
3. Compute density halves each time the temporal distance doubles, with decay
   0.5 ([RA-blog] "How Radial Attention Works", first bullet; [RA-skill]
   hyper-parameter table, "0.5 is standard"), and each token attends to
   spatially nearby tokens through a window that shrinks for distant frames
   ([RA-blog], second bullet; [RA-summary] "Outline").

   Reading taken where the pages leave the step open: the spatial distance is
   the 1-D in-frame index distance; band ``r`` keeps a window of exactly
   ``S >> r`` keys centred on the query's in-frame index and clamped inside the
   frame; once a window would be narrower than one block (``r > r*`` with
   ``r* = max{r : S >> r >= B}``, or 0 when ``S < B``) the window stops
   shrinking at ``S >> r*`` and the density keeps halving by keeping only the
   frames whose distance is a multiple of ``2^(r - r*)``.
4. The mask runs at block granularity ([RA-blog], third bullet, 128x128
   blocks): block ``(qb, kb)`` is active when at least one admitted token pair
   falls inside it.
"""

from __future__ import annotations

import numpy as np


def band_index(d):
    """Temporal band ``floor(log2(max(d, 1)))`` for integer distances ``d >= 0``.

    [RA-skill] Step 1, ``should_attend_radial`` (band from log2 of the distance).
    Works on Python ints and on integer NumPy arrays. ``np.frexp`` returns the
    exact binary exponent of an integer held in float64, so this is exact.
    """
    d = np.maximum(np.asarray(d, dtype=np.int64), 1)
    _, e = np.frexp(d.astype(np.float64))
    r = (e - 1).astype(np.int64)
    return int(r) if r.ndim == 0 else r


def r_star(S: int, B: int) -> int:
    """Last band whose window ``S >> r`` still holds at least one block of ``B`` keys.

    Returns 0 when ``S < B`` (the dense band is then the only unthinned band).
    Reading of [RA-skill] hyper-parameter table ("minimum density") and
    [RA-blog] (128x128 blocks): the window stops shrinking at one block.
    """
    if S < B:
        return 0
    r = 0
    while (S >> (r + 1)) >= B:
        r += 1
    return r


def window_width(S: int, B: int, r):
    """Keys a query attends in one kept frame of band ``r``: ``max(1, S >> min(r, r*))``.

    Density ``decay**band`` with decay 0.5 ([RA-skill] Step 1 ``density``;
    [RA-skill] table "0.5 is standard"; [RA-blog] "density halving").
    """
    rs = r_star(S, B)
    r = np.minimum(np.asarray(r, dtype=np.int64), rs)
    w = np.maximum(1, np.right_shift(np.int64(S), r))
    return int(w) if w.ndim == 0 else w


def keep_frame(d, S: int, B: int):
    """Whether a key frame at temporal distance ``d`` is attended at all.

    Bands up to ``r*`` keep every frame; beyond it only frames whose distance is
    a multiple of ``2^(r - r*)`` (so density keeps halving per band once the
    window is one block wide).
    """
    d = np.asarray(d, dtype=np.int64)
    r = np.asarray(band_index(d), dtype=np.int64)
    rs = r_star(S, B)
    step = np.left_shift(np.int64(1), np.maximum(r - rs, 0))
    k = (r <= rs) | (np.mod(d, step) == 0)
    return bool(k) if k.ndim == 0 else k


def window_start(si, w, S: int):
    """First in-frame key index of a width-``w`` window centred on ``si``, clamped into the frame."""
    st = np.asarray(si, dtype=np.int64) - np.asarray(w, dtype=np.int64) // 2
    st = np.clip(st, 0, S - np.asarray(w, dtype=np.int64))
    return int(st) if np.ndim(st) == 0 else st


def radial_token_mask(F: int, S: int, B: int) -> np.ndarray:
    """Dense ``[n, n]`` boolean mask, ``n = F*S``, each element from the token rule.

    Brute force: every (i, j) pair is evaluated from the definition. Use only
    on tiny grids (``n`` up to a few thousand).
    """
    n = F * S
    j = np.arange(n, dtype=np.int64)
    fj = j // S
    sj = j % S
    mask = np.zeros((n, n), dtype=bool)
    for i in range(n):
        fi, si = divmod(i, S)
        d = np.abs(fi - fj)
        r = band_index(d)
        w = window_width(S, B, r)
        st = window_start(si, w, S)
        mask[i] = keep_frame(d, S, B) & (st <= sj) & (sj < st + w)
    return mask


def block_lists_from_token_mask(mask: np.ndarray, B: int):
    """Reduce a token mask to per-query-block sorted key-block lists (CSR).

    Block ``(qb, kb)`` is active when any admitted pair falls inside it
    ([RA-blog], block sparsity at block granularity). Returns ``(row_ptr,
    col_idx)`` as int32 arrays; ``row_ptr`` has ``nqb + 1`` entries.
    """
    n = mask.shape[0]
    nb = -(-n // B)
    pad = np.zeros((nb * B, nb * B), dtype=bool)
    pad[:n, :n] = mask
    active = pad.reshape(nb, B, nb, B).any(axis=(1, 3))
    return _csr_from_dense(active)


def _csr_from_dense(active: np.ndarray):
    counts = active.sum(axis=1)
    row_ptr = np.zeros(active.shape[0] + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    _, cols = np.nonzero(active)  # row-major, so each row's columns ascend
    return row_ptr.astype(np.int32), cols.astype(np.int32)


def radial_block_lists_bruteforce(F: int, S: int, B: int):
    """Block lists from the brute-force token mask (tiny grids only)."""
    return block_lists_from_token_mask(radial_token_mask(F, S, B), B)


def radial_block_lists_intervals(F: int, S: int, B: int):
    """Block lists from per-token key intervals, for grids too big for the token mask.

    For each query token ``i`` and key frame ``f_j`` the admitted keys form the
    interval ``[f_j*S + st, f_j*S + st + w)``; every block the interval touches
    is active for ``i``'s query block. Coverage is accumulated per query block
    with a difference array, one query frame at a time.
    """
    n = F * S
    nb = -(-n // B)
    diff = np.zeros((nb, nb + 1), dtype=np.int64)
    si = np.arange(S, dtype=np.int64)
    fj = np.arange(F, dtype=np.int64)
    for fi in range(F):
        d = np.abs(fi - fj)                       # [F]
        r = np.asarray(band_index(d))
        w = np.asarray(window_width(S, B, r))      # [F]
        keep = np.asarray(keep_frame(d, S, B))     # [F]
        st = window_start(si[:, None], w[None, :], S)   # [S, F]
        lo = fj[None, :] * S + st
        hi = lo + w[None, :]                       # exclusive
        qb = np.broadcast_to(((fi * S + si) // B)[:, None], lo.shape)
        sel = np.broadcast_to(keep[None, :], lo.shape)
        qb, lo_b, hi_b = qb[sel], lo[sel] // B, (hi[sel] - 1) // B
        np.add.at(diff, (qb, lo_b), 1)
        np.add.at(diff, (qb, hi_b + 1), -1)
    active = np.cumsum(diff, axis=1)[:, :nb] > 0
    return _csr_from_dense(active)


def radial_block_lists(F: int, S: int, B: int, method: str = "auto"):
    """Radial block lists; brute force on tiny grids, per-token intervals otherwise."""
    if method == "bruteforce" or (method == "auto" and F * S <= 4096):
        return radial_block_lists_bruteforce(F, S, B)
    return radial_block_lists_intervals(F, S, B)


# ------------------------------------------------- joint text + video tokens --
#
# Reading (the pages are silent on text tokens): a video DiT that runs joint
# attention over its video tokens and T text tokens appends the text tokens
# after the F*S video tokens. The radial rule applies between video tokens
# only; a text query attends to every token and every query attends to every
# text key (text is global context, never thinned). Blocks are cut over the
# whole joint sequence from token 0, so the block holding the last video
# tokens may also hold the first text tokens.


def joint_token_mask(F: int, S: int, T: int, B: int) -> np.ndarray:
    """Dense ``[n, n]`` mask, ``n = F*S + T``: the radial token rule among the
    video tokens, every pair with a text token (row or column) admitted.
    Brute force; tiny grids only."""
    nv = F * S
    mask = np.ones((nv + T, nv + T), dtype=bool)
    mask[:nv, :nv] = radial_token_mask(F, S, B)
    return mask


def joint_block_lists_bruteforce(F: int, S: int, T: int, B: int):
    """Joint block lists from the brute-force token mask (tiny grids only)."""
    return block_lists_from_token_mask(joint_token_mask(F, S, T, B), B)


def joint_block_lists(F: int, S: int, T: int, B: int, method: str = "auto"):
    """Joint block lists for any size.

    Composed from the radial block lists of the video tokens alone: a query
    block holding only video tokens keeps its radial key blocks and gains
    every key block that holds a text token (blocks ``>= (F*S) // B``); a
    query block holding any text token lists every key block.
    """
    nv = F * S
    n = nv + T
    if method == "bruteforce" or (method == "auto" and n <= 4096):
        return joint_block_lists_bruteforce(F, S, T, B)
    # method "compose" (or "auto" above 4096 tokens)
    nb = -(-n // B)
    rp_v, ci_v = radial_block_lists(F, S, B)
    first_text_block = nv // B if T > 0 else nb
    active = np.zeros((nb, nb), dtype=bool)
    for qb in range(nb):
        if min(n, (qb + 1) * B) > nv:  # holds a text query
            active[qb] = True
            continue
        active[qb, ci_v[rp_v[qb]:rp_v[qb + 1]]] = True
        active[qb, first_text_block:] = True
    return _csr_from_dense(active)
