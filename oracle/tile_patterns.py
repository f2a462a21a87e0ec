"""Oracle: per-head tile patterns (diagonal, multi-diagonal, vertical stripes,
dual window) expanded into block lists.

TEST INFRASTRUCTURE ONLY (see the package docstring). Plain NumPy; written to
be checked by eye against the definitions below, not to be fast.

The pattern families (page tags are defined in ``oracle/__init__.py``):

* [vDiT-skill] "Sparse attention patterns": a *diagonal* head attends to the
  positions within a window of the diagonal, ``|i - j| <= w``; a
  *multi-diagonal* head to diagonal bands at a set of offsets from it; a
  *vertical-stripe* head to a fixed set of key columns in every row; a
  *mixed* head to the union of those.
* [CA-abstract]: a *dual-window* head attends to a local window plus an axial
  window, both tile-aligned.

Readings taken where the pages leave the step open:

* Patterns are defined on tiles (query block ``qb``, key block ``kb``), since
  the kernels the pages describe run on tiles; ``rel = kb - qb``.
* Every family is a union of three kinds of term, so one descriptor covers
  them all (a dict):

  - ``bands``: a list of ``(lo, hi)``; the term holds ``lo <= rel <= hi``
    (empty when ``lo > hi``). Diagonal window ``w``: ``(-w, w)``. A diagonal
    band at offset ``o`` and half-width ``h``: ``(o - h, o + h)`` (``h = 0``
    is the page's single diagonal). A local window of ``W`` tiles:
    ``(-(W // 2), W - W // 2 - 1)``.
  - ``axial``: ``None`` or ``(P, a)`` with ``P >= 1``, ``a >= 0``; the term
    holds when ``rel`` is congruent modulo ``P`` to some ``t`` with
    ``|t| <= a``. This is the axial window read on a video's tile sequence:
    tiles a whole number of frame periods away, give or take ``a``.
  - ``columns``: key blocks listed in every row (vertical stripes).

* Key blocks outside ``[0, nkb)`` do not exist; a row may end up empty.
"""

from __future__ import annotations

import numpy as np


def tile_pattern_mask(pattern: dict, nqb: int, nkb: int | None = None) -> np.ndarray:
    """Boolean ``[nqb, nkb]`` tile mask of one head: the union of its terms.

    [vDiT-skill] "Sparse attention patterns" (diagonal, multi-diagonal,
    vertical stripe, mixed = union); [CA-abstract] (local + axial window).
    """
    nkb = nqb if nkb is None else nkb
    qb = np.arange(nqb, dtype=np.int64)[:, None]
    kb = np.arange(nkb, dtype=np.int64)[None, :]
    rel = kb - qb
    mask = np.zeros((nqb, nkb), dtype=bool)
    for lo, hi in pattern.get("bands", ()):
        mask |= (rel >= lo) & (rel <= hi)
    axial = pattern.get("axial")
    if axial is not None:
        period, a = axial
        residue = np.mod(rel, period)            # in [0, period)
        mask |= (residue <= a) | (residue >= period - a)
    cols = np.asarray(pattern.get("columns", ()), dtype=np.int64)
    if cols.size:
        mask |= np.isin(kb, cols)
    return mask


def tile_pattern_lists(patterns: list[dict], nqb: int):
    """CSR block lists of one pattern per head (``num_lists = len(patterns)``).

    Head ``h``'s rows start at ``h * nqb``; each row holds its key blocks in
    ascending order. Returns ``(row_ptr int32[len * nqb + 1], col_idx int32[nnz])``.
    """
    masks = [tile_pattern_mask(p, nqb) for p in patterns]
    allm = np.concatenate(masks, axis=0) if masks else np.zeros((0, nqb), dtype=bool)
    row_ptr = np.zeros(allm.shape[0] + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(allm.sum(axis=1))
    _, cols = np.nonzero(allm)
    return row_ptr.astype(np.int32), cols.astype(np.int32)
