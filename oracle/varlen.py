"""Variable-length batches for the oracle (TEST INFRASTRUCTURE ONLY).

The pages treat one video at a time ([RA-skill] Step 2 takes x of shape
[batch, seq_len, dim] with one mask for the whole batch); they say nothing
about batching sequences of different lengths. The reading taken here is the
plainest one: each item of a variable-length batch is its own problem, with
its own radial (or joint text + video) lists and its own attention, and
nothing crosses from one item to another. So the oracle is the single-item
oracle applied item by item, and the batch's lists are the items' lists
concatenated (item b's query-block rows after those of items 0..b-1, its
column indices counted inside the item).
"""

from __future__ import annotations

import numpy as np

from .attention import masked_attention_fp64
from .attention_backward import masked_attention_backward_fp64
from .radial_mask import joint_block_lists


def varlen_block_lists(items, block: int):
    """Concatenated joint lists of ``items`` = [(frames, tokens_per_frame,
    text_tokens), ...]: ``(row_ptr, col_idx)`` with sum of the items' query-block
    counts rows."""
    rps, cis = [], []
    offset = 0
    for F, S, T in items:
        rp, ci = joint_block_lists(F, S, T, block)
        rps.append(np.asarray(rp[:-1], dtype=np.int64) + offset)
        cis.append(np.asarray(ci, dtype=np.int64))
        offset += int(rp[-1])
    row_ptr = np.concatenate(rps + [np.array([offset])])
    return row_ptr, np.concatenate(cis) if cis else np.zeros(0, dtype=np.int64)


def split_item_lists(row_ptr, col_idx, nqbs, num_lists: int = 1):
    """The items' own CSR lists back out of a concatenation: item b's block of
    ``num_lists * nqbs[b]`` rows, rebased to start at entry 0."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    out, r0 = [], 0
    for nqb in nqbs:
        rows = num_lists * nqb
        rp = row_ptr[r0:r0 + rows + 1]
        out.append((rp - rp[0], col_idx[rp[0]:rp[-1]]))
        r0 += rows
    return out


def varlen_masked_attention_fp64(q, k, v, cu_seqlens, item_lists, num_lists: int, block: int,
                                 scale: float | None = None):
    """Attention of a packed batch ``q, k, v: [total, heads, D]``: item b =
    tokens ``cu_seqlens[b]..cu_seqlens[b+1]``, attended with its own lists
    ``item_lists[b] = (row_ptr, col_idx)``. Returns ``(out [total, heads, D],
    lse [heads, total])``."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    total, H, D = q.shape
    out = np.zeros((total, H, D))
    lse = np.full((H, total), -np.inf)
    for b, (rp, ci) in enumerate(item_lists):
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        if t1 == t0:
            continue
        sl = slice(t0, t1)
        as_bhnd = lambda x: np.transpose(x[sl], (1, 0, 2))[None]  # noqa: E731
        o, l_ = masked_attention_fp64(as_bhnd(q), as_bhnd(k), as_bhnd(v), rp, ci, num_lists,
                                      block, scale=scale)
        out[sl] = np.transpose(o[0], (1, 0, 2))
        lse[:, sl] = l_[0]
    return out, lse


def varlen_masked_attention_backward_fp64(q, k, v, do, cu_seqlens, item_lists, num_lists: int,
                                          block: int, scale: float | None = None):
    """Gradients of ``varlen_masked_attention_fp64``: item by item, the
    single-problem gradients (dQ, dK, dV) on the item's tokens; packed
    ``[total, heads, D]`` float64 arrays, zero on no token."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    total, H, D = q.shape
    grads = [np.zeros((total, H, D)) for _ in range(3)]
    for b, (rp, ci) in enumerate(item_lists):
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        if t1 == t0:
            continue
        sl = slice(t0, t1)
        as_bhnd = lambda x: np.transpose(x[sl], (1, 0, 2))[None]  # noqa: E731
        gs = masked_attention_backward_fp64(as_bhnd(q), as_bhnd(k), as_bhnd(v), as_bhnd(do), rp,
                                            ci, num_lists, block, scale=scale)
        for g, gi in zip(grads, gs):
            g[sl] = np.transpose(gi[0], (1, 0, 2))
    return tuple(grads)
