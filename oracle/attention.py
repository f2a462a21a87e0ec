"""Oracle: masked softmax attention over key-block lists, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is computed ([RA-skill] Step 2, ``RadialAttention.forward``): scores
``Q K^T * scale`` with ``scale = head_dim ** -0.5``, masked positions set to
``-inf`` before the softmax (``apply_radial_attention_mask``), softmax over the
keys, then the weighted sum of ``V``. Layout ``[batch, heads, n, head_dim]``.

Block granularity ([RA-blog], 128x128 blocks): a query attends to every key
``j < n`` inside every active key block of its query block. ``lse`` is the
natural-log log-sum-exp of the row's admitted scaled scores. A row with no
admitted key returns zeros and ``lse = -inf`` (the pages are silent; this is
the reading taken).

Inputs are whatever the GPU receives (bf16 values), promoted to float64.
"""

from __future__ import annotations

import numpy as np


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor (any dtype); promote through fp32 exactly
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def expand_row_mask(row_ptr, col_idx, list_base: int, rows, n: int, block: int) -> np.ndarray:
    """Admitted key columns of the given query rows, as a ``[len(rows), n]`` bool array.

    ``list_base`` is the CSR row of query block 0 for this head's list.
    """
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, n), dtype=bool)
    for t, i in enumerate(rows):
        r = list_base + int(i) // block
        for kb in col_idx[row_ptr[r]:row_ptr[r + 1]]:
            out[t, int(kb) * block:min(n, (int(kb) + 1) * block)] = True
    return out


def masked_attention_rows(q_rows, k, v, admitted: np.ndarray, scale: float):
    """Masked softmax attention for a few query rows of one (batch, head).

    ``q_rows [R, D]``, ``k, v [n, D]``, ``admitted [R, n]`` bool. Returns
    ``out [R, D]`` and ``lse [R]`` in float64.
    """
    q_rows, k, v = _as_f64(q_rows), _as_f64(k), _as_f64(v)
    s = (q_rows @ k.T) * scale
    s = np.where(admitted, s, -np.inf)
    m = s.max(axis=1)
    m0 = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(s - m0[:, None])            # exp(-inf) = 0 on masked keys
    l = p.sum(axis=1)
    has = l > 0
    out = np.zeros((q_rows.shape[0], v.shape[1]), dtype=np.float64)
    out[has] = (p[has] @ v) / l[has, None]
    lse = np.full(q_rows.shape[0], -np.inf)
    lse[has] = m0[has] + np.log(l[has])
    return out, lse


def masked_attention_fp64(q, k, v, row_ptr, col_idx, num_lists: int, block: int,
                          scale: float | None = None, rows=None, heads=None,
                          batches=None, chunk: int = 256):
    """Masked attention over block lists for a ``[batch, heads, n, D]`` problem.

    ``num_lists`` is 1 (one list shared by all heads) or ``heads`` (head ``h``
    uses list ``h``; its CSR rows start at ``h * nqb``). ``rows`` restricts the
    computation to some query rows (the same rows for every selected head);
    ``heads`` / ``batches`` restrict the heads / batch items. Returns
    ``(out, lse)`` with shapes ``[len(batches), len(heads), len(rows), D]`` and
    ``[len(batches), len(heads), len(rows)]``.
    """
    Bt, H, n, D = q.shape
    if scale is None or scale <= 0:
        scale = D ** -0.5
    nqb = -(-n // block)
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = range(H) if heads is None else list(heads)
    batches = range(Bt) if batches is None else list(batches)
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    out = np.zeros((len(batches), len(heads), rows.size, D))
    lse = np.zeros((len(batches), len(heads), rows.size))
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            qq, kk, vv = _as_f64(q[b, h]), _as_f64(k[b, h]), _as_f64(v[b, h])
            base = (h if num_lists > 1 else 0) * nqb
            for c0 in range(0, rows.size, chunk):
                rr = rows[c0:c0 + chunk]
                adm = expand_row_mask(row_ptr, col_idx, base, rr, n, block)
                o, l_ = masked_attention_rows(qq[rr], kk, vv, adm, scale)
                out[bi, hi, c0:c0 + rr.size] = o
                lse[bi, hi, c0:c0 + rr.size] = l_
    return out, lse


def bf16_round(x) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even), returned as float64.

    Used by tests that build their own inputs without torch.
    """
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)
