"""Oracle: gradients of masked softmax attention over key-block lists, float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is computed: the backward pass that ``loss.backward()`` runs through the
radial attention module when it is fine-tuned with LoRA for longer sequences
([RA-skill] Step 4; the training-cost claim of [RA-summary] and [RA-blog]).
The pages print no backward formulas, so the oracle is the plain derivative
of the forward definition in ``attention.py``. For one (batch, head), with
``A`` the admitted (query, key) pairs of the block lists:

    S = Q K^T * scale,  S[~A] = -inf,  P = softmax_rows(S),  O = P V
    given dO:  dV = P^T dO
               dP = dO V^T
               delta_i = sum_d dO[i, d] O[i, d]      (= sum_j P_ij dP_ij)
               dS = P * (dP - delta[:, None])
               dQ = dS K * scale,   dK = dS^T Q * scale

A row with no admitted key has ``O = 0`` whatever Q, K, V are, so it gives no
gradient (dQ row 0, no contribution to dK or dV). Inputs are the values the
GPU receives (bf16), promoted to float64.

Functions:

* ``masked_attention_backward_fp64``: dQ, dK, dV of whole heads (small n).
* ``masked_attention_dq_rows``: dQ of selected query rows (any n).
* ``masked_attention_dkdv_keys``: dK, dV of selected key rows (any n): only
  the query rows whose lists hold those keys' blocks are visited.
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64, expand_row_mask, masked_attention_rows


def _softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax with fully masked rows (all -inf) mapped to zeros."""
    m = s.max(axis=1)
    m0 = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(s - m0[:, None])
    l = p.sum(axis=1)
    out = np.zeros_like(p)
    has = l > 0
    out[has] = p[has] / l[has, None]
    return out


def _head_backward(q, k, v, do, adm, scale):
    """dQ, dK, dV of one (batch, head); ``adm [n, n]`` is the admitted mask."""
    s = np.where(adm, (q @ k.T) * scale, -np.inf)
    p = _softmax_rows(s)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    delta = (do * o).sum(axis=1)
    ds = p * (dp - delta[:, None])
    dq = (ds @ k) * scale
    dk = (ds.T @ q) * scale
    return dq, dk, dv


def _list_base(h: int, num_lists: int, nqb: int) -> int:
    return (h if num_lists > 1 else 0) * nqb


def masked_attention_backward_fp64(q, k, v, do, row_ptr, col_idx, num_lists: int, block: int,
                                   scale: float | None = None):
    """dQ, dK, dV for a ``[batch, heads, n, D]`` problem (whole heads, small n).

    Lists as in ``masked_attention_fp64``. Returns three float64 arrays of
    shape ``[batch, heads, n, D]``.
    """
    Bt, H, n, D = q.shape
    if scale is None or scale <= 0:
        scale = D ** -0.5
    nqb = -(-n // block)
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    dq = np.zeros((Bt, H, n, D))
    dk = np.zeros((Bt, H, n, D))
    dv = np.zeros((Bt, H, n, D))
    rows = np.arange(n)
    for h in range(H):
        adm = expand_row_mask(row_ptr, col_idx, _list_base(h, num_lists, nqb), rows, n, block)
        for b in range(Bt):
            g = _head_backward(_as_f64(q[b, h]), _as_f64(k[b, h]), _as_f64(v[b, h]),
                               _as_f64(do[b, h]), adm, scale)
            dq[b, h], dk[b, h], dv[b, h] = g
    return dq, dk, dv


def masked_attention_dq_rows(q, k, v, do, row_ptr, col_idx, num_lists: int, block: int,
                             b: int, h: int, rows, scale: float | None = None):
    """dQ of the given query rows of (batch ``b``, head ``h``): ``[len(rows), D]``.

    Each row needs only its own scores: delta_i comes from the row's own
    output, recomputed here.
    """
    n, D = q.shape[2], q.shape[3]
    if scale is None or scale <= 0:
        scale = D ** -0.5
    nqb = -(-n // block)
    rows = np.asarray(rows, dtype=np.int64)
    qq, kk, vv, dd = (_as_f64(t[b, h]) for t in (q, k, v, do))
    adm = expand_row_mask(np.asarray(row_ptr), np.asarray(col_idx),
                          _list_base(h, num_lists, nqb), rows, n, block)
    s = np.where(adm, (qq[rows] @ kk.T) * scale, -np.inf)
    p = _softmax_rows(s)
    o = p @ vv
    dp = dd[rows] @ vv.T
    delta = (dd[rows] * o).sum(axis=1)
    ds = p * (dp - delta[:, None])
    return (ds @ kk) * scale


def masked_attention_dkdv_keys(q, k, v, do, row_ptr, col_idx, num_lists: int, block: int,
                               b: int, h: int, keys, scale: float | None = None,
                               chunk: int = 512):
    """dK and dV of the given key rows of (batch ``b``, head ``h``).

    Visits only query blocks whose lists hold one of the keys' blocks; for
    those rows the softmax normaliser is the row's full log-sum-exp (from
    ``masked_attention_rows``). Returns ``(dk, dv)``, each ``[len(keys), D]``.
    """
    n, D = q.shape[2], q.shape[3]
    if scale is None or scale <= 0:
        scale = D ** -0.5
    nqb = -(-n // block)
    base = _list_base(h, num_lists, nqb)
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    keys = np.asarray(keys, dtype=np.int64)
    kblocks = set(int(j) // block for j in keys)
    qblocks = [qb for qb in range(nqb)
               if kblocks & set(col_idx[row_ptr[base + qb]:row_ptr[base + qb + 1]].tolist())]
    qrows = np.concatenate([np.arange(qb * block, min(n, (qb + 1) * block)) for qb in qblocks]) \
        if qblocks else np.zeros(0, dtype=np.int64)
    qq, kk, vv, dd = (_as_f64(t[b, h]) for t in (q, k, v, do))
    dk = np.zeros((keys.size, D))
    dv = np.zeros((keys.size, D))
    for c0 in range(0, qrows.size, chunk):
        rr = qrows[c0:c0 + chunk]
        adm = expand_row_mask(row_ptr, col_idx, base, rr, n, block)
        o, lse = masked_attention_rows(qq[rr], kk, vv, adm, scale)
        delta = (dd[rr] * o).sum(axis=1)
        a = adm[:, keys]
        s = (qq[rr] @ kk[keys].T) * scale
        p = np.where(a, np.exp(s - np.where(np.isfinite(lse), lse, 0.0)[:, None]), 0.0)
        dp = dd[rr] @ vv[keys].T
        ds = p * (dp - delta[:, None])
        dv += p.T @ dd[rr]
        dk += (ds.T @ qq[rr]) * scale
    return dk, dv
