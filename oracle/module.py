"""Oracle: the radial attention module, forward and backward, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is computed ([RA-skill] Step 2, the ``RadialAttention`` module), in the
page's order:

1. ``Q = q_proj(x)``, ``K = k_proj(x)``, ``V = v_proj(x)``: ``nn.Linear``
   layers, ``y = x W^T + b`` with ``W`` in ``[out_features, in_features]``.
2. Each is viewed as ``[batch, n, heads, head_dim]`` and transposed to
   ``[batch, heads, n, head_dim]``: head ``h`` is columns
   ``[h*head_dim, (h+1)*head_dim)`` of the projection.
3. Masked softmax attention (``attention.masked_attention_fp64``; the page
   applies the radial mask to dense scores, which over block lists is the
   block-granular restriction of that module).
4. The result is transposed back to ``[batch, n, heads, head_dim]``, viewed as
   ``[batch, n, heads*head_dim]`` and passed through ``out_proj``.

The three input projections are given stacked, as the library takes them:
``w_qkv = [q_proj.weight; k_proj.weight; v_proj.weight]`` (``[3C, C]``) and
``b_qkv`` likewise (``[3C]``, or ``None`` for no bias).

Functions:

* ``radial_attention_module_fp64``: ``y [batch, n, C]`` of whole problems
  (small n).
* ``radial_attention_module_backward_fp64``: the gradients of the output
  with respect to x and to the four layers' weights and biases, given dy
  (small n): the chain rule through the same steps in reverse order.
* ``radial_attention_module_rows``: ``y`` of selected tokens of one batch
  item (any n). It writes ``out_proj`` as the sum over heads of
  ``O_h W_out[:, cols_h]^T`` (the same product, split by the columns of the
  head merge), so it can be restricted to a subset of heads: with
  ``heads_used`` given, it is the module's output exactly when ``w_out``'s
  columns of the other heads are zero, which the caller arranges.
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64, expand_row_mask, masked_attention_fp64, masked_attention_rows
from .attention_backward import masked_attention_backward_fp64


def _linear(x, w, b):
    """``nn.Linear``: ``x W^T + b`` (``b`` may be None)."""
    y = x @ w.T
    return y if b is None else y + b


def _split_qkv(w_qkv, b_qkv, C: int):
    w = _as_f64(w_qkv)
    b = None if b_qkv is None else _as_f64(b_qkv)
    ws = (w[:C], w[C:2 * C], w[2 * C:3 * C])
    bs = (None, None, None) if b is None else (b[:C], b[C:2 * C], b[2 * C:3 * C])
    return ws, bs


def radial_attention_module_fp64(x, w_qkv, b_qkv, w_out, b_out, heads: int, row_ptr, col_idx,
                                 num_lists: int, block: int, scale: float | None = None):
    """The module's output ``y [batch, n, C]`` for ``x [batch, n, C]``,
    ``C = heads * head_dim``; lists as in ``masked_attention_fp64``."""
    x = _as_f64(x)
    Bt, n, C = x.shape
    D = C // heads
    (wq, wk, wv), (bq, bk, bv) = _split_qkv(w_qkv, b_qkv, C)

    def heads_first(t):  # [Bt, n, C] -> view [Bt, n, H, D] -> [Bt, H, n, D]
        return t.reshape(Bt, n, heads, D).transpose(0, 2, 1, 3)

    q = heads_first(_linear(x, wq, bq))
    k = heads_first(_linear(x, wk, bk))
    v = heads_first(_linear(x, wv, bv))
    o, _ = masked_attention_fp64(q, k, v, row_ptr, col_idx, num_lists, block, scale)
    merged = o.transpose(0, 2, 1, 3).reshape(Bt, n, C)
    return _linear(merged, _as_f64(w_out), None if b_out is None else _as_f64(b_out))


def radial_attention_module_rows(x, w_qkv, b_qkv, w_out, b_out, heads: int, row_ptr, col_idx,
                                 num_lists: int, block: int, b: int, rows, heads_used=None,
                                 scale: float | None = None):
    """``y[b, rows, :]`` (``[len(rows), C]``). Keys and values are projected
    for all ``n`` tokens but only for the heads in ``heads_used`` (default:
    every head)."""
    Bt, n, C = x.shape
    D = C // heads
    if scale is None or scale <= 0:
        scale = D ** -0.5
    nqb = -(-n // block)
    rows = np.asarray(rows, dtype=np.int64)
    heads_used = range(heads) if heads_used is None else list(heads_used)
    xb = _as_f64(x[b])
    wq_all, wo = w_qkv, _as_f64(w_out)
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    y = np.zeros((rows.size, C)) if b_out is None else np.tile(_as_f64(b_out), (rows.size, 1))
    bias = None if b_qkv is None else _as_f64(b_qkv)
    for h in heads_used:
        cq = slice(h * D, (h + 1) * D)
        ck = slice(C + h * D, C + (h + 1) * D)
        cv = slice(2 * C + h * D, 2 * C + (h + 1) * D)
        q_h = _linear(xb[rows], _as_f64(wq_all[cq]), None if bias is None else bias[cq])
        k_h = _linear(xb, _as_f64(wq_all[ck]), None if bias is None else bias[ck])
        v_h = _linear(xb, _as_f64(wq_all[cv]), None if bias is None else bias[cv])
        base = (h if num_lists > 1 else 0) * nqb
        adm = expand_row_mask(row_ptr, col_idx, base, rows, n, block)
        o_h, _ = masked_attention_rows(q_h, k_h, v_h, adm, scale)
        y += o_h @ wo[:, cq].T
    return y


def radial_attention_module_backward_fp64(x, w_qkv, b_qkv, w_out, b_out, dy, heads: int, row_ptr,
                                          col_idx, num_lists: int, block: int,
                                          scale: float | None = None):
    """Gradients of ``radial_attention_module_fp64``'s output, given ``dy``
    (``[batch, n, C]``). Returns ``(dx, dw_qkv, db_qkv, dw_out, db_out)`` with
    the shapes of ``x``, ``w_qkv``, ``[3C]``, ``w_out``, ``[C]`` (the bias
    gradients also when the biases are None: the layer's bias gradient).

    Reverse order of the forward's steps:

    * ``out_proj`` (``y = A W_out^T + b_out``): ``dA = dy W_out``,
      ``dW_out = sum over tokens of dy^T A``, ``db_out = sum of dy``;
    * head merge and split are reshapes: their gradients reshape back;
    * the attention: ``masked_attention_backward_fp64``;
    * each projection (``P = x W^T + b``): ``dW = dP^T x``, ``db = sum of dP``,
      and ``dx`` sums ``dP W`` over the three projections.
    """
    x = _as_f64(x)
    Bt, n, C = x.shape
    D = C // heads
    (wq, wk, wv), (bq, bk, bv) = _split_qkv(w_qkv, b_qkv, C)
    wo = _as_f64(w_out)
    dy = _as_f64(dy)

    def heads_first(t):
        return t.reshape(Bt, n, heads, D).transpose(0, 2, 1, 3)

    def heads_merged(t):
        return t.transpose(0, 2, 1, 3).reshape(Bt, n, C)

    q = heads_first(_linear(x, wq, bq))
    k = heads_first(_linear(x, wk, bk))
    v = heads_first(_linear(x, wv, bv))
    o, _ = masked_attention_fp64(q, k, v, row_ptr, col_idx, num_lists, block, scale)
    a = heads_merged(o)
    # out_proj
    da = dy @ wo
    dw_out = dy.reshape(-1, C).T @ a.reshape(-1, C)  # sum over (batch, token) of dy^T A
    db_out = dy.sum(axis=(0, 1))
    # attention
    dq, dk, dv = masked_attention_backward_fp64(q, k, v, heads_first(da), row_ptr, col_idx,
                                                num_lists, block, scale)
    dqm, dkm, dvm = heads_merged(dq), heads_merged(dk), heads_merged(dv)
    # projections
    xr = x.reshape(-1, C)
    dw_qkv = np.concatenate([g.reshape(-1, C).T @ xr for g in (dqm, dkm, dvm)], axis=0)
    db_qkv = np.concatenate([g.sum(axis=(0, 1)) for g in (dqm, dkm, dvm)])
    dx = dqm @ wq + dkm @ wk + dvm @ wv
    return dx, dw_qkv, db_qkv, dw_out, db_out
