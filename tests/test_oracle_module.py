"""Pins of the module oracle (oracle/module.py) to things other than its own
formulas: PyTorch's multi-head attention forward (float64, with the block mask
as its attention mask), the identity-projection special case that reduces the
module to the (separately pinned) attention oracle, the all-empty lists case
(output = out_proj's bias), and agreement of the per-row form with the
whole-problem form. A plausible slip in the head split is shown to be caught."""

import numpy as np
import pytest
import torch

import oracle
from workloads import make_module_inputs, random_block_lists


def _f64(t):
    return None if t is None else t.float().double()


def _torch_mha(x, w_qkv, b_qkv, w_out, b_out, heads, allowed):
    """torch.nn.functional.multi_head_attention_forward in float64; ``allowed``
    is the admitted mask, ``[n, n]`` or ``[batch*heads, n, n]``."""
    xt = _f64(x).transpose(0, 1)  # [n, batch, C]
    C = xt.shape[-1]
    y, _ = torch.nn.functional.multi_head_attention_forward(
        xt, xt, xt, C, heads, _f64(w_qkv), _f64(b_qkv), None, None, False, 0.0,
        _f64(w_out), _f64(b_out) if b_out is not None else None, training=False,
        need_weights=False, attn_mask=torch.from_numpy(~allowed))
    return y.transpose(0, 1).numpy()


@pytest.mark.parametrize("B,n,H,D,blk,L,bias,seed", [
    (2, 70, 2, 8, 16, 1, True, 1),
    (1, 100, 3, 4, 32, 3, True, 2),     # per-head lists
    (1, 64, 1, 16, 8, 1, False, 3),     # no biases
])
def test_matches_torch_multi_head_attention(B, n, H, D, blk, L, bias, seed):
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, seed, bias=bias)
    nqb = -(-n // blk)
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, seed + 10)
    empty = np.nonzero(np.diff(rp) == 0)[0]  # torch's softmax of an all-masked row is NaN
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, seed + 10,
                                force={int(r): [int(r) % nqb] for r in empty})
    assert np.all(np.diff(rp) > 0) and np.diff(rp).max() > 1
    y = oracle.radial_attention_module_fp64(x, wqkv, bqkv, wo, bo, H, rp, ci, L, blk)
    rows = np.arange(n)
    if L == 1:
        allowed = oracle.expand_row_mask(rp, ci, 0, rows, n, blk)
    else:
        per_head = [oracle.expand_row_mask(rp, ci, h * nqb, rows, n, blk) for h in range(H)]
        allowed = np.stack([per_head[h] for _ in range(B) for h in range(H)])
    ref = _torch_mha(x, wqkv, bqkv, wo, bo, H, allowed)
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-11)


def test_identity_projections_reduce_to_attention():
    """q_proj = k_proj = v_proj = out_proj = I, no biases: the module is the
    attention of x split into heads, merged back."""
    B, n, H, D, blk = 2, 48, 2, 8, 16
    C = H * D
    x, _, _, _, _ = make_module_inputs(B, n, H, D, 7, bias=False)
    eye = np.eye(C)
    nqb = n // blk
    rp, ci = random_block_lists(nqb, nqb, 0.6, 8, force={0: [2]})
    y = oracle.radial_attention_module_fp64(x, np.vstack([eye] * 3), None, eye, None, H, rp, ci, 1,
                                            blk)
    xs = x.float().double().numpy().reshape(B, n, H, D).transpose(0, 2, 1, 3)
    o, _ = oracle.masked_attention_fp64(xs, xs, xs, rp, ci, 1, blk)
    np.testing.assert_allclose(y, o.transpose(0, 2, 1, 3).reshape(B, n, C), rtol=0, atol=0)


def test_empty_lists_give_the_output_bias():
    B, n, H, D, blk = 1, 40, 2, 4, 8
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, 9)
    nqb = n // blk
    rp = np.zeros(nqb + 1, dtype=np.int64)
    y = oracle.radial_attention_module_fp64(x, wqkv, bqkv, wo, bo, H, rp, np.zeros(0), 1, blk)
    np.testing.assert_array_equal(y, np.broadcast_to(bo.float().double().numpy(), y.shape))


def test_rows_form_agrees_with_whole_problem():
    B, n, H, D, blk, L = 2, 90, 3, 8, 16, 3
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, 11)
    nqb = -(-n // blk)
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, 12, empty_rows=[4])
    y = oracle.radial_attention_module_fp64(x, wqkv, bqkv, wo, bo, H, rp, ci, L, blk)
    rows = np.array([0, 17, 33, 64, 89])
    for b in range(B):
        yr = oracle.radial_attention_module_rows(x, wqkv, bqkv, wo, bo, H, rp, ci, L, blk, b, rows)
        np.testing.assert_allclose(yr, y[b, rows], rtol=1e-10, atol=1e-12)
    # heads_used: exact when w_out's columns of the other heads are zero
    wo2 = wo.clone()
    wo2[:, D:2 * D] = 0
    y2 = oracle.radial_attention_module_fp64(x, wqkv, bqkv, wo2, bo, H, rp, ci, L, blk)
    yr2 = oracle.radial_attention_module_rows(x, wqkv, bqkv, wo2, bo, H, rp, ci, L, blk, 1, rows,
                                              heads_used=[0, 2])
    np.testing.assert_allclose(yr2, y2[1, rows], rtol=1e-10, atol=1e-12)


def test_planted_head_split_slip_is_caught():
    """Splitting heads as view(batch, n, head_dim, heads) instead of
    view(batch, n, heads, head_dim) changes the output well beyond the pin's
    tolerance."""
    B, n, H, D, blk = 1, 32, 2, 4, 8
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, 13)
    C = H * D
    nqb = n // blk
    rp, ci = random_block_lists(nqb, nqb, 0.5, 14, force={0: [0]})
    good = oracle.radial_attention_module_fp64(x, wqkv, bqkv, wo, bo, H, rp, ci, 1, blk)
    xf, w, b = (t.float().double().numpy() for t in (x, wqkv, bqkv))
    proj = [xf @ w[i * C:(i + 1) * C].T + b[i * C:(i + 1) * C] for i in range(3)]
    wrong = [p.reshape(B, n, D, H).transpose(0, 3, 1, 2) for p in proj]
    o, _ = oracle.masked_attention_fp64(*wrong, rp, ci, 1, blk)
    y_wrong = o.transpose(0, 2, 1, 3).reshape(B, n, C) @ wo.float().double().numpy().T \
        + bo.float().double().numpy()
    assert np.abs(y_wrong - good).max() > 1e-2



def _torch_mha_grads(x, w_qkv, b_qkv, w_out, b_out, dy, heads, allowed):
    """float64 autograd through torch's multi_head_attention_forward."""
    leaves = [_f64(t).clone().requires_grad_() for t in (x, w_qkv, b_qkv, w_out, b_out)]
    xl, wq, bq, wo, bo = leaves
    xt = xl.transpose(0, 1)
    C = xt.shape[-1]
    y, _ = torch.nn.functional.multi_head_attention_forward(
        xt, xt, xt, C, heads, wq, bq, None, None, False, 0.0, wo, bo, training=False,
        need_weights=False, attn_mask=torch.from_numpy(~allowed))
    (y.transpose(0, 1) * _f64(dy)).sum().backward()
    return [t.grad.numpy() for t in leaves]


@pytest.mark.parametrize("B,n,H,D,blk,L,seed", [(2, 70, 2, 8, 16, 1, 61), (1, 100, 3, 4, 32, 3, 62)])
def test_backward_matches_torch_autograd(B, n, H, D, blk, L, seed):
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, seed)
    dy, _, _, _, _ = make_module_inputs(B, n, H, D, seed + 1, bias=False)
    nqb = -(-n // blk)
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, seed + 10)
    empty = np.nonzero(np.diff(rp) == 0)[0]
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, seed + 10,
                                force={int(r): [int(r) % nqb] for r in empty})
    got = oracle.radial_attention_module_backward_fp64(x, wqkv, bqkv, wo, bo, dy, H, rp, ci, L,
                                                       blk)
    rows = np.arange(n)
    if L == 1:
        allowed = oracle.expand_row_mask(rp, ci, 0, rows, n, blk)
    else:
        per_head = [oracle.expand_row_mask(rp, ci, h * nqb, rows, n, blk) for h in range(H)]
        allowed = np.stack([per_head[h] for _ in range(B) for h in range(H)])
    ref = _torch_mha_grads(x, wqkv, bqkv, wo, bo, dy, H, allowed)
    for name, g, r in zip(("dx", "dw_qkv", "db_qkv", "dw_out", "db_out"), got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-9, atol=1e-10, err_msg=name)


def test_backward_finite_differences():
    """Central differences of the forward oracle on sampled entries of every
    gradient (rows with empty lists included)."""
    B, n, H, D, blk = 1, 24, 2, 4, 8
    x, wqkv, bqkv, wo, bo = (t.float().double().numpy()
                             for t in make_module_inputs(B, n, H, D, 71))
    dy = np.random.default_rng(72).standard_normal((B, n, H * D))
    nqb = n // blk
    rp, ci = random_block_lists(nqb, nqb, 0.5, 73, empty_rows=[1], force={0: [2]})
    grads = oracle.radial_attention_module_backward_fp64(x, wqkv, bqkv, wo, bo, dy, H, rp, ci, 1,
                                                         blk)
    params = [x, wqkv, bqkv, wo, bo]

    def loss(ps):
        return float((oracle.radial_attention_module_fp64(*ps, H, rp, ci, 1, blk) * dy).sum())

    rng = np.random.default_rng(74)
    eps = 1e-6
    for i, (p_, g) in enumerate(zip(params, grads)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in p_.shape)
            hi = [q.copy() for q in params]
            lo = [q.copy() for q in params]
            hi[i][idx] += eps
            lo[i][idx] -= eps
            fd = (loss(hi) - loss(lo)) / (2 * eps)
            np.testing.assert_allclose(g[idx], fd, rtol=1e-5, atol=1e-7)


def test_backward_planted_slip_is_caught():
    """Taking dw_out as A^T dy (transposed) is caught by the autograd pin's tolerance."""
    B, n, H, D, blk = 1, 32, 2, 4, 8
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, 81)
    dy, _, _, _, _ = make_module_inputs(B, n, H, D, 82, bias=False)
    nqb = n // blk
    rp, ci = random_block_lists(nqb, nqb, 0.6, 83, force={0: [0]})
    _, _, _, dwo, _ = oracle.radial_attention_module_backward_fp64(x, wqkv, bqkv, wo, bo, dy, H, rp,
                                                                   ci, 1, blk)
    assert np.abs(dwo - dwo.T).max() > 1e-3
