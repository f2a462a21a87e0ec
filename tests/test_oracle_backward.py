"""Pins of the backward oracle (oracle/attention_backward.py) to things other
than its own formulas: central finite differences of the forward oracle,
float64 autograd through an independent dense masked attention, PyTorch's
scaled_dot_product_attention backward for all-ones lists, and structural
cases (rows with no key, keys no row admits)."""

import numpy as np
import pytest
import torch

import oracle
from workloads import random_block_lists


def _problem(B, H, n, D, seed):
    g = np.random.default_rng(seed)
    mk = lambda: oracle.bf16_round(g.standard_normal((B, H, n, D)))  # noqa: E731
    return mk(), mk(), mk(), mk()


def _lists(n, block, L, seed, empty_rows=()):
    nqb = -(-n // block)
    rp, ci = random_block_lists(L * nqb, nqb, 0.45, seed, empty_rows=empty_rows,
                                force={0: [nqb - 1]})
    return rp, ci


def test_finite_differences_of_the_forward_oracle():
    """d(sum(O * G))/dX by central differences of masked_attention_fp64
    matches the backward oracle for X in Q, K, V (every entry)."""
    B, H, n, D, blk = 1, 2, 20, 4, 8
    q, k, v, g = _problem(B, H, n, D, 5)
    rp, ci = _lists(n, blk, 2, 6, empty_rows=[1])  # head 0 row block 1 empty
    dq, dk, dv = oracle.masked_attention_backward_fp64(q, k, v, g, rp, ci, 2, blk)

    def loss(q_, k_, v_):
        o, _ = oracle.masked_attention_fp64(q_, k_, v_, rp, ci, 2, blk)
        return float((o * g).sum())

    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-5, atol=1e-7, err_msg=f"d{name}")


def _autograd_dense(q, k, v, g, adm, scale):
    """Independent dense masked attention in torch float64 with autograd."""
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = (qt @ kt.transpose(-1, -2)) * scale
    s = s.masked_fill(~torch.tensor(adm), float("-inf"))
    has = torch.tensor(adm).any(-1, keepdim=True)
    p = torch.where(has, torch.softmax(torch.where(has, s, torch.zeros_like(s)), -1),
                    torch.zeros_like(s))
    o = p @ vt
    (o * torch.tensor(g)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("n,D,blk,L,seed", [(70, 16, 16, 1, 11), (129, 8, 32, 3, 12)])
def test_matches_float64_autograd(n, D, blk, L, seed):
    B, H = 2, 3
    q, k, v, g = _problem(B, H, n, D, seed)
    rp, ci = _lists(n, blk, L, seed + 1, empty_rows=[2])
    dq, dk, dv = oracle.masked_attention_backward_fp64(q, k, v, g, rp, ci, L, blk)
    nqb = -(-n // blk)
    for h in range(H):
        base = (h if L > 1 else 0) * nqb
        adm = oracle.expand_row_mask(rp, ci, base, np.arange(n), n, blk)
        for b in range(B):
            aq, ak, av = _autograd_dense(q[b, h], k[b, h], v[b, h], g[b, h], adm, D ** -0.5)
            np.testing.assert_allclose(dq[b, h], aq, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(dk[b, h], ak, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(dv[b, h], av, rtol=1e-10, atol=1e-12)


def test_all_ones_lists_match_sdpa_backward():
    B, H, n, D, blk = 1, 2, 96, 32, 32
    q, k, v, g = _problem(B, H, n, D, 21)
    nqb = n // blk
    rp = np.arange(0, nqb * nqb + 1, nqb)
    ci = np.tile(np.arange(nqb), nqb)
    dq, dk, dv = oracle.masked_attention_backward_fp64(q, k, v, g, rp, ci, 1, blk)
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    (o * torch.tensor(g)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_structural_zeros():
    """Rows with no admitted key give dQ = 0; keys no row admits give dK = dV = 0;
    with a single admitted key per row, dV of that key is the sum of dO over
    its rows and dQ, dK vanish (the softmax is constant 1)."""
    B, H, n, D, blk = 1, 1, 48, 8, 8
    q, k, v, g = _problem(B, H, n, D, 31)
    nqb = n // blk
    # query block 0 empty, others attend only key block 2
    rp = np.array([0, 0] + list(range(1, nqb)), dtype=np.int64)
    ci = np.full(nqb - 1, 2, dtype=np.int64)
    dq, dk, dv = oracle.masked_attention_backward_fp64(q, k, v, g, rp, ci, 1, blk)
    assert np.all(dq[0, 0, :blk] == 0)
    other = np.r_[0:2 * blk, 3 * blk:n]
    assert np.all(dk[0, 0, other] == 0) and np.all(dv[0, 0, other] == 0)
    # one key per row: block size 1
    rp1 = np.arange(n + 1)
    ci1 = np.full(n, 7)
    dq1, dk1, dv1 = oracle.masked_attention_backward_fp64(q, k, v, g, rp1, ci1, 1, 1)
    np.testing.assert_allclose(dv1[0, 0, 7], g[0, 0].sum(axis=0), rtol=1e-12)
    np.testing.assert_allclose(dq1, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk1, 0.0, atol=1e-12)


def test_sampled_functions_agree_with_whole_heads():
    B, H, n, D, blk, L = 2, 2, 100, 8, 16, 2
    q, k, v, g = _problem(B, H, n, D, 41)
    rp, ci = _lists(n, blk, L, 42, empty_rows=[3])
    dq, dk, dv = oracle.masked_attention_backward_fp64(q, k, v, g, rp, ci, L, blk)
    rows = np.array([0, 5, 17, 50, 99])
    keys = np.array([1, 16, 33, 64, 98])
    for b in range(B):
        for h in range(H):
            sq = oracle.masked_attention_dq_rows(q, k, v, g, rp, ci, L, blk, b, h, rows)
            np.testing.assert_allclose(sq, dq[b, h, rows], rtol=1e-10, atol=1e-12)
            sk, sv = oracle.masked_attention_dkdv_keys(q, k, v, g, rp, ci, L, blk, b, h, keys,
                                                       chunk=37)
            np.testing.assert_allclose(sk, dk[b, h, keys], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(sv, dv[b, h, keys], rtol=1e-10, atol=1e-12)


def test_planted_mistake_is_caught():
    """A plausible slip (delta taken as the row sum of dP instead of of
    P * dP) is caught by the finite-difference pin's tolerance."""
    B, H, n, D, blk = 1, 1, 16, 4, 8
    q, k, v, g = _problem(B, H, n, D, 51)
    rp, ci = _lists(n, blk, 1, 52)
    adm = oracle.expand_row_mask(rp, ci, 0, np.arange(n), n, blk)
    scale = D ** -0.5
    qq, kk, vv, gg = q[0, 0], k[0, 0], v[0, 0], g[0, 0]
    s = np.where(adm, (qq @ kk.T) * scale, -np.inf)
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    dp = gg @ vv.T
    wrong_dq = (p * (dp - dp.sum(1, keepdims=True))) @ kk * scale
    dq, _, _ = oracle.masked_attention_backward_fp64(q, k, v, g, rp, ci, 1, blk)
    assert np.abs(wrong_dq - dq[0, 0]).max() > 1e-3
