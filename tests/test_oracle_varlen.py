"""Pins of the variable-length oracle (oracle/varlen.py) on the CPU.

The pages batch nothing of different lengths; the reading is that each item is
its own problem. These checks tie the oracle to constructions that do not go
through it: dense softmax attention with a block-diagonal mask over the packed
sequence (torch SDPA in float64, the mask built here; its gradients by torch
autograd), the batched oracle for items of equal length, and the items' own
lists split back out.
"""

import numpy as np
import torch

import oracle


def _packed(total, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((total, H, D), generator=g, dtype=torch.float64) for _ in range(3)]


def _ones_lists(n, block):
    nqb = -(-n // block)
    rp = np.arange(nqb + 1) * nqb
    ci = np.tile(np.arange(nqb), nqb)
    return rp, ci


def test_varlen_lists_are_the_items_lists_concatenated():
    items = [(3, 96, 0), (2, 200, 37), (4, 64, 129)]
    rp, ci = oracle.varlen_block_lists(items, 64)
    nqbs = [-(-(f * s + t) // 64) for f, s, t in items]
    assert rp.size == sum(nqbs) + 1 and rp[0] == 0 and rp[-1] == ci.size
    for (f, s, t), (rpi, cii) in zip(items, oracle.split_item_lists(rp, ci, nqbs)):
        rpo, cio = oracle.joint_block_lists(f, s, t, 64)
        assert np.array_equal(rpi, rpo) and np.array_equal(cii, cio)


def test_all_ones_lists_equal_block_diagonal_dense_attention():
    cu = np.array([0, 70, 70, 200, 333])      # includes an empty item
    H, D, block = 2, 16, 32
    q, k, v = _packed(int(cu[-1]), H, D, 1)
    lists = [_ones_lists(int(cu[b + 1] - cu[b]), block) for b in range(len(cu) - 1)]
    out, lse = oracle.varlen_masked_attention_fp64(q.numpy(), k.numpy(), v.numpy(), cu, lists,
                                                   1, block)
    item = np.repeat(np.arange(len(cu) - 1), np.diff(cu))
    mask = torch.as_tensor(item[:, None] == item[None, :])
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1), attn_mask=mask)
    assert np.allclose(out, ref.transpose(0, 1).numpy(), atol=1e-12, rtol=1e-12)
    s = torch.einsum("thd,shd->hts", q, k) * D ** -0.5
    s = s.masked_fill(~mask, float("-inf"))
    assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def test_equal_items_match_the_batched_oracle():
    F, S, T, block, H, D = 3, 80, 20, 64, 2, 8
    n = F * S + T
    rp, ci = oracle.joint_block_lists(F, S, T, block)
    B = 3
    q, k, v = _packed(B * n, H, D, 2)
    cu = np.arange(B + 1) * n
    out, lse = oracle.varlen_masked_attention_fp64(q.numpy(), k.numpy(), v.numpy(), cu,
                                                   [(rp, ci)] * B, 1, block)
    bq, bk, bv = (x.reshape(B, n, H, D).permute(0, 2, 1, 3).numpy() for x in (q, k, v))
    ref_o, ref_l = oracle.masked_attention_fp64(bq, bk, bv, rp, ci, 1, block)
    assert np.allclose(out.reshape(B, n, H, D).transpose(0, 2, 1, 3), ref_o, atol=1e-13)
    assert np.allclose(lse.reshape(H, B, n).transpose(1, 0, 2), ref_l, atol=1e-13)


def test_a_token_never_sees_another_item():
    # perturbing item 1's keys and values leaves items 0 and 2 untouched
    cu = np.array([0, 90, 170, 300])
    H, D, block = 1, 8, 32
    q, k, v = _packed(300, H, D, 3)
    lists = [_ones_lists(int(cu[b + 1] - cu[b]), block) for b in range(3)]
    o1, _ = oracle.varlen_masked_attention_fp64(q.numpy(), k.numpy(), v.numpy(), cu, lists, 1,
                                                block)
    k2, v2 = k.clone(), v.clone()
    k2[90:170] += 5.0
    v2[90:170] -= 3.0
    o2, _ = oracle.varlen_masked_attention_fp64(q.numpy(), k2.numpy(), v2.numpy(), cu, lists, 1,
                                                block)
    assert np.array_equal(o1[:90], o2[:90]) and np.array_equal(o1[170:], o2[170:])
    assert not np.allclose(o1[90:170], o2[90:170])


def _token_mask(rp, ci, n, block):
    """Dense [n, n] mask of one item's single-list block lists (built here)."""
    m = np.zeros((n, n), dtype=bool)
    for qb in range(len(rp) - 1):
        for kb in ci[rp[qb]:rp[qb + 1]]:
            m[qb * block:(qb + 1) * block, kb * block:(kb + 1) * block] = True
    return m


def test_backward_equals_autograd_of_block_diagonal_masked_attention():
    # radial items of different lengths, an empty one, and a query block whose
    # row is empty (no key admitted: zero output, zero gradient)
    items = [(3, 40, 10), (0, 0, 0), (4, 48, 0), (2, 30, 5)]
    block, H, D = 32, 2, 8
    lengths = [f * s + t for f, s, t in items]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    total = int(cu[-1])
    lists = []
    for (f, s, t), n in zip(items, lengths):
        lists.append(oracle.joint_block_lists(f, s, t, block) if n else
                     (np.zeros(1, dtype=np.int64), np.zeros(0, dtype=np.int64)))
    rp0, ci0 = lists[2]
    ci0 = np.array(ci0)
    keep = np.ones(ci0.size, dtype=bool)
    keep[rp0[1]:rp0[2]] = False                      # item 2's query block 1: no keys
    counts = np.diff(rp0)
    counts[1] = 0
    lists[2] = (np.concatenate([[0], np.cumsum(counts)]), ci0[keep])
    q, k, v = _packed(total, H, D, 5)
    do = torch.randn((total, H, D), generator=torch.Generator().manual_seed(6),
                     dtype=torch.float64)
    dq, dk, dv = oracle.varlen_masked_attention_backward_fp64(q.numpy(), k.numpy(), v.numpy(),
                                                              do.numpy(), cu, lists, 1, block)
    mask = np.zeros((total, total), dtype=bool)
    for b, n in enumerate(lengths):
        if n:
            t0 = int(cu[b])
            mask[t0:t0 + n, t0:t0 + n] = _token_mask(*lists[b], n, block)
    mask = torch.as_tensor(mask)
    qa, ka, va = (x.clone().requires_grad_(True) for x in (q, k, v))
    s = torch.einsum("thd,shd->hts", qa, ka) * D ** -0.5
    s = s.masked_fill(~mask, float("-inf"))
    p = torch.softmax(s, dim=-1).nan_to_num(0.0)     # rows with no key: all zero
    o = torch.einsum("hts,shd->thd", p, va)
    (o * do).sum().backward()
    for got, ref, name in ((dq, qa.grad, "dq"), (dk, ka.grad, "dk"), (dv, va.grad, "dv")):
        assert np.allclose(got, ref.numpy(), atol=1e-12, rtol=1e-10), name
    t0 = int(cu[2]) + block
    assert np.all(dq[t0:t0 + block] == 0)            # the row with no keys
    assert np.any(dq[int(cu[0]):int(cu[1])] != 0)
