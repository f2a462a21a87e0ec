"""Pins of the variable-length oracle (oracle/varlen.py) on the CPU.

The pages batch nothing of different lengths; the reading is that each item is
its own problem. These checks tie the oracle to constructions that do not go
through it: dense softmax attention with a block-diagonal mask over the packed
sequence (torch SDPA in float64, the mask built here), the batched oracle for
items of equal length, and the items' own lists split back out.
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
