"""Variable-length batches on the GPU: the concatenated list builder
(bsa_joint_mask_build_varlen) bit-exact against the oracle, and the varlen
forward (bsa_attn_fwd_varlen) and backward (bsa_attn_bwd_varlen) against the
float64 oracle item by item and, bit for bit, against the regular entries run
on each item alone.

Items differ in frame count, tokens per frame and text length, so their token
counts, query-block counts and lists all differ; one forward launch serves
them all, at block 128 and at block 64 (quarter tiles). Backward bars as the regular backward's (relative RMS 5e-3, max-abs
2e-2 of the oracle's largest entry, per item and tensor).
"""

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close
from workloads import random_block_lists

pytestmark = pytest.mark.gpu

REL_RMS = 5e-3
MAX_REL = 2e-2

ITEMS = [(4, 320, 0), (3, 256, 77), (5, 200, 130)]   # (frames, tokens_per_frame, text)


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


def _packed(total, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((total, H, D), generator=g).to(torch.bfloat16) for _ in range(3)]


def _item_view(x, t0, t1):
    """[1, H, n_b, D] contiguous copy of item tokens t0..t1 of a packed tensor."""
    return x[t0:t1].permute(1, 0, 2).unsqueeze(0).contiguous()


@pytest.mark.parametrize("block", [64, 128])
def test_varlen_lists_bit_exact(bsa, block):
    items = ITEMS + [(1, 50, 0), (21, 1560, 256)]
    lists = bsa.radial_block_lists_varlen(items, block)
    rp, ci = oracle.varlen_block_lists(items, block)
    assert bsa.bsa_get_device_status() == 0
    assert np.array_equal(lists.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(lists.col_idx.cpu().numpy(), ci)
    nqbs = [-(-(f * s + t) // block) for f, s, t in items]
    assert lists.num_q_blocks == sum(nqbs) and lists.num_k_blocks == max(nqbs)


@pytest.mark.parametrize("D", [64, 128])
def test_varlen_radial_against_oracle_and_single_items(bsa, D):
    H = 3
    lengths = [f * s + t for f, s, t in ITEMS]
    cu = _cu(lengths)
    q, k, v = _packed(int(cu[-1]), H, D, seed=D)
    lists = bsa.radial_block_lists_varlen(ITEMS, 128)
    out, lse = bsa.attention_varlen(q.cuda(), k.cuda(), v.cuda(), cu, lists)
    assert bsa.bsa_get_device_status() == 0
    rp, ci = oracle.varlen_block_lists(ITEMS, 128)
    nqbs = [-(-n // 128) for n in lengths]
    item_lists = oracle.split_item_lists(rp, ci, nqbs)
    ref_o, ref_l = oracle.varlen_masked_attention_fp64(q.float().numpy(), k.float().numpy(),
                                                       v.float().numpy(), cu, item_lists, 1, 128)
    o, l_ = out.cpu(), lse.cpu()
    for b, (f, s, t) in enumerate(ITEMS):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        assert_close(o[t0:t1].float().numpy(), ref_o[t0:t1], l_[:, t0:t1].numpy(),
                     ref_l[:, t0:t1], f"varlen item {b} ({f}x{s}+{t})")
        # the same item through the regular entry, alone: identical bits
        one = bsa.radial_block_lists(f, s, 128, text_tokens=t)
        qi, ki, vi = (_item_view(x, t0, t1).cuda() for x in (q, k, v))
        oi, li = bsa.attention(qi, ki, vi, one)
        assert torch.equal(oi[0].permute(1, 0, 2).cpu(), o[t0:t1]), f"item {b} output differs"
        assert torch.equal(li[0].cpu(), l_[:, t0:t1]), f"item {b} lse differs"


def test_varlen_per_head_lists_and_an_empty_item(bsa):
    H, D, blk = 4, 128, 128
    lengths = [500, 0, 1, 383, 1024]
    cu = _cu(lengths)
    q, k, v = _packed(int(cu[-1]), H, D, seed=7)
    nqbs = [-(-n // blk) for n in lengths]
    rps, cis, item_lists, off = [], [], [], 0
    for b, nqb in enumerate(nqbs):
        if nqb == 0:
            item_lists.append((np.zeros(1, dtype=np.int64), np.zeros(0, dtype=np.int64)))
            continue
        rp, ci = random_block_lists(H * nqb, nqb, 0.5, seed=20 + b)
        item_lists.append((rp, ci))
        rps.append(np.asarray(rp[:-1]) + off)
        cis.append(np.asarray(ci))
        off += int(rp[-1])
    row_ptr = np.concatenate(rps + [np.array([off])])
    col_idx = np.concatenate(cis)
    lists = bsa.block_lists_from_csr(row_ptr, col_idx, H, sum(nqbs), blk)
    lists.k_blocks = max(nqbs)
    out, lse = bsa.attention_varlen(q.cuda(), k.cuda(), v.cuda(), cu, lists)
    assert bsa.bsa_get_device_status() == 0
    ref_o, ref_l = oracle.varlen_masked_attention_fp64(q.float().numpy(), k.float().numpy(),
                                                       v.float().numpy(), cu, item_lists, H, blk)
    assert_close(out.cpu().float().numpy(), ref_o, lse.cpu().numpy(), ref_l, "per-head varlen")


def test_varlen_medium_batch_matches_single_items(bsa):
    # larger items, many work items per launch: every item bit-identical to
    # its own regular call (itself checked against the oracle elsewhere)
    items = [(8, 1560, 256), (5, 3600, 0), (12, 780, 64)]
    H, D = 8, 128
    lengths = [f * s + t for f, s, t in items]
    cu = _cu(lengths)
    g = torch.Generator(device="cuda").manual_seed(3)
    q, k, v = (torch.randn((int(cu[-1]), H, D), generator=g, device="cuda").to(torch.bfloat16)
               for _ in range(3))
    lists = bsa.radial_block_lists_varlen(items, 128)
    out, lse = bsa.attention_varlen(q, k, v, cu, lists)
    assert bsa.bsa_get_device_status() == 0
    for b, (f, s, t) in enumerate(items):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        one = bsa.radial_block_lists(f, s, 128, text_tokens=t)
        oi, li = bsa.attention(*(_item_view(x, t0, t1) for x in (q, k, v)), one)
        assert torch.equal(oi[0].permute(1, 0, 2), out[t0:t1]), f"item {b} output differs"
        assert torch.equal(li[0], lse[:, t0:t1]), f"item {b} lse differs"


def _grad_close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = got - ref
    rel_rms = np.sqrt((err ** 2).mean()) / max(np.sqrt((ref ** 2).mean()), 1e-30)
    max_rel = np.abs(err).max() / max(np.abs(ref).max(), 1e-30)
    assert rel_rms <= REL_RMS, f"{what}: relative RMS {rel_rms:.3e}"
    assert max_rel <= MAX_REL, f"{what}: max-abs {max_rel:.3e} of max |ref|"


def _nan_grads(q):
    return tuple(torch.full_like(q, float("nan")) for _ in range(3))


@pytest.mark.parametrize("D", [64, 128])
def test_varlen_backward_against_oracle_and_single_items(bsa, D):
    H = 3
    lengths = [f * s + t for f, s, t in ITEMS]
    cu = _cu(lengths)
    total = int(cu[-1])
    q, k, v = _packed(total, H, D, seed=10 + D)
    do = torch.randn((total, H, D), generator=torch.Generator().manual_seed(D)).to(torch.bfloat16)
    lists = bsa.radial_block_lists_varlen(ITEMS, 128)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    out, lse = bsa.attention_varlen(qd, kd, vd, cu, lists)
    dq, dk, dv = _nan_grads(qd)
    bsa.bsa_attn_bwd_varlen(qd, kd, vd, out, dod, lse, cu, lists, dq, dk, dv)
    assert bsa.bsa_get_device_status() == 0
    rp, ci = oracle.varlen_block_lists(ITEMS, 128)
    item_lists = oracle.split_item_lists(rp, ci, [-(-n // 128) for n in lengths])
    refs = oracle.varlen_masked_attention_backward_fp64(
        q.float().numpy(), k.float().numpy(), v.float().numpy(), do.float().numpy(), cu,
        item_lists, 1, 128)
    got = [g.cpu() for g in (dq, dk, dv)]
    for b, (f, s, t) in enumerate(ITEMS):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        for g, r, name in zip(got, refs, ("dq", "dk", "dv")):
            _grad_close(g[t0:t1].float().numpy(), r[t0:t1], f"varlen item {b} {name}")
        # the item alone through bsa_attn_bwd: identical bits
        one = bsa.radial_block_lists(f, s, 128, text_tokens=t)
        views = [_item_view(x, t0, t1) for x in (qd, kd, vd, out, dod)]
        li = lse[:, t0:t1].contiguous().unsqueeze(0)
        gi = bsa.attention_backward(*views, li, one)
        for g, g1, name in zip(got, gi, ("dq", "dk", "dv")):
            assert torch.equal(g1[0].permute(1, 0, 2).cpu(), g[t0:t1]), f"item {b} {name} differs"


def test_varlen_backward_per_head_lists_and_edge_items(bsa):
    # per-head lists; an empty item, a one-token item, an item of exactly one
    # block and rows with no listed key (zero gradients there)
    H, D, blk = 2, 128, 128
    lengths = [300, 0, 1, 128, 700]
    cu = _cu(lengths)
    total = int(cu[-1])
    q, k, v = _packed(total, H, D, seed=17)
    do = torch.randn((total, H, D), generator=torch.Generator().manual_seed(18)).to(torch.bfloat16)
    nqbs = [-(-n // blk) for n in lengths]
    rps, cis, item_lists, off = [], [], [], 0
    for b, nqb in enumerate(nqbs):
        if nqb == 0:
            item_lists.append((np.zeros(1, dtype=np.int64), np.zeros(0, dtype=np.int64)))
            continue
        rp, ci = random_block_lists(H * nqb, nqb, 0.5, seed=40 + b)
        item_lists.append((rp, ci))
        rps.append(np.asarray(rp[:-1]) + off)
        cis.append(np.asarray(ci))
        off += int(rp[-1])
    row_ptr = np.concatenate(rps + [np.array([off])])
    col_idx = np.concatenate(cis)
    lists = bsa.block_lists_from_csr(row_ptr, col_idx, H, sum(nqbs), blk)
    lists.k_blocks = max(nqbs)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    out, lse = bsa.attention_varlen(qd, kd, vd, cu, lists)
    dq, dk, dv = bsa.attention_varlen_backward(qd, kd, vd, out, dod, lse, cu, lists)
    assert bsa.bsa_get_device_status() == 0
    refs = oracle.varlen_masked_attention_backward_fp64(
        q.float().numpy(), k.float().numpy(), v.float().numpy(), do.float().numpy(), cu,
        item_lists, H, blk)
    for g, r, name in zip((dq, dk, dv), refs, ("dq", "dk", "dv")):
        _grad_close(g.cpu().float().numpy(), r, f"per-head varlen {name}")


def test_varlen_backward_medium_batch_matches_single_items(bsa):
    items = [(8, 1560, 256), (5, 3600, 0), (12, 780, 64)]
    H, D = 4, 128
    lengths = [f * s + t for f, s, t in items]
    cu = _cu(lengths)
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v, do = (torch.randn((int(cu[-1]), H, D), generator=g, device="cuda")
                   .to(torch.bfloat16) for _ in range(4))
    lists = bsa.radial_block_lists_varlen(items, 128)
    out, lse = bsa.attention_varlen(q, k, v, cu, lists)
    dq, dk, dv = bsa.attention_varlen_backward(q, k, v, out, do, lse, cu, lists)
    assert bsa.bsa_get_device_status() == 0
    for b, (f, s, t) in enumerate(items):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        one = bsa.radial_block_lists(f, s, 128, text_tokens=t)
        views = [_item_view(x, t0, t1) for x in (q, k, v, out, do)]
        gi = bsa.attention_backward(*views, lse[:, t0:t1].contiguous().unsqueeze(0), one)
        for got, g1, name in zip((dq, dk, dv), gi, ("dq", "dk", "dv")):
            assert torch.equal(g1[0].permute(1, 0, 2), got[t0:t1]), f"item {b} {name} differs"


@pytest.mark.parametrize("D", [64, 128])
def test_varlen_block64_forward_and_backward(bsa, D):
    """Block-64 lists of a variable-length batch (items merged into 128-row
    tiles with quarter masks, item by item): forward and backward against the
    float64 oracle per item and bit-identical to the regular block-64 entries
    on each item alone."""
    H = 2
    items = ITEMS + [(1, 50, 0)]                  # the last item: one block of 64
    lengths = [f * s + t for f, s, t in items]
    cu = _cu(lengths)
    total = int(cu[-1])
    q, k, v = _packed(total, H, D, seed=30 + D)
    do = torch.randn((total, H, D), generator=torch.Generator().manual_seed(D + 1)).to(torch.bfloat16)
    lists = bsa.radial_block_lists_varlen(items, 64)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    out, lse = bsa.attention_varlen(qd, kd, vd, cu, lists)
    dq, dk, dv = bsa.attention_varlen_backward(qd, kd, vd, out, dod, lse, cu, lists)
    assert bsa.bsa_get_device_status() == 0
    rp, ci = oracle.varlen_block_lists(items, 64)
    item_lists = oracle.split_item_lists(rp, ci, [-(-n // 64) for n in lengths])
    qf, kf, vf, df = (x.float().numpy() for x in (q, k, v, do))
    ref_o, ref_l = oracle.varlen_masked_attention_fp64(qf, kf, vf, cu, item_lists, 1, 64)
    refs = oracle.varlen_masked_attention_backward_fp64(qf, kf, vf, df, cu, item_lists, 1, 64)
    o, l_ = out.cpu(), lse.cpu()
    got = [g.cpu() for g in (dq, dk, dv)]
    for b, (f, s_, t) in enumerate(items):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        assert_close(o[t0:t1].float().numpy(), ref_o[t0:t1], l_[:, t0:t1].numpy(),
                     ref_l[:, t0:t1], f"block-64 varlen item {b}")
        for g, r, name in zip(got, refs, ("dq", "dk", "dv")):
            _grad_close(g[t0:t1].float().numpy(), r[t0:t1], f"block-64 varlen item {b} {name}")
        one = bsa.radial_block_lists(f, s_, 64, text_tokens=t)
        views = [_item_view(x, t0, t1) for x in (qd, kd, vd)]
        oi, li = bsa.attention(*views, one)
        assert torch.equal(oi[0].permute(1, 0, 2).cpu(), o[t0:t1]), f"item {b} output differs"
        assert torch.equal(li[0].cpu(), l_[:, t0:t1]), f"item {b} lse differs"
        gi = bsa.attention_backward(*views, _item_view(out, t0, t1), _item_view(dod, t0, t1),
                                    lse[:, t0:t1].contiguous().unsqueeze(0), one)
        for g, g1, name in zip(got, gi, ("dq", "dk", "dv")):
            assert torch.equal(g1[0].permute(1, 0, 2).cpu(), g[t0:t1]), f"item {b} {name} differs"


def test_varlen_block64_per_head_lists_and_edge_items(bsa):
    # per-head random block-64 lists; an empty item, a one-token item and an
    # item of an odd number of 64-blocks; forward and backward against the oracle
    H, D, blk = 2, 64, 64
    lengths = [300, 0, 1, 192, 700]
    cu = _cu(lengths)
    total = int(cu[-1])
    q, k, v = _packed(total, H, D, seed=51)
    do = torch.randn((total, H, D), generator=torch.Generator().manual_seed(52)).to(torch.bfloat16)
    nqbs = [-(-n // blk) for n in lengths]
    rps, cis, item_lists, off = [], [], [], 0
    for b, nqb in enumerate(nqbs):
        if nqb == 0:
            item_lists.append((np.zeros(1, dtype=np.int64), np.zeros(0, dtype=np.int64)))
            continue
        rp, ci = random_block_lists(H * nqb, nqb, 0.5, seed=60 + b)
        item_lists.append((rp, ci))
        rps.append(np.asarray(rp[:-1]) + off)
        cis.append(np.asarray(ci))
        off += int(rp[-1])
    row_ptr = np.concatenate(rps + [np.array([off])])
    col_idx = np.concatenate(cis)
    lists = bsa.block_lists_from_csr(row_ptr, col_idx, H, sum(nqbs), blk)
    lists.k_blocks = max(nqbs)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    out, lse = bsa.attention_varlen(qd, kd, vd, cu, lists)
    dq, dk, dv = bsa.attention_varlen_backward(qd, kd, vd, out, dod, lse, cu, lists)
    assert bsa.bsa_get_device_status() == 0
    qf, kf, vf, df = (x.float().numpy() for x in (q, k, v, do))
    ref_o, ref_l = oracle.varlen_masked_attention_fp64(qf, kf, vf, cu, item_lists, H, blk)
    assert_close(out.cpu().float().numpy(), ref_o, lse.cpu().numpy(), ref_l,
                 "per-head block-64 varlen")
    refs = oracle.varlen_masked_attention_backward_fp64(qf, kf, vf, df, cu, item_lists, H, blk)
    for g, r, name in zip((dq, dk, dv), refs, ("dq", "dk", "dv")):
        _grad_close(g.cpu().float().numpy(), r, f"per-head block-64 varlen {name}")
