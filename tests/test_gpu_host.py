"""bsa_attn_fwd_host and bsa_attn_bwd_host: the forward and the backward on
host buffers (copies pipelined with the kernels by head groups) give
bit-identical results to bsa_attn_fwd / bsa_attn_bwd on device copies of the
same inputs: same kernels, same per-head arithmetic."""

import numpy as np
import pytest
import torch

from workloads import WORKLOADS, make_generic_lists, make_qkv, make_random_qkv, random_block_lists

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _check(bsa, q, k, v, lists, pin=True, want_lse=True):
    ref_o, ref_l = bsa.attention(q.cuda(), k.cuda(), v.cuda(), lists)
    qh, kh, vh = (t.cpu().contiguous() for t in (q, k, v))
    oh = torch.full(q.shape, float("nan"), dtype=torch.bfloat16)
    lh = torch.full(q.shape[:3], float("nan"), dtype=torch.float32) if want_lse else None
    if pin:
        qh, kh, vh, oh = (t.pin_memory() for t in (qh, kh, vh, oh))
        lh = lh.pin_memory() if lh is not None else None
    stream = torch.cuda.current_stream()
    bsa.bsa_attn_fwd_host(qh, kh, vh, lists, oh, lh, stream=stream)
    stream.synchronize()
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(oh, ref_o.cpu())
    if want_lse:
        assert torch.equal(lh, ref_l.cpu())


def test_wan_heads_in_groups(bsa):
    w = WORKLOADS["wan"]
    q, k, v = make_qkv(w, "cpu", heads=12)   # groups of 2 heads
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    _check(bsa, q, k, v, lists)


def test_per_head_lists_batch_two(bsa):
    B, H, n, D, blk = 2, 5, 1000, 64, 128
    q, k, v = make_random_qkv(B, H, n, D, 3)
    nqb = -(-n // blk)
    rp, ci = random_block_lists(H * nqb, nqb, 0.5, 4, empty_rows=[7], force={0: [nqb - 1]})
    lists = bsa.block_lists_from_csr(rp, ci, H, nqb, blk)
    _check(bsa, q, k, v, lists)


def test_tiny_block64_pageable_no_lse(bsa):
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w, "cpu")
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    _check(bsa, q, k, v, lists, pin=False, want_lse=False)


def test_generic_lists_full_heads(bsa):
    w = WORKLOADS["generic"]
    q, k, v = make_qkv(w, "cpu")
    rp, ci, _ = make_generic_lists(w.heads, w.nqb)
    lists = bsa.block_lists_from_csr(rp, ci, w.heads, w.nqb, w.block)
    _check(bsa, q, k, v, lists)


def _check_bwd(bsa, q, k, v, lists, seed, pin=True):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, lse = bsa.attention(qd, kd, vd, lists)
    g = torch.Generator().manual_seed(seed)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    ref = bsa.attention_backward(qd, kd, vd, out, do.cuda(), lse, lists)
    ins = [t.cpu().contiguous() for t in (q, k, v, out, do, lse)]
    grads = [torch.full(q.shape, float("nan"), dtype=torch.bfloat16) for _ in range(3)]
    if pin:
        ins = [t.pin_memory() for t in ins]
        grads = [t.pin_memory() for t in grads]
    stream = torch.cuda.current_stream()
    bsa.bsa_attn_bwd_host(*ins, lists, *grads, stream=stream)
    stream.synchronize()
    assert bsa.bsa_get_device_status() == 0
    for got, want in zip(grads, ref):
        assert torch.equal(got, want.cpu())


def test_bwd_wan_heads_in_groups(bsa):
    w = WORKLOADS["wan"]
    q, k, v = make_qkv(w, "cpu", heads=12)   # groups of 2 heads
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    _check_bwd(bsa, q, k, v, lists, 11)


def test_bwd_per_head_lists_batch_two(bsa):
    B, H, n, D, blk = 2, 5, 1000, 64, 128
    q, k, v = make_random_qkv(B, H, n, D, 3)
    nqb = -(-n // blk)
    rp, ci = random_block_lists(H * nqb, nqb, 0.5, 4, empty_rows=[7], force={0: [nqb - 1]})
    lists = bsa.block_lists_from_csr(rp, ci, H, nqb, blk)
    _check_bwd(bsa, q, k, v, lists, 12)


def test_bwd_block64_pageable(bsa):
    B, H, n, D, blk = 1, 3, 700, 128, 64
    q, k, v = make_random_qkv(B, H, n, D, 5)
    nqb = -(-n // blk)
    rp, ci = random_block_lists(H * nqb, nqb, 0.4, 6)
    lists = bsa.block_lists_from_csr(rp, ci, H, nqb, blk)
    _check_bwd(bsa, q, k, v, lists, 13, pin=False)


def test_bwd_generic_lists_full_heads(bsa):
    w = WORKLOADS["generic"]
    q, k, v = make_qkv(w, "cpu")
    rp, ci, _ = make_generic_lists(w.heads, w.nqb)
    lists = bsa.block_lists_from_csr(rp, ci, w.heads, w.nqb, w.block)
    _check_bwd(bsa, q, k, v, lists, 14)
