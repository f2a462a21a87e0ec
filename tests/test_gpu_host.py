"""bsa_attn_fwd_host: the forward on host buffers (copies pipelined with the
kernels by head groups) gives bit-identical out and lse to bsa_attn_fwd on
device copies of the same inputs: same kernels, same per-head arithmetic."""

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
