"""Block-64 lists on the two-tile kernel: the 64-blocks merged into 128-row
tile lists whose entries carry the mask of their listed 64 x 64 quarters; the
softmax masks the unlisted quarters.

Checked against the float64 oracle on cases aimed at the packing: a query
half whose listed blocks start late (it carries no reference maximum while its
first tiles are all masked), a query half with nothing listed at all next to
one with keys, score jumps that force a rescale, per-head lists; against the
one-tile kernel (test hook) on the same inputs; and the radial Wan grid at
block 64 on sampled rows.
"""

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, assert_close_device
from workloads import WORKLOADS, make_qkv, make_random_qkv, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _csr(rows):
    rp = np.zeros(len(rows) + 1, dtype=np.int32)
    rp[1:] = np.cumsum([len(set(r)) for r in rows])
    ci = np.array([c for r in rows for c in sorted(set(r))], dtype=np.int32)
    return rp, ci


def test_late_and_empty_query_halves(bsa):
    n, D = 1000, 128                       # 16 blocks of 64 (ragged last)
    nqb = -(-n // 64)
    rows = []
    for q in range(nqb):
        if q == 5:
            rows.append([])                # empty half next to a listed one (q = 4)
        elif q % 2 == 0:
            rows.append([12, 13, nqb - 1])  # even halves list only late key blocks
        else:
            rows.append([0, 1, 2, q])       # odd halves list early ones
    rp, ci = _csr(rows)
    q_, k, v = (t.cuda() for t in make_random_qkv(2, 2, n, D, seed=41))
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, 64)
    out, lse = bsa.attention(q_, k, v, lists)
    assert bsa.bsa_get_device_status() == 0
    ref_o, ref_l = oracle.masked_attention_fp64(q_, k, v, rp, ci, 1, 64)
    assert_close(out, ref_o, lse, ref_l, "late and empty query halves")


def test_rescale_with_quarters(bsa):
    # scores jump upward block after block, so the running maximum moves past
    # the rescale threshold while some quarters are masked
    n, D = 768, 64
    nqb = n // 64
    g = torch.Generator().manual_seed(3)
    q_ = torch.randn((1, 1, n, D), generator=g)
    k = torch.randn((1, 1, n, D), generator=g)
    v = torch.randn((1, 1, n, D), generator=g)
    k *= torch.linspace(0.2, 12.0, n).view(1, 1, n, 1)
    q_, k, v = (t.to(torch.bfloat16) for t in (q_, k, v))
    rows = [[b for b in range(nqb) if (b + q) % 3 != 0 or b == q] for q in range(nqb)]
    rp, ci = _csr(rows)
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, 64)
    out, lse = bsa.attention(q_.cuda(), k.cuda(), v.cuda(), lists)
    assert bsa.bsa_get_device_status() == 0
    ref_o, ref_l = oracle.masked_attention_fp64(q_, k, v, rp, ci, 1, 64)
    assert_close(out, ref_o, lse, ref_l, "rescale with masked quarters")


@pytest.mark.parametrize("D", [64, 128])
def test_two_tile_and_one_tile_kernels_agree(bsa, D):
    H, n = 3, 3000
    q_, k, v = (t.cuda() for t in make_random_qkv(2, H, n, D, seed=D))
    nqb = -(-n // 64)
    rng = np.random.default_rng(D)
    rows = [sorted(set(rng.choice(nqb, size=int(rng.integers(0, 20)), replace=False).tolist()))
            for _ in range(H * nqb)]
    rp, ci = _csr(rows)
    lists = bsa.block_lists_from_csr(rp, ci, H, nqb, 64)
    out2, lse2 = bsa.attention(q_, k, v, lists)
    try:
        bsa.bsa_set_test_hooks(0, 2)       # bit 1: the one-tile kernel
        out1, lse1 = bsa.attention(q_, k, v, lists)
    finally:
        bsa.bsa_set_test_hooks(0, 0)
    assert bsa.bsa_get_device_status() == 0
    ref_o, ref_l = oracle.masked_attention_fp64(q_, k, v, rp, ci, H, 64)
    assert_close(out2, ref_o, lse2, ref_l, "two-tile (quarters) vs oracle")
    assert_close(out1, ref_o, lse1, ref_l, "one-tile vs oracle")


def test_wan_grid_at_block_64(bsa):
    w = WORKLOADS["wan"]
    q_, k, v = make_qkv(w, "cuda", heads=4)
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, 64)
    out, lse = bsa.attention(q_, k, v, lists)
    assert bsa.bsa_get_device_status() == 0
    rp, ci = oracle.radial_block_lists(w.frames, w.tokens_per_frame, 64)
    assert np.array_equal(lists.row_ptr.cpu().numpy(), rp)
    rows = sample_rows(w.n, 64, w.tokens_per_frame, 192, seed=9)
    heads = [0, 3]
    ref_o, ref_l = oracle.masked_attention_fp64(q_.cpu(), k.cpu(), v.cpu(), rp, ci, 1, 64,
                                                rows=rows, heads=heads)
    idx_h = torch.as_tensor(heads, device="cuda")
    idx_r = torch.as_tensor(rows, device="cuda")
    got_o = out.index_select(1, idx_h).index_select(2, idx_r).cpu()
    got_l = lse.index_select(1, idx_h).index_select(2, idx_r).cpu()
    assert_close(got_o, ref_o, got_l, ref_l, "wan grid at block 64 (sampled rows)")
    # the whole output against the fp32 reference kernel
    ro, rl = bsa.dense_masked_reference(q_, k, v, lists)
    assert_close_device(out, ro, lse, rl, "wan grid at block 64 vs fp32 reference")
