"""Attention parity: the tcgen05 kernel and the fp32 reference kernel against the
float64 CPU oracle on the same seeded bf16 inputs, plus edge cases."""

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, assert_close_device
from workloads import WORKLOADS, make_generic_lists, make_qkv, make_random_qkv, random_block_lists, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _run(bsa, q, k, v, lists, scale=0.0):
    out, lse = bsa.attention(q, k, v, lists, softmax_scale=scale)
    ref_o, ref_l = bsa.dense_masked_reference(q, k, v, lists, softmax_scale=scale)
    assert bsa.bsa_get_device_status() == 0
    return out, lse, ref_o, ref_l


def _host_lists(lists):
    return lists.row_ptr.cpu().numpy(), lists.col_idx.cpu().numpy()


def test_tiny_config_full(bsa):
    w = WORKLOADS["tiny"]
    q, k, v = (t.cuda() for t in make_qkv(w, "cpu"))
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    out, lse, ro, rl = _run(bsa, q, k, v, lists)
    rp, ci = _host_lists(lists)
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, w.block)
    assert_close(out, ref_o, lse, ref_l, "tcgen05 vs oracle")
    assert_close(ro, ref_o, rl, ref_l, "fp32 reference vs oracle")


CASES = [
    # (batch, heads, n, D, block, num_lists, seed)
    (1, 1, 256, 64, 64, 1, 1),
    (2, 3, 1000, 64, 64, 3, 2),        # ragged, per-head lists, batch > 1
    (1, 2, 1025, 128, 64, 1, 3),       # last block holds one valid key
    (2, 2, 640, 128, 128, 2, 4),       # ragged at block 128
    (1, 2, 1024, 64, 128, 1, 5),
    (1, 1, 129, 128, 128, 1, 6),       # two blocks, second with one key
    (1, 4, 2048, 128, 128, 4, 7),
    (3, 1, 384, 128, 64, 1, 8),
]


@pytest.mark.parametrize("B,H,n,D,blk,L,seed", CASES)
def test_random_lists_full(bsa, B, H, n, D, blk, L, seed):
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, seed))
    nqb = -(-n // blk)
    force = {1 % (L * nqb): [nqb - 1], (2 % (L * nqb)): [0]}
    rp, ci = random_block_lists(L * nqb, nqb, 0.4, seed + 100,
                                empty_rows=[L * nqb - 1] if L * nqb > 3 else [], force=force)
    lists = bsa.block_lists_from_csr(rp, ci, L, nqb, blk)
    assert bsa.bsa_validate_lists(lists) == 0
    out, lse, ro, rl = _run(bsa, q, k, v, lists)
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, L, blk)
    assert_close(out, ref_o, lse, ref_l, "tcgen05 vs oracle")
    assert_close(ro, ref_o, rl, ref_l, "fp32 reference vs oracle")


@pytest.mark.parametrize("D,blk", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_all_ones_lists_is_dense_attention(bsa, D, blk):
    n = 1000
    q, k, v = (t.cuda() for t in make_random_qkv(1, 2, n, D, seed=21))
    nqb = -(-n // blk)
    rp = np.arange(nqb + 1, dtype=np.int32) * nqb
    ci = np.tile(np.arange(nqb, dtype=np.int32), nqb)
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, blk)
    out, lse = bsa.attention(q, k, v, lists)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double().cpu(), k.double().cpu(),
                                                           v.double().cpu()).numpy()
    ref_l = torch.logsumexp(q.double().cpu() @ k.double().cpu().transpose(-1, -2) * D ** -0.5,
                            dim=-1).numpy()
    assert_close(out, ref, lse, ref_l, "dense")


def test_running_max_jumps_trigger_rescale(bsa):
    """Later key blocks score far higher, so the running max jumps past the
    lazy-rescale threshold several times."""
    n, D, blk = 1024, 128, 128
    q, k, v = make_random_qkv(1, 2, n, D, seed=31)
    ramp = torch.linspace(0.2, 6.0, n).view(1, 1, n, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    nqb = n // blk
    rp = np.arange(nqb + 1, dtype=np.int32) * nqb
    ci = np.tile(np.arange(nqb, dtype=np.int32), nqb)
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, blk)
    out, lse, ro, rl = _run(bsa, q, k, v, lists)
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, blk)
    assert_close(out, ref_o, lse, ref_l, "tcgen05 vs oracle")
    assert_close(ro, ref_o, rl, ref_l, "fp32 reference vs oracle")


@pytest.mark.parametrize("top", [12.0, 40.0])
def test_running_max_jump_forces_a_rescale(bsa, top):
    """Scores of later key blocks exceed the first block's maximum by tens of
    log2 units: with the smaller ramp P grows to about 2^50 against the first
    block's reference (no rescale needed); with the larger one a row sum
    leaves [0, 2^64] or overflows to inf, and the kernels take the row
    maximum again and rescale O and l."""
    n, D, blk = 1024, 128, 128
    q, k, v = make_random_qkv(1, 2, n, D, seed=32)
    ramp = torch.linspace(0.2, top, n).view(1, 1, n, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    # such peaked rows return about one V row each: V at a quarter of unit
    # scale keeps |out| (and its bf16 rounding) inside the absolute bound
    v = (v.float() * 0.25).to(torch.bfloat16)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    nqb = n // blk
    rp = np.arange(nqb + 1, dtype=np.int32) * nqb
    ci = np.tile(np.arange(nqb, dtype=np.int32), nqb)
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, blk)
    out, lse, ro, rl = _run(bsa, q, k, v, lists)
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, blk)
    assert_close(out, ref_o, lse, ref_l, "tcgen05 vs oracle")


def test_explicit_scale_and_no_lse(bsa):
    n, D, blk = 512, 64, 64
    q, k, v = (t.cuda() for t in make_random_qkv(1, 1, n, D, seed=41))
    nqb = n // blk
    rp, ci = random_block_lists(nqb, nqb, 0.5, seed=42, force={0: [0]})
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, blk)
    out, _ = bsa.attention(q, k, v, lists, softmax_scale=0.3, want_lse=False)
    ref_o, _ = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, blk, scale=0.3)
    assert_close(out, ref_o, what="scale 0.3")


def test_repeat_calls_are_bitwise_identical(bsa):
    w = WORKLOADS["wan"]
    q, k, v = make_qkv(w, "cuda", heads=4)
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    o1, l1 = bsa.attention(q, k, v, lists)
    o2, l2 = bsa.attention(q, k, v, lists)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _check_large(bsa, name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, "cuda")
    if w.radial:
        lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block,
                                       text_tokens=w.text_tokens)
        num_lists = 1
    else:
        rp, ci, _ = make_generic_lists(w.heads, w.nqb)
        lists = bsa.block_lists_from_csr(rp, ci, w.heads, w.nqb, w.block)
        num_lists = w.heads
    out, lse, ro, rl = _run(bsa, q, k, v, lists)
    # full tensors against the fp32 reference kernel
    assert_close_device(out, ro, lse, rl, f"{name}: tcgen05 vs fp32 reference")
    # sampled rows of three heads against the float64 oracle, for both kernels
    rp, ci = _host_lists(lists)
    rows = sample_rows(w.n, w.block, w.tokens_per_frame, 512, seed=w.seed)
    if w.text_tokens:  # both sides of the video / text boundary (a mixed block)
        nv = w.n - w.text_tokens
        rows = np.unique(np.r_[rows, nv - 16, nv - 1, nv, nv + 1])
    heads = sorted({0, w.heads // 2, w.heads - 1})
    ref_o = np.zeros((1, len(heads), rows.size, w.head_dim))
    ref_l = np.zeros((1, len(heads), rows.size))
    for i, h in enumerate(heads):
        base = (h if num_lists > 1 else 0) * w.nqb
        rph = rp[base:base + w.nqb + 1] - rp[base]
        cih = ci[rp[base]:rp[base + w.nqb]]
        o_h, l_h = oracle.masked_attention_fp64(q[:, h:h + 1].cpu(), k[:, h:h + 1].cpu(),
                                                v[:, h:h + 1].cpu(), rph, cih, 1, w.block,
                                                rows=rows)
        ref_o[:, i], ref_l[:, i] = o_h[:, 0], l_h[:, 0]
    sel = lambda t: t[:, heads][:, :, torch.as_tensor(rows, device=t.device)]
    assert_close(sel(out), ref_o, sel(lse), ref_l, f"{name}: tcgen05 vs oracle (sampled)")
    assert_close(sel(ro), ref_o, sel(rl), ref_l, f"{name}: fp32 reference vs oracle (sampled)")


@pytest.mark.parametrize("name", ["wan", "hunyuan", "long4x", "generic", "hunyuan_text"])
def test_full_size_configs(bsa, name):
    _check_large(bsa, name)


@pytest.mark.parametrize("B,H,n,D,L,seed", [(1, 2, 640, 128, 1, 21), (2, 1, 1152, 64, 1, 22),
                                            (1, 3, 1000, 128, 3, 23)])
def test_one_tile_and_two_tile_schedules_agree(bsa, B, H, n, D, L, seed):
    """Block-128 problems run on the two-tile kernel by default; hook bit 1
    routes them to the one-tile kernel. Both match the oracle, and an odd
    number of query blocks leaves the last pair with a single tile."""
    blk = 128
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, seed))
    nqb = -(-n // blk)
    rp, ci = random_block_lists(L * nqb, nqb, 0.45, seed + 7, empty_rows=[1] if L * nqb > 2 else [],
                                force={0: [nqb - 1]})
    lists = bsa.block_lists_from_csr(rp, ci, L, nqb, blk)
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, L, blk)
    o2, l2 = bsa.attention(q, k, v, lists)
    try:
        bsa.bsa_set_test_hooks(0, 2)
        o1, l1 = bsa.attention(q, k, v, lists)
    finally:
        bsa.bsa_set_test_hooks(0, 0)
    assert bsa.bsa_get_device_status() == 0
    assert_close(o2, ref_o, l2, ref_l, "two-tile vs oracle")
    assert_close(o1, ref_o, l1, ref_l, "one-tile vs oracle")
