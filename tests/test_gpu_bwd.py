"""Backward parity: bsa_attn_bwd (tcgen05 kernels) against the float64 backward
oracle on the same seeded bf16 inputs.

Tolerance (derived from the arithmetic, not from the pages, which fix no
precision for the backward): P, dS and the output O that delta is built from
are rounded to bf16 (relative 2^-9 each) before the bf16 x bf16 -> fp32 MMAs,
and dQ, dK, dV are rounded to bf16 on output (2^-9). The gradient of a row
is a sum of many such terms with independent rounding, so the relative RMS
error stays near a few 2^-9; dS = P (dP - delta) loses relative accuracy where
dP is close to delta, which the max-abs bound (relative to the tensor's
largest entry) absorbs. Bars: the forward's relative RMS 5e-3 and max-abs
2e-2, the max-abs taken relative to the oracle's largest entry, per tensor
(measured: about 2.4e-3 and 4e-3 on the random cases).
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_qkv, make_random_qkv, random_block_lists

pytestmark = pytest.mark.gpu

REL_RMS = 5e-3
MAX_REL = 2e-2


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    scale = max(np.abs(ref).max(), 1e-30)
    err = got - ref
    rel_rms = np.sqrt((err ** 2).mean()) / max(np.sqrt((ref ** 2).mean()), 1e-30)
    max_rel = np.abs(err).max() / scale
    assert rel_rms <= REL_RMS, f"{what}: relative RMS {rel_rms:.3e}"
    assert max_rel <= MAX_REL, f"{what}: max-abs {max_rel:.3e} of max |ref|"
    return rel_rms, max_rel


def _dout(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def _run(bsa, q, k, v, lists, do, scale=0.0):
    out, lse = bsa.attention(q, k, v, lists, softmax_scale=scale)
    dq, dk, dv = bsa.attention_backward(q, k, v, out, do, lse, lists, softmax_scale=scale)
    assert bsa.bsa_get_device_status() == 0
    return dq, dk, dv


CASES = [
    # (batch, heads, n, D, num_lists, seed)
    (1, 1, 256, 128, 1, 1),
    (1, 2, 640, 128, 2, 2),      # per-head lists
    (2, 2, 1000, 64, 1, 3),      # batch > 1, ragged last block
    (1, 3, 1153, 128, 3, 4),     # last block holds one row
    (1, 1, 129, 64, 1, 5),
]


@pytest.mark.parametrize("B,H,n,D,L,seed", CASES)
def test_random_lists_full(bsa, B, H, n, D, L, seed):
    _random_case(bsa, B, H, n, D, L, seed, 128)


CASES_64 = [
    # block 64: the kernels run 128-row tiles with a per-entry mask of the
    # listed 64 x 64 pairs
    (1, 1, 256, 64, 1, 31),
    (1, 2, 1000, 128, 2, 32),    # per-head lists, ragged
    (2, 2, 1050, 64, 1, 33),     # odd number of 64-blocks, batch > 1
    (1, 3, 640, 128, 3, 34),
]


@pytest.mark.parametrize("B,H,n,D,L,seed", CASES_64)
def test_random_lists_full_block64(bsa, B, H, n, D, L, seed):
    _random_case(bsa, B, H, n, D, L, seed, 64)


def _random_case(bsa, B, H, n, D, L, seed, blk):
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, seed))
    nqb = -(-n // blk)
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, seed + 100,
                                empty_rows=[L * nqb - 1] if L * nqb > 3 else [],
                                force={0: [nqb - 1]})
    lists = bsa.block_lists_from_csr(rp, ci, L, nqb, blk)
    do = _dout((B, H, n, D), seed + 7).cuda()
    dq, dk, dv = _run(bsa, q, k, v, lists, do)
    rq, rk, rv = oracle.masked_attention_backward_fp64(q, k, v, do, rp, ci, L, blk)
    _close(dq.float().cpu(), rq, "dq")
    _close(dk.float().cpu(), rk, "dk")
    _close(dv.float().cpu(), rv, "dv")


def test_tiny_radial_block64(bsa):
    """The tiny radial configuration (4 x 256 tokens, block 64, D = 64)."""
    w = WORKLOADS["tiny"]
    q, k, v = (t.cuda() for t in make_qkv(w, "cpu"))
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    rp, ci = oracle.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    do = _dout(q.shape, 51).cuda()
    dq, dk, dv = _run(bsa, q, k, v, lists, do)
    rq, rk, rv = oracle.masked_attention_backward_fp64(q, k, v, do, rp, ci, 1, w.block)
    _close(dq.float().cpu(), rq, "dq")
    _close(dk.float().cpu(), rk, "dk")
    _close(dv.float().cpu(), rv, "dv")


def test_all_ones_lists_match_float64_sdpa(bsa):
    B, H, n, D = 1, 2, 512, 128
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, 11))
    nqb = n // 128
    rp = np.arange(0, nqb * nqb + 1, nqb)
    ci = np.tile(np.arange(nqb), nqb)
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, 128)
    do = _dout((B, H, n, D), 12).cuda()
    dq, dk, dv = _run(bsa, q, k, v, lists, do)
    qt, kt, vt = (t.cpu().double().requires_grad_() for t in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    (o * do.cpu().double()).sum().backward()
    _close(dq.float().cpu(), qt.grad, "dq")
    _close(dk.float().cpu(), kt.grad, "dk")
    _close(dv.float().cpu(), vt.grad, "dv")


def test_empty_lists_give_zero_gradients(bsa):
    B, H, n, D = 1, 1, 384, 64
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, 21))
    nqb = 3
    rp = np.array([0, 0, 1, 1])
    ci = np.array([1])   # only query block 1 attends, to key block 1
    lists = bsa.block_lists_from_csr(rp, ci, 1, nqb, 128)
    do = _dout((B, H, n, D), 22).cuda()
    dq, dk, dv = _run(bsa, q, k, v, lists, do)
    assert torch.all(dq[:, :, :128] == 0) and torch.all(dq[:, :, 256:] == 0)
    assert torch.all(dk[:, :, :128] == 0) and torch.all(dv[:, :, 256:] == 0)
    rq, rk, rv = oracle.masked_attention_backward_fp64(q, k, v, do, rp, ci, 1, 128)
    _close(dq.float().cpu(), rq, "dq")
    _close(dv.float().cpu(), rv, "dv")


def test_backward_is_deterministic(bsa):
    w = WORKLOADS["wan"]
    q, k, v = make_qkv(w, "cuda", heads=4)
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    do = _dout(q.shape, 31).cuda()
    out, lse = bsa.attention(q, k, v, lists)
    g1 = bsa.attention_backward(q, k, v, out, do, lse, lists)
    g2 = bsa.attention_backward(q, k, v, out, do, lse, lists)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_wan_sampled_rows_and_keys(bsa):
    """Full-size Wan layout (radial lists, n = 32760) on 4 heads; dQ checked on
    sampled query rows and dK, dV on sampled keys of two key blocks, against
    the oracle's per-row and per-key functions."""
    w = WORKLOADS["wan"]
    H = 4
    q, k, v = make_qkv(w, "cuda", heads=H)
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    rp, ci = lists.row_ptr.cpu().numpy(), lists.col_idx.cpu().numpy()
    do = _dout(q.shape, 41).cuda()
    dq, dk, dv = _run(bsa, q, k, v, lists, do)
    qc, kc, vc, dc = (t.cpu() for t in (q, k, v, do))
    rng = np.random.default_rng(5)
    rows = np.unique(np.r_[0, w.n - 1, rng.integers(0, w.n, 60)])
    keys = np.r_[np.arange(5) * 25, 128 * 200 + np.arange(5) * 25, w.n - 1]
    for h in (0, H - 1):
        rq = oracle.masked_attention_dq_rows(qc, kc, vc, dc, rp, ci, 1, w.block, 0, h, rows)
        _close(dq[0, h, rows].float().cpu(), rq, f"dq head {h}")
    rk, rv = oracle.masked_attention_dkdv_keys(qc, kc, vc, dc, rp, ci, 1, w.block, 0, 0, keys)
    _close(dk[0, 0, keys].float().cpu(), rk, "dk head 0")
    _close(dv[0, 0, keys].float().cpu(), rv, "dv head 0")


@pytest.mark.parametrize("B,H,n,D,blk,L,seed", [(1, 3, 1000, 128, 128, 1, 61),
                                                (2, 2, 700, 64, 64, 2, 62)])
def test_strided_views_match_contiguous_bit_for_bit(bsa, B, H, n, D, blk, L, seed):
    """q, k, v as slices of a [B, n, 3, H, D] projection buffer, out and dout
    token-major, gradients into the slices of a second such buffer: the same
    bits as the contiguous entry point."""
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, seed))
    nqb = -(-n // blk)
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, seed + 100, force={0: [nqb - 1]})
    lists = bsa.block_lists_from_csr(rp, ci, L, nqb, blk)
    do = _dout((B, H, n, D), seed + 7).cuda()
    out, lse = bsa.attention(q, k, v, lists)
    ref = bsa.attention_backward(q, k, v, out, do, lse, lists)
    tok = lambda t: t.transpose(1, 2).contiguous().transpose(1, 2)  # noqa: E731
    buf = torch.stack([t.transpose(1, 2) for t in (q, k, v)], dim=2).contiguous()
    qv, kv, vv = (buf[:, :, i].transpose(1, 2) for i in range(3))
    gbuf = torch.full((B, n, 3, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    grads = tuple(gbuf[:, :, i].transpose(1, 2) for i in range(3))
    got = bsa.attention_backward(qv, kv, vv, tok(out), tok(do), lse, lists, grads=grads)
    assert bsa.bsa_get_device_status() == 0
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        assert torch.equal(a, b), name
    assert not torch.isnan(gbuf.float()).any()


@pytest.mark.parametrize("B,H,n,D,L,seed", [(1, 2, 1000, 128, 2, 71), (2, 1, 1280, 64, 1, 72),
                                            (1, 1, 2048, 128, 1, 73)])
def test_one_pass_and_two_kernel_paths_agree(bsa, B, H, n, D, L, seed):
    """Block 128: bsa_attn_bwd_one_pass (dQ parts added in each query row's
    key order) and bsa_attn_bwd (dK/dV, then dQ with S and dP recomputed) both
    within the bars of the oracle, rows with many parts (dense lists: up to
    16 key blocks per row) and empty rows included; the one pass repeats bit
    for bit."""
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, seed))
    nqb = -(-n // 128)
    dens = 0.9 if n >= 2048 else 0.5
    rp, ci = random_block_lists(L * nqb, nqb, dens, seed + 100,
                                empty_rows=[L * nqb - 1], force={0: [nqb - 1]})
    lists = bsa.block_lists_from_csr(rp, ci, L, nqb, 128)
    do = _dout((B, H, n, D), seed + 7).cuda()
    g2 = _run(bsa, q, k, v, lists, do)
    out, lse = bsa.attention(q, k, v, lists)
    g1 = tuple(torch.empty_like(q) for _ in range(3))
    bsa.bsa_attn_bwd_one_pass(q, k, v, out, do, lse, lists, *g1)
    g3 = tuple(torch.empty_like(q) for _ in range(3))
    bsa.bsa_attn_bwd_one_pass(q, k, v, out, do, lse, lists, *g3)
    assert bsa.bsa_get_device_status() == 0
    assert all(torch.equal(a, b) for a, b in zip(g1, g3))
    refs = oracle.masked_attention_backward_fp64(q, k, v, do, rp, ci, L, 128)
    for a, b, r, name in zip(g1, g2, refs, ("dq", "dk", "dv")):
        _close(a.float().cpu(), r, f"{name} one pass")
        _close(b.float().cpu(), r, f"{name} two kernels")
    # dK and dV come from the same products in the same order on both paths
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
