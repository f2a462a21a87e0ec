"""GPU parity of the strided forward (bsa_attn_fwd_strided) and of the module
forward and backward (bsa_attn_module_fwd / _bwd) against the float64 oracles.

Strided views: the kernels read q, k, v through the strides and write out
through its strides, with the same arithmetic as the contiguous entry point,
so the results must be bit-identical to bsa_attn_fwd on contiguous copies.

Module tolerance (derived from the arithmetic; the pages fix no precision):
the projections accumulate in fp32 and round q, k, v to bf16 (relative
2^-9), the attention output carries its own error (relative RMS about 2e-3,
rounded to bf16) and out_proj's output is rounded to bf16 again. Each y entry
sums heads*head_dim such terms with independent rounding, so the relative RMS
error stays near a few 2^-9. Bars: the forward's relative RMS 5e-3 and
max-abs 2e-2, the max-abs taken relative to the oracle's largest |y|. The backward's gradients (dA, dQKV rounded to
bf16 once each, the weight gradients summed over up to a few thousand tokens
in fp32) take the same bars per tensor.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_module_inputs, make_random_qkv, random_block_lists

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
    err = got - ref
    rel_rms = np.sqrt((err ** 2).mean()) / max(np.sqrt((ref ** 2).mean()), 1e-30)
    max_rel = np.abs(err).max() / max(np.abs(ref).max(), 1e-30)
    assert rel_rms <= REL_RMS, f"{what}: relative RMS {rel_rms:.3e}"
    assert max_rel <= MAX_REL, f"{what}: max-abs {max_rel:.3e} of max |ref|"


def _lists(bsa, L, n, blk, seed):
    nqb = -(-n // blk)
    rp, ci = random_block_lists(L * nqb, nqb, 0.5, seed, empty_rows=[L * nqb - 1],
                                force={0: [nqb - 1]})
    return rp, ci, bsa.block_lists_from_csr(rp, ci, L, nqb, blk)


STRIDED_CASES = [
    # (batch, heads, n, D, block, num_lists, seed)
    (1, 3, 1000, 128, 128, 1, 1),    # two-tile kernel, ragged last block
    (2, 2, 700, 64, 64, 1, 2),       # one-tile kernel, batch > 1
    (2, 2, 1000, 128, 128, 2, 3),    # per-head lists, batch > 1
    (1, 2, 385, 64, 128, 1, 4),      # last block holds one row
]


@pytest.mark.parametrize("B,H,n,D,blk,L,seed", STRIDED_CASES)
def test_strided_views_match_contiguous_bit_for_bit(bsa, B, H, n, D, blk, L, seed):
    q, k, v = (t.cuda() for t in make_random_qkv(B, H, n, D, seed))
    _, _, lists = _lists(bsa, L, n, blk, seed + 50)
    ref_out, ref_lse = bsa.attention(q, k, v, lists)
    # the token-major layout of a fused projection: [B, n, 3, H, D]
    buf = torch.stack([t.transpose(1, 2) for t in (q, k, v)], dim=2).contiguous()
    qv, kv, vv = (buf[:, :, i].transpose(1, 2) for i in range(3))
    assert not qv.is_contiguous() and qv.stride(2) == 3 * H * D
    out_tok = torch.full((B, n, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    out, lse = bsa.attention(qv, kv, vv, lists, out=out_tok.transpose(1, 2))
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)
    assert torch.equal(out_tok.transpose(1, 2), ref_out)


MODULE_CASES = [
    # (batch, n, heads, D, block, num_lists, bias, seed)
    (2, 1000, 2, 64, 128, 1, True, 11),
    (1, 640, 3, 128, 64, 3, True, 12),   # block 64, per-head lists
    (1, 129, 1, 128, 128, 1, False, 13),  # no biases, one-row last block
]


@pytest.mark.parametrize("B,n,H,D,blk,L,bias,seed", MODULE_CASES)
def test_module_matches_oracle(bsa, B, n, H, D, blk, L, bias, seed):
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, seed, bias=bias)
    rp, ci, lists = _lists(bsa, L, n, blk, seed + 50)
    dev = [None if t is None else t.cuda() for t in (x, wqkv, bqkv, wo, bo)]
    y = bsa.attention_module(*dev, H, lists)
    assert bsa.bsa_get_device_status() == 0
    ref = oracle.radial_attention_module_fp64(x, wqkv, bqkv, wo, bo, H, rp, ci, L, blk)
    _close(y.float().cpu(), ref, "y")


def test_module_wan_size_sampled_tokens(bsa):
    """Wan-size module (C = 40 x 128, n = 32760, radial lists) on sampled
    tokens. out_proj's columns are zeroed except those of heads 0 and 39, so
    the oracle needs the key / value projections of two heads only."""
    w = WORKLOADS["wan"]
    H, D = w.heads, w.head_dim
    x, wqkv, bqkv, wo, bo = make_module_inputs(1, w.n, H, D, 21)
    keep = torch.zeros(H * D, dtype=torch.bool)
    keep[:D] = True
    keep[(H - 1) * D:] = True
    wo = (wo * keep).contiguous()
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)
    rp, ci = lists.row_ptr.cpu().numpy(), lists.col_idx.cpu().numpy()
    dev = [t.cuda() for t in (x, wqkv, bqkv, wo, bo)]
    y = bsa.attention_module(*dev, H, lists)
    assert bsa.bsa_get_device_status() == 0
    rng = np.random.default_rng(22)
    rows = np.unique(np.r_[0, w.n - 1, w.n - 100, rng.integers(0, w.n, 45)])
    ref = oracle.radial_attention_module_rows(x, wqkv, bqkv, wo, bo, H, rp, ci, 1, w.block, 0,
                                              rows, heads_used=[0, H - 1])
    _close(y[0, rows].float().cpu(), ref, "y rows")


MODULE_BWD_CASES = [
    # (batch, n, heads, D, block, num_lists, bias, seed)
    (2, 1000, 2, 64, 128, 1, True, 31),
    (1, 640, 3, 128, 64, 3, True, 32),    # block 64, per-head lists
    (1, 129, 1, 128, 128, 1, False, 33),  # no biases in the forward
]


def _module_grads(bsa, x, wqkv, bqkv, wo, bo, dy, H, lists):
    dev = [None if t is None else t.cuda() for t in (x, wqkv, bqkv, wo, bo, dy)]
    B, n, C = x.shape
    fws = torch.empty(bsa.bsa_attn_module_workspace_bytes(B, n, H, C // H, lists),
                      dtype=torch.uint8, device="cuda")
    bsa.attention_module(*dev[:5], H, lists, workspace=fws)
    grads = bsa.attention_module_backward(dev[0], dev[1], dev[3], dev[5], H, lists, fws)
    assert bsa.bsa_get_device_status() == 0
    return grads


@pytest.mark.parametrize("B,n,H,D,blk,L,bias,seed", MODULE_BWD_CASES)
def test_module_backward_matches_oracle(bsa, B, n, H, D, blk, L, bias, seed):
    x, wqkv, bqkv, wo, bo = make_module_inputs(B, n, H, D, seed, bias=bias)
    dy, _, _, _, _ = make_module_inputs(B, n, H, D, seed + 1, bias=False)
    rp, ci, lists = _lists(bsa, L, n, blk, seed + 50)
    got = _module_grads(bsa, x, wqkv, bqkv, wo, bo, dy, H, lists)
    ref = oracle.radial_attention_module_backward_fp64(x, wqkv, bqkv, wo, bo, dy, H, rp, ci, L,
                                                       blk)
    for name, g, r in zip(("dx", "dw_qkv", "db_qkv", "dw_out", "db_out"), got, ref):
        _close(g.float().cpu(), r, name)


def test_module_backward_wan_width(bsa):
    """Wan width (C = 40 x 128 = 5120) on a 4 x 256 token radial grid (block
    128): every gradient whole against the oracle; the backward is
    bit-reproducible."""
    H, D, F, S, blk = 40, 128, 4, 256, 128
    n = F * S
    x, wqkv, bqkv, wo, bo = make_module_inputs(1, n, H, D, 41)
    dy, _, _, _, _ = make_module_inputs(1, n, H, D, 42, bias=False)
    lists = bsa.radial_block_lists(F, S, blk)
    rp, ci = oracle.radial_block_lists(F, S, blk)
    got = _module_grads(bsa, x, wqkv, bqkv, wo, bo, dy, H, lists)
    again = _module_grads(bsa, x, wqkv, bqkv, wo, bo, dy, H, lists)
    for a, b in zip(got, again):
        assert torch.equal(a, b)
    ref = oracle.radial_attention_module_backward_fp64(x, wqkv, bqkv, wo, bo, dy, H, rp, ci, 1,
                                                       blk)
    for name, g, r in zip(("dx", "dw_qkv", "db_qkv", "dw_out", "db_out"), got, ref):
        _close(g.float().cpu(), r, name)
