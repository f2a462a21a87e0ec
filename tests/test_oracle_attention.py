"""Pins for the oracle's masked attention (CPU only).

The oracle is tied to library routines and closed forms it does not use
itself: torch's scaled_dot_product_attention in float64 (with and without a
boolean mask built here by a separate loop), scipy's logsumexp, a row with a
single admissible key (returns that key's value exactly), and permutation
invariance inside the admitted set.
"""

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from workloads import make_random_qkv, random_block_lists


def _dense_lists(nqb, nkb):
    row_ptr = np.arange(nqb + 1, dtype=np.int32) * nkb
    col_idx = np.tile(np.arange(nkb, dtype=np.int32), nqb)
    return row_ptr, col_idx


def _sdpa64(q, k, v, mask=None, scale=None):
    t = lambda x: torch.as_tensor(np.asarray(x, dtype=np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else torch.as_tensor(mask),
        scale=scale).numpy()


def _mask_by_loop(row_ptr, col_idx, nqb, n, block, num_lists, H):
    """[H, n, n] bool mask written out element by element from the lists."""
    m = np.zeros((H, n, n), dtype=bool)
    for h in range(H):
        base = (h if num_lists > 1 else 0) * nqb
        for i in range(n):
            r = base + i // block
            for kb in col_idx[row_ptr[r]:row_ptr[r + 1]]:
                for j in range(kb * block, (kb + 1) * block):
                    if j < n:
                        m[h, i, j] = True
    return m


@pytest.mark.parametrize("n,block,D", [(200, 64, 64), (256, 64, 128), (130, 128, 64), (1, 64, 64)])
def test_all_ones_lists_equal_dense_attention(n, block, D):
    q, k, v = (x.double().numpy() for x in make_random_qkv(2, 3, n, D, seed=11))
    nqb = -(-n // block)
    rp, ci = _dense_lists(nqb, nqb)
    out, lse = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, block)
    ref = _sdpa64(q, k, v)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    s = np.einsum("bhid,bhjd->bhij", q, k) * D ** -0.5
    assert np.allclose(lse, logsumexp(s, axis=-1), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("num_lists", [1, 3])
def test_block_lists_equal_masked_sdpa(num_lists):
    n, block, D, H = 150, 32, 64, 3
    q, k, v = (x.double().numpy() for x in make_random_qkv(1, H, n, D, seed=5))
    nqb = -(-n // block)
    rp, ci = random_block_lists(num_lists * nqb, nqb, 0.45, seed=7,
                                force={0: [0], 1: [nqb - 1]})
    scale = 0.37
    out, lse = oracle.masked_attention_fp64(q, k, v, rp, ci, num_lists, block, scale=scale)
    m = _mask_by_loop(rp, ci, nqb, n, block, num_lists, H)
    ref = _sdpa64(q, k, v, mask=m[None], scale=scale)
    live = m.any(axis=-1)[None]
    assert np.allclose(out[live], ref[live], rtol=1e-12, atol=1e-12)
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    s = np.where(m[None], s, -np.inf)
    assert np.allclose(lse[live], logsumexp(s, axis=-1)[live], rtol=1e-12, atol=1e-12)


def test_single_admissible_key_returns_its_value():
    # n = 65 with block 64: key block 1 holds exactly one valid key (token 64).
    n, block, D = 65, 64, 64
    q, k, v = (x.double().numpy() for x in make_random_qkv(1, 1, n, D, seed=3, scale=3.0))
    rp = np.array([0, 1, 2], dtype=np.int32)
    ci = np.array([1, 1], dtype=np.int32)
    out, lse = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, block)
    assert np.array_equal(out[0, 0], np.broadcast_to(v[0, 0, 64], (n, D)))
    s = q[0, 0] @ k[0, 0, 64] * D ** -0.5
    assert np.allclose(lse[0, 0], s, rtol=0, atol=1e-12)


def test_permuting_admitted_keys_leaves_output_unchanged():
    n, block, D = 256, 64, 64
    q, k, v = (x.double().numpy() for x in make_random_qkv(1, 1, n, D, seed=9))
    rp = np.array([0, 2, 3, 5, 6], dtype=np.int32)
    ci = np.array([0, 2, 1, 0, 3, 2], dtype=np.int32)
    out, lse = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, block)
    # swap keys (with their values) inside block 2, which every row listing it admits as a whole
    perm = np.arange(n)
    rng = np.random.default_rng(0)
    perm[128:192] = 128 + rng.permutation(64)
    out2, lse2 = oracle.masked_attention_fp64(q, k[:, :, perm], v[:, :, perm], rp, ci, 1, block)
    assert np.allclose(out, out2, rtol=1e-12, atol=1e-13)
    assert np.allclose(lse, lse2, rtol=1e-12, atol=1e-13)


def test_empty_row_gives_zero_and_minus_inf():
    n, block, D = 128, 64, 64
    q, k, v = (x.double().numpy() for x in make_random_qkv(1, 1, n, D, seed=1))
    rp = np.array([0, 0, 1], dtype=np.int32)
    ci = np.array([0], dtype=np.int32)
    out, lse = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, block)
    assert np.all(out[0, 0, :64] == 0) and np.all(np.isneginf(lse[0, 0, :64]))
    assert np.all(np.isfinite(lse[0, 0, 64:]))


def test_rows_subset_matches_full():
    n, block, D = 300, 64, 64
    q, k, v = (x.double().numpy() for x in make_random_qkv(1, 2, n, D, seed=2))
    nqb = -(-n // block)
    rp, ci = random_block_lists(nqb, nqb, 0.5, seed=4, force={0: [4]})
    full_o, full_l = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, block)
    rows = np.array([0, 5, 63, 64, 299])
    o, l = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, block, rows=rows, heads=[1])
    assert np.array_equal(o[0, 0], full_o[0, 1, rows]) and np.array_equal(l[0, 0], full_l[0, 1, rows])


def test_bf16_round_matches_torch():
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32) * 7
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.bf16_round(x), ref)
