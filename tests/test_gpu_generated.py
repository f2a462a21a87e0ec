"""Rows generated inside the attention kernel (bsa_attn_fwd_patterns,
bsa_attn_fwd_radial): no column list is written; the producer generates each
row's key blocks from the tile-pattern descriptors or the radial geometry.

They must reproduce bsa_attn_fwd on the lists the builders write, bit for bit
(the same rows in the same order give the same MMAs and the same softmax), and
match the float64 oracle directly on a small case. Covered: ragged sequence
lengths, tokens per frame below, at and above the block, text tokens, the
Wan / Hunyuan-like grids, every tile-pattern family with edge terms (empty and
inverted bands, a half-width covering every residue, repeated and unsorted
stripe columns), and heads sharing patterns through a head -> pattern map.
"""

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close
from workloads import WORKLOADS, generic_tile_patterns, make_qkv, make_random_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _out_lse(q):
    B, H, n, D = q.shape
    return (torch.full_like(q, float("nan")),
            torch.full((B, H, n), float("nan"), dtype=torch.float32, device=q.device))


RADIAL = [  # (frames, tokens_per_frame, text_tokens, heads, head_dim)
    (4, 320, 0, 2, 128),
    (3, 100, 0, 1, 64),       # frames shorter than a block
    (6, 1000, 37, 2, 128),    # ragged frames, a few text tokens
    (2, 128, 300, 1, 128),    # text longer than a block
    (5, 777, 129, 3, 64),
]


@pytest.mark.parametrize("F,S,T,H,D", RADIAL)
def test_radial_generated_equals_lists(bsa, F, S, T, H, D):
    n = F * S + T
    q, k, v = (t.cuda() for t in make_random_qkv(2, H, n, D, seed=F * 31 + S))
    lists = bsa.radial_block_lists(F, S, 128, text_tokens=T)
    ref_o, ref_l = bsa.attention(q, k, v, lists)
    out, lse = _out_lse(q)
    bsa.bsa_attn_fwd_radial(q, k, v, F, S, out, lse, text_tokens=T)
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


@pytest.mark.parametrize("name", ["wan", "hunyuan_text"])
def test_radial_generated_full_grids(bsa, name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, "cuda", heads=4)
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, 128, text_tokens=w.text_tokens)
    ref_o, ref_l = bsa.attention(q, k, v, lists)
    out, lse = _out_lse(q)
    bsa.bsa_attn_fwd_radial(q, k, v, w.frames, w.tokens_per_frame, out, lse,
                            text_tokens=w.text_tokens)
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_radial_generated_against_oracle(bsa):
    F, S, T, H, D = 5, 300, 70, 2, 128
    n = F * S + T
    q, k, v = make_random_qkv(1, H, n, D, seed=3)
    out, lse = _out_lse(q.cuda())
    bsa.bsa_attn_fwd_radial(q.cuda(), k.cuda(), v.cuda(), F, S, out, lse, text_tokens=T)
    assert bsa.bsa_get_device_status() == 0
    rp, ci = oracle.joint_block_lists(F, S, T, 128)
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, 128)
    assert_close(out, ref_o, lse, ref_l, "radial rows generated in the kernel")


PATTERNS = [
    {"bands": [(-8, 8)]},                                          # diagonal window
    {"bands": [(-1, 1), (5, 9), (-30, -26), (100, 104)]},          # multi-diagonal
    {"bands": [(-2, 2)], "columns": [0, 7, 7, 3, 31, 20]},         # stripes, repeated, unsorted
    {"bands": [(-3, 3)], "axial": (8, 1)},                         # dual window
    {"bands": [(4, 2), (0, 0)], "axial": (5, 3)},                  # inverted band, every residue
    {"bands": [(200, 300)]},                                       # outside every row: empty rows
    {"axial": (16, 0), "columns": [1]},
]


def _expanded_lists(bsa, pats, head_pattern, nqb):
    """Per-head CSR lists built by the list builder from the heads' patterns."""
    per_head = [pats[i] for i in head_pattern]
    return bsa.tile_pattern_block_lists(per_head, nqb, 128, device="cuda:0")


@pytest.mark.parametrize("n,D", [(5000, 128), (4097, 64)])
def test_patterns_generated_equal_lists(bsa, n, D):
    H = len(PATTERNS)
    nqb = -(-n // 128)
    q, k, v = (t.cuda() for t in make_random_qkv(1, H, n, D, seed=n))
    lists = _expanded_lists(bsa, PATTERNS, range(H), nqb)
    ref_o, ref_l = bsa.attention(q, k, v, lists)
    raw, cols = bsa.pack_tile_patterns(PATTERNS, "cuda")
    out, lse = _out_lse(q)
    bsa.bsa_attn_fwd_patterns(q, k, v, raw, cols, out, lse)
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_heads_sharing_patterns(bsa):
    # eight heads over three patterns: one set of row lengths and one work
    # order per pattern, each head attending with its pattern's rows
    pats = [PATTERNS[1], PATTERNS[3], PATTERNS[2]]
    head_pattern = [0, 2, 2, 1, 0, 1, 2, 0]
    H, n, D = len(head_pattern), 4000, 128       # 32 query blocks: every stripe column valid
    nqb = -(-n // 128)
    q, k, v = (t.cuda() for t in make_random_qkv(2, H, n, D, seed=11))
    lists = _expanded_lists(bsa, pats, head_pattern, nqb)
    ref_o, ref_l = bsa.attention(q, k, v, lists)
    raw, cols = bsa.pack_tile_patterns(pats, "cuda")
    hp = torch.tensor(head_pattern, dtype=torch.int32, device="cuda")
    out, lse = _out_lse(q)
    bsa.bsa_attn_fwd_patterns(q, k, v, raw, cols, out, lse, head_pattern=hp)
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_generic_workload_generated(bsa):
    w = WORKLOADS["generic"]
    q, k, v = make_qkv(w, "cuda")
    pats = generic_tile_patterns(w.heads, w.nqb)
    lists = bsa.tile_pattern_block_lists(pats, w.nqb, 128, device="cuda:0")
    ref_o, ref_l = bsa.attention(q, k, v, lists)
    raw, cols = bsa.pack_tile_patterns(pats, "cuda")
    out, lse = _out_lse(q)
    bsa.bsa_attn_fwd_patterns(q, k, v, raw, cols, out, lse)
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_patterns_generated_against_oracle(bsa):
    pats = [PATTERNS[0], PATTERNS[3], {"bands": [(-2, 2)], "columns": [0, 7, 7, 3, 11]}]
    H, n, D = 3, 1500, 64
    nqb = -(-n // 128)
    q, k, v = make_random_qkv(1, H, n, D, seed=5)
    raw, cols = bsa.pack_tile_patterns(pats, "cuda")
    out, lse = _out_lse(q.cuda())
    bsa.bsa_attn_fwd_patterns(q.cuda(), k.cuda(), v.cuda(), raw, cols, out, lse)
    assert bsa.bsa_get_device_status() == 0
    rp, ci = oracle.tile_pattern_lists(pats, nqb)
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, H, 128)
    assert_close(out, ref_o, lse, ref_l, "tile-pattern rows generated in the kernel")
