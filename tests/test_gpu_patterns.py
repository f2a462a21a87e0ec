"""GPU tile-pattern list builder: lists bit-exact against the CPU oracle.

Families (diagonal window, multi-diagonal bands, vertical stripes, dual
window), their unions, edge terms (bands outside the row, inverted bands,
offsets near the int32 limits, a period of 1, a half-width covering every
residue, repeated and unsorted columns, empty patterns), row counts that are
not a multiple of 32, the seeded generic workload (its lists and its
attention output, against the host-built lists), capacity errors and
malformed patterns reported through the device status.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, generic_tile_patterns, make_generic_lists, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _random_patterns(count, nqb, seed):
    rng = np.random.default_rng(seed)
    pats = []
    for _ in range(count):
        p = {"bands": [], "axial": None, "columns": []}
        for _ in range(int(rng.integers(0, 17))):
            o = int(rng.integers(-nqb - 4, nqb + 4))
            h = int(rng.integers(-2, 9))          # h < 0 gives an inverted, empty band
            p["bands"].append((o - h, o + h))
        if rng.random() < 0.5:
            P = int(rng.integers(1, 40))
            p["axial"] = (P, int(rng.integers(0, 6)))
        if rng.random() < 0.5:
            p["columns"] = rng.integers(0, nqb, size=int(rng.integers(0, 40))).tolist()
        pats.append(p)
    return pats


def _check(bsa, patterns, nqb):
    lists = bsa.tile_pattern_block_lists(patterns, nqb, 128, device="cuda:0")
    rp, ci = oracle.tile_pattern_lists(patterns, nqb)
    assert bsa.bsa_get_device_status() == 0
    assert np.array_equal(lists.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(lists.col_idx.cpu().numpy(), ci)
    return lists


FAMILIES = [
    {"bands": [(-8, 8)]},                                          # diagonal window
    {"bands": [(-1, 1), (5, 9), (-30, -26), (100, 104)]},          # multi-diagonal
    {"bands": [(-2, 2)], "columns": [0, 7, 7, 3, 63, 200, 31]},    # stripes + diagonal
    {"bands": [(-3, 4)], "axial": (16, 1)},                        # dual window
    {"axial": (8, 0)},
    {"axial": (1, 0)},                                             # every tile
    {"axial": (7, 3)},                                             # every residue
    {"bands": [(5, 2)]},                                           # inverted: empty
    {"bands": [(-(1 << 31) + 1, -(1 << 30)), ((1 << 30), (1 << 31) - 1)]},  # outside
    {"bands": [(-(1 << 31), (1 << 31) - 1)]},                      # every tile
    {},                                                            # empty
    {"columns": [5]},
]


@pytest.mark.parametrize("nqb", [1, 7, 31, 32, 33, 256, 1025])
def test_families_bit_exact(bsa, nqb):
    pats = [dict(p, columns=[c for c in p.get("columns", []) if c < nqb]) for p in FAMILIES]
    _check(bsa, pats, nqb)


@pytest.mark.parametrize("count,nqb,seed", [(3, 50, 0), (24, 256, 1), (40, 1024, 2), (5, 4099, 3)])
def test_random_patterns_bit_exact(bsa, count, nqb, seed):
    lists = _check(bsa, _random_patterns(count, nqb, seed), nqb)
    if lists.nnz:
        assert bsa.bsa_validate_lists(lists) == 0


def test_generic_workload_lists_and_attention(bsa):
    w = WORKLOADS["generic"]
    rp, ci, _ = make_generic_lists(w.heads, w.nqb)
    built = _check(bsa, generic_tile_patterns(w.heads, w.nqb), w.nqb)
    assert np.array_equal(built.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(built.col_idx.cpu().numpy(), ci)
    q, k, v = make_qkv(w, "cuda")
    host = bsa.block_lists_from_csr(rp, ci, w.heads, w.nqb, w.block)
    o1, l1 = bsa.attention(q, k, v, built)
    o2, l2 = bsa.attention(q, k, v, host)
    assert bsa.bsa_get_device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_async_build_and_capacity(bsa):
    pats = _random_patterns(6, 300, 7)
    rp, ci = oracle.tile_pattern_lists(pats, 300)
    raw, cols = bsa.pack_tile_patterns(pats)
    row_ptr = torch.full((rp.size,), -7, dtype=torch.int32, device="cuda")
    col_idx = torch.full((ci.size + 50,), -7, dtype=torch.int32, device="cuda")
    assert bsa.bsa_tile_pattern_lists_build(6, 300, raw, cols, row_ptr, col_idx, col_idx.numel(),
                                            want_nnz=False) is None
    assert bsa.bsa_get_device_status() == 0
    assert np.array_equal(row_ptr.cpu().numpy(), rp)
    assert np.array_equal(col_idx[:ci.size].cpu().numpy(), ci)
    assert (col_idx[ci.size:] == -7).all()
    # too small: with nnz requested the call fails on the host and writes nothing
    small = torch.full((ci.size - 1,), -7, dtype=torch.int32, device="cuda")
    with pytest.raises(bsa.BsaError, match="CAPACITY"):
        bsa.bsa_tile_pattern_lists_build(6, 300, raw, cols, row_ptr, small, small.numel())
    assert (small == -7).all()
    # without it the kernel stops at the capacity and records the overflow
    bsa.bsa_tile_pattern_lists_build(6, 300, raw, cols, row_ptr, small, small.numel(),
                                     want_nnz=False)
    assert bsa.bsa_get_device_status() == 6
    assert np.array_equal(small.cpu().numpy(), ci[:ci.size - 1])


def test_malformed_patterns_reported(bsa):
    nqb = 40
    good = {"bands": [(-1, 1)]}
    pats = [good, {"bands": [(0, 0)] * 3}, good]
    raw, _ = bsa.pack_tile_patterns(pats)
    words = raw.view(torch.int32).view(3, -1)
    words[1, 0] = 17                               # num_bands beyond the maximum
    row_ptr = torch.empty(3 * nqb + 1, dtype=torch.int32, device="cuda")
    bsa.bsa_tile_pattern_lists_build(3, nqb, raw, None, row_ptr)
    assert bsa.bsa_get_device_status() == 1
    counts = np.diff(row_ptr.cpu().numpy())
    expect = np.diff(oracle.tile_pattern_lists([good], nqb)[0])
    assert np.array_equal(counts[:nqb], expect) and np.array_equal(counts[2 * nqb:], expect)
    assert (counts[nqb:2 * nqb] == 0).all()
    # a stripe column out of range is left out and reported
    raw, cols = bsa.pack_tile_patterns([{"columns": [3, 9]}])
    cols[1] = nqb + 5
    bsa.bsa_tile_pattern_lists_build(1, nqb, raw, cols, row_ptr[:nqb + 1])
    assert bsa.bsa_get_device_status() == 1
    assert (torch.diff(row_ptr[:nqb + 1]) == 1).all()
