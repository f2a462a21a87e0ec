"""The allocation-free entry point against the regular one.

bsa_attn_fwd_noalloc serves callers that cannot allocate device memory (for
example a plugin that its host framework hands only input and output buffers,
or a runtime whose memory plan is fixed at start-up), so they cannot pass the
workspace bsa_attn_fwd needs. Its scratch is a fixed array inside the library,
shared by every call. These tests call it through the C ABI on several
problems in a row, so later calls reuse the array earlier ones filled, and
compare each result with bsa_attn_fwd on the same inputs. Both entries run the
same kernels on the same lists in the same order, so the results must be
bit-identical (at block 64 the allocation-free entry runs the one-tile kernel,
and the reference is taken on that kernel too). The file is collected last so that a run stopping at the first
failure has already run everything else; it also passes alone in a fresh
process.
"""

import ctypes

import pytest
import torch

from workloads import WORKLOADS, make_generic_lists, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _problem_radial(bsa):
    w = WORKLOADS["wan"]
    q, k, v = make_qkv(w, "cuda", heads=6)
    return q, k, v, bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block)


def _problem_per_head(bsa):
    w = WORKLOADS["generic"]
    q, k, v = make_qkv(w, "cuda", heads=8)
    rp, ci, _ = make_generic_lists(8, w.nqb)
    return q, k, v, bsa.block_lists_from_csr(rp, ci, 8, w.nqb, w.block)


def _band_lists(bsa, nqb, block):
    """Each query block lists itself and the block before it (one list)."""
    qb = torch.arange(nqb, dtype=torch.int64, device="cuda")
    counts = torch.where(qb == 0, 1, 2)
    rp = torch.zeros(nqb + 1, dtype=torch.int64, device="cuda")
    rp[1:] = torch.cumsum(counts, 0)
    ci = torch.empty(int(rp[-1].item()), dtype=torch.int64, device="cuda")
    ci[rp[1:] - 1] = qb                                  # the diagonal, last in each row
    ci[rp[2:] - 2] = qb[1:] - 1                          # the block before it
    return bsa.block_lists_from_csr(rp, ci, 1, nqb, block)


def _long_sequence(bsa, nqb, block=64, d=64, seed=11):
    n = nqb * block
    g = torch.Generator(device="cuda").manual_seed(seed)
    q, k, v = (torch.randn((1, 1, n, d), generator=g, device="cuda").to(torch.bfloat16)
               for _ in range(3))
    return q, k, v, _band_lists(bsa, nqb, block)


def _run_noalloc(bsa, q, k, v, lists):
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
    bsa.bsa_attn_fwd_noalloc(q, k, v, lists, out, lse)
    return out, lse


def _assert_identical(got, ref, what):
    (out, lse), (ref_o, ref_l) = got, ref
    assert torch.equal(out, ref_o), f"{what}: outputs differ"
    assert torch.equal(lse, ref_l), f"{what}: lse differs"


def test_noalloc_matches_workspace_entry_two_calls(bsa):
    problems = [_problem_per_head(bsa), _problem_radial(bsa)]
    refs = [bsa.attention(q, k, v, lists) for q, k, v, lists in problems]
    results = [_run_noalloc(bsa, *p) for p in problems]   # two calls in a row, one scratch array
    assert bsa.bsa_get_device_status() == 0
    for got, ref, name in zip(results, refs, ("per-head lists", "radial")):
        _assert_identical(got, ref, f"noalloc vs workspace entry ({name})")


def test_noalloc_at_the_scratch_limit(bsa):
    # Block 64 runs the one-tile kernel, whose work order takes one entry per
    # query block per list: a single list of exactly the maximum number of
    # query blocks fills the whole array, and the work counter sits after it.
    nqb = bsa.NOALLOC_MAX_ORDER_ENTRIES
    q, k, v, lists = _long_sequence(bsa, nqb)
    # the workspace entry packs block-64 problems into 128-row tiles on the
    # two-tile kernel; the allocation-free entry has no room for those tile
    # lists and runs the one-tile kernel, so the reference takes that kernel
    # too (test hook bit 1) and the results must again be identical
    try:
        bsa.bsa_set_test_hooks(0, 2)
        ref = bsa.attention(q, k, v, lists)
    finally:
        bsa.bsa_set_test_hooks(0, 0)
    got = _run_noalloc(bsa, q, k, v, lists)
    assert bsa.bsa_get_device_status() == 0
    _assert_identical(got, ref, "noalloc at the limit (block 64, one list)")
    # a block-128 call right after it reuses the filled array (two-tile kernel)
    p = _problem_radial(bsa)
    _assert_identical(_run_noalloc(bsa, *p), bsa.attention(*p), "noalloc after the limit case")
    assert bsa.bsa_get_device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch(bsa):
    from block_sparse_attention_radial_b200 import _lib

    # one query block more than the array holds, on real device buffers: the
    # call must refuse it on the host (status 7) and leave out untouched
    nqb = bsa.NOALLOC_MAX_ORDER_ENTRIES + 1
    q, k, v, lists = _long_sequence(bsa, nqb, seed=12)
    out = torch.zeros_like(q)
    ls = lists.c_struct()
    lib = _lib.load()
    B, H, n, D = q.shape
    st = lib.bsa_attn_fwd_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                  ctypes.c_void_p(v.data_ptr()), B, H, n, D, 0.0,
                                  ctypes.byref(ls), ctypes.c_void_p(out.data_ptr()), None, None)
    assert st == 7
    assert "scratch" in bsa.bsa_status_string(st)
    torch.cuda.synchronize()
    assert bsa.bsa_get_device_status() == 0
    assert not out.any()
