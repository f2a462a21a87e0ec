"""Error paths on the GPU: list validation, and a device-side wait that runs out.

The timeout test leaves one K-tile load un-issued (a test hook) so that the
MMA issuer's bounded wait on that tile expires. The kernel then records
BSA_ERR_DEVICE_TIMEOUT, every role leaves its loop, copies in flight are
drained, tensor memory is freed, and the context stays usable: the next call
succeeds. Nothing here traps, faults or hangs the GPU.
"""

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close
from workloads import make_random_qkv, random_block_lists

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _lists(bsa, rp, ci, nqb, blk=64, L=1):
    return bsa.block_lists_from_csr(rp, ci, L, nqb, blk)


def test_validate_lists_detects_malformed(bsa):
    nqb = 8
    rp, ci = random_block_lists(nqb, nqb, 0.5, seed=3, force={0: [1, 2, 5]})
    assert bsa.bsa_validate_lists(_lists(bsa, rp, ci, nqb)) == 0
    bad = ci.copy()
    bad[1], bad[2] = bad[2], bad[1]           # unsorted row 0
    assert bsa.bsa_validate_lists(_lists(bsa, rp, bad, nqb)) == 5
    bad = ci.copy()
    bad[0] = nqb                               # out of range
    assert bsa.bsa_validate_lists(_lists(bsa, rp, bad, nqb)) == 5
    badrp = rp.copy()
    badrp[3] = badrp[4] + 1                    # not monotone
    assert bsa.bsa_validate_lists(_lists(bsa, badrp, ci, nqb)) == 5
    assert bsa.bsa_get_device_status() == 0    # validation leaves the status word alone


def test_malformed_lists_never_read_out_of_bounds(bsa):
    """Entries out of range are clamped by the kernels: wrong values, no fault."""
    n, D, blk = 512, 64, 64
    nqb = n // blk
    q, k, v = (t.cuda() for t in make_random_qkv(1, 1, n, D, seed=5))
    rp = np.arange(nqb + 1, dtype=np.int32)
    ci = np.full(nqb, 10 ** 6, dtype=np.int32)
    lists = _lists(bsa, rp, ci, nqb, blk)
    out, lse = bsa.attention(q, k, v, lists)
    ref_o, _ = bsa.dense_masked_reference(q, k, v, lists)
    assert bsa.bsa_get_device_status() == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(ref_o.float()).all()


def test_device_wait_timeout_is_reported_and_recoverable(bsa):
    n, D, blk = 2048, 128, 128
    nqb = n // blk
    q, k, v = (t.cuda() for t in make_random_qkv(1, 2, n, D, seed=9))
    rp, ci = random_block_lists(nqb, nqb, 0.5, seed=10, force={0: [0, 3]})
    lists = _lists(bsa, rp, ci, nqb, blk)
    assert bsa.bsa_get_device_status() == 0
    bsa.bsa_set_test_hooks(wait_limit_ns=50_000_000, fault_flags=1)
    try:
        bsa.attention(q, k, v, lists)
        assert bsa.bsa_get_device_status() == 4
        role, bar, counter, cta = bsa.bsa_get_timeout_detail()
        assert role in (1, 2, 3) and bar >= 1
    finally:
        bsa.bsa_set_test_hooks(0, 0)
    # the context is still usable and the next launch is correct
    out, lse = bsa.attention(q, k, v, lists)
    assert bsa.bsa_get_device_status() == 0
    ref_o, ref_l = oracle.masked_attention_fp64(q, k, v, rp, ci, 1, blk)
    assert_close(out, ref_o, lse, ref_l, "after timeout")
