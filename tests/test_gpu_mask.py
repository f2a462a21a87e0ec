"""GPU radial mask builder: block lists bit-exact against the CPU oracle."""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TINY_GRIDS = [(1, 64, 64), (2, 64, 64), (3, 96, 64), (5, 255, 64), (8, 256, 64), (17, 16, 64),
              (6, 48, 128), (9, 100, 128), (12, 64, 64), (4, 256, 64), (31, 64, 64),
              (64, 32, 64), (7, 255, 128), (33, 130, 128), (40, 1, 64), (1, 4000, 128)]
RADIAL_CONFIGS = [(4, 256, 64), (21, 1560, 128), (33, 3600, 128), (84, 1560, 128)]


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


@pytest.mark.parametrize("F,S,B", TINY_GRIDS + RADIAL_CONFIGS)
def test_lists_bit_exact(bsa, F, S, B):
    lists = bsa.radial_block_lists(F, S, B, device="cuda:0")
    rp, ci = oracle.radial_block_lists(F, S, B)
    assert np.array_equal(lists.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(lists.col_idx.cpu().numpy(), ci)
    assert bsa.bsa_get_device_status() == 0
    assert bsa.bsa_validate_lists(lists) == 0


def test_async_build_into_preallocated(bsa):
    F, S, B = 21, 1560, 128
    rp, ci = oracle.radial_block_lists(F, S, B)
    nqb = rp.size - 1
    row_ptr = torch.full((nqb + 1,), -7, dtype=torch.int32, device="cuda")
    col_idx = torch.full((ci.size + 100,), -7, dtype=torch.int32, device="cuda")
    got = bsa.bsa_radial_mask_build(F, S, B, row_ptr, col_idx, col_idx.numel(), want_nnz=False)
    assert got is None
    assert bsa.bsa_get_device_status() == 0
    assert np.array_equal(row_ptr.cpu().numpy(), rp)
    assert np.array_equal(col_idx[:ci.size].cpu().numpy(), ci)
    assert (col_idx[ci.size:] == -7).all()


def test_count_only(bsa):
    F, S, B = 33, 3600, 128
    rp, _ = oracle.radial_block_lists(F, S, B)
    row_ptr = torch.empty(rp.size, dtype=torch.int32, device="cuda")
    nnz = bsa.bsa_radial_mask_build(F, S, B, row_ptr)
    assert nnz == int(rp[-1])
    assert np.array_equal(row_ptr.cpu().numpy(), rp)


def test_capacity_too_small(bsa):
    F, S, B = 8, 256, 64
    rp, ci = oracle.radial_block_lists(F, S, B)
    row_ptr = torch.empty(rp.size, dtype=torch.int32, device="cuda")
    col_idx = torch.full((ci.size - 5,), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_radial_mask_build(F, S, B, row_ptr, col_idx, col_idx.numel())
    assert e.value.status == 6
    assert (col_idx == -1).all()          # nothing was written
    # asynchronous form: the fill stops at the capacity and the status word reports it
    bsa.bsa_radial_mask_build(F, S, B, row_ptr, col_idx, col_idx.numel(), want_nnz=False)
    assert bsa.bsa_get_device_status() == 6
    assert bsa.bsa_get_device_status() == 0
    assert np.array_equal(col_idx.cpu().numpy(), ci[:col_idx.numel()])


JOINT = [(4, 64, 16, 64), (3, 40, 21, 64), (5, 48, 7, 128), (2, 100, 130, 64), (6, 33, 1, 64),
         (4, 256, 77, 64), (33, 3600, 256, 128), (21, 1560, 512, 128), (8, 256, 0, 64)]


@pytest.mark.parametrize("F,S,T,B", JOINT)
def test_joint_text_video_lists_bit_exact(bsa, F, S, T, B):
    lists = bsa.radial_block_lists(F, S, B, device="cuda:0", text_tokens=T)
    rp, ci = oracle.joint_block_lists(F, S, T, B)
    assert np.array_equal(lists.row_ptr.cpu().numpy(), rp)
    assert np.array_equal(lists.col_idx.cpu().numpy(), ci)
    assert bsa.bsa_get_device_status() == 0
    assert bsa.bsa_validate_lists(lists) == 0
