"""The softmax's two exponential paths against CUDA's exp2f.

Of every eight column pairs, some take 2^x from a degree-3 polynomial on the
FMA pipe (range reduction to [-1/2, 1/2], Remez-fitted coefficients) instead of
the MUFU unit. Its relative error must stay far below the bf16 rounding of P
(2^-9), and it must never produce a non-finite or wrapped value for the
arguments the kernel can see (x <= 8 after the lazy max, anything below).
"""

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_polynomial_exp2_error_bound():
    import block_sparse_attention_radial_b200 as bsa

    torch.cuda.set_device(0)
    x = torch.cat([torch.linspace(-124.0, 9.0, 2_000_000), torch.tensor([0.0, 0.5, -0.5, 1e-7])])
    x = x[: x.numel() // 2 * 2].cuda()
    poly, mufu, ref = bsa.bsa_selftest_exp2(x)
    rel = ((poly.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel < 1.0e-4, rel
    rel_mufu = ((mufu.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel_mufu < 1.0e-5, rel_mufu
    # far below the range: tiny, finite, never wrapped into a large value
    lo = torch.tensor([-125.0, -126.0, -200.0, -1e30, float("-inf"), -130.5], device="cuda")
    p, _, _ = bsa.bsa_selftest_exp2(lo)
    assert torch.isfinite(p).all() and (p >= 0).all() and (p < 1e-37).all()
