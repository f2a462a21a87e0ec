"""GPU parity of the library's tcgen05 GEMM (bsa_gemm_bf16), the matrix
product behind the module's q/k/v and out projections and their gradients.

Reference: the float64 product of the same bf16 operands (numpy matmul).
Error bound per element, derived from the arithmetic: the kernel accumulates
in fp32 and rounds the result to bf16 once, so
|got - ref| <= 2^-8 |ref| + 2^-16 sum_k |a_ik b_kj|
(the first term covers the bf16 rounding, half an ulp = 2^-9 relative, with
a factor two of margin; the second bounds fp32 accumulation error for the k
values used here, k * 2^-24 <= 2^-16 up to k = 256, and the block-wise
summation keeps it far smaller for longer k).
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_radial_b200 as m

    torch.cuda.set_device(0)
    return m


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _ref(a, b, a_mn, b_mn, bias):
    A = a.double().numpy()
    B = b.double().numpy()
    A = A.T if a_mn else A            # [m, k]
    B = B if b_mn else B.T            # [k, n]
    ref = A @ B
    mag = np.abs(A) @ np.abs(B)
    if bias is not None:
        ref = ref + bias.double().numpy()[None, :]
        mag = mag + np.abs(bias.double().numpy())[None, :]
    return ref, mag


def _check(got, ref, mag, what):
    g = got.double().cpu().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * mag + 1e-30
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{what}: error {worst:.2f} x the bound"


def _padded(rows, cols, seed):
    """[rows, cols] bf16 view of a wider array whose row stride is a multiple
    of 8 elements (the entry's alignment rule); the padding is never read."""
    wide = _rand((rows, -(-cols // 8) * 8), seed)
    return wide[:, :cols]


def _operands(m, n, k, a_mn, b_mn, seed):
    a = _padded(k, m, seed) if a_mn else _padded(m, k, seed)
    b = _padded(k, n, seed + 1) if b_mn else _padded(n, k, seed + 1)
    return a, b


def _dev(t):
    """Device copy keeping the row stride (contiguous last axis)."""
    base = t.as_strided((t.shape[0], t.stride(0)), (t.stride(0), 1))
    return base.cuda()[:, :t.shape[1]]


SHAPES = [
    (128, 256, 64),      # exactly one tile and one K block
    (300, 264, 200),     # ragged rows, columns and K
    (1, 8, 1),           # smallest
    (777, 520, 1000),    # several tiles both ways, K not a multiple of 64
    (129, 512, 130),     # one row past a tile, two column tiles
]


@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (False, True), (True, False), (True, True)])
@pytest.mark.parametrize("m,n,k", SHAPES)
def test_gemm_against_float64(bsa, m, n, k, a_mn, b_mn):
    a, b = _operands(m, n, k, a_mn, b_mn, seed=m + 7 * n + 13 * k)
    bias = _rand((n,), seed=k, scale=0.5) if (m + n) % 2 == 0 else None
    out = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
    bsa.bsa_gemm_bf16(_dev(a), _dev(b), out, None if bias is None else bias.cuda(), a_mn, b_mn)
    assert bsa.bsa_get_device_status() == 0
    ref, mag = _ref(a, b, a_mn, b_mn, bias)
    _check(out, ref, mag, f"gemm m={m} n={n} k={k} a_mn={a_mn} b_mn={b_mn}")


def test_gemm_strided_operands_and_output(bsa):
    m, n, k = 200, 136, 96
    A = _rand((m, k + 40), 1).cuda()          # row stride k + 40
    B = _rand((k, n + 24), 2).cuda()          # B stored [k][n], row stride n + 24
    out = torch.full((m, n + 16), float("nan"), dtype=torch.bfloat16, device="cuda")
    a, b, o = A[:, :k], B[:, :n], out[:, :n]
    bsa.bsa_gemm_bf16(a, b, o, None, False, True)
    assert bsa.bsa_get_device_status() == 0
    ref, mag = _ref(a.cpu(), b.cpu(), False, True, None)
    _check(o, ref, mag, "strided gemm")
    assert torch.isnan(out[:, n:].float()).all(), "columns past n were written"


def test_gemm_is_deterministic(bsa):
    m, n, k = 1000, 768, 2048
    a, b = _operands(m, n, k, True, True, seed=5)
    a, b = _dev(a), _dev(b)
    outs = []
    for _ in range(2):
        out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        bsa.bsa_gemm_bf16(a, b, out, None, True, True)
        outs.append(out)
    assert torch.equal(outs[0], outs[1])


def test_gemm_wan_width_sampled(bsa):
    # the q/k/v projection's shape at the Wan width (C = 40 x 128), fewer rows
    m, C = 2048, 5120
    x = _rand((m, C), 11)
    w = _rand((3 * C, C), 12, scale=C ** -0.5)
    bias = _rand((3 * C,), 13, scale=0.1)
    out = torch.empty((m, 3 * C), dtype=torch.bfloat16, device="cuda")
    bsa.bsa_gemm_bf16(x.cuda(), w.cuda(), out, bias.cuda(), False, False)
    assert bsa.bsa_get_device_status() == 0
    rows = np.r_[0:3, 127:130, 1000:1003, m - 3:m]
    xs = x[rows].double().numpy()
    W = w.double().numpy()
    ref = xs @ W.T + bias.double().numpy()[None, :]
    mag = np.abs(xs) @ np.abs(W).T + np.abs(bias.double().numpy())[None, :]
    got = out[torch.as_tensor(rows, device="cuda")]
    _check(got, ref, mag, "wan-width projection (sampled rows)")
