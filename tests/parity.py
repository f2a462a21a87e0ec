"""Comparison helpers shared by the GPU parity tests (test code only)."""

from __future__ import annotations

import numpy as np

# Tolerances for bf16 outputs against the float64 oracle.
MAX_ABS = 2e-2
REL_RMS = 5e-3
LSE_ABS = 1e-3


def to64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(out, ref_out, lse=None, ref_lse=None):
    o = out if isinstance(out, np.ndarray) else to64(out)
    d = o - ref_out
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    denom = float((ref_out ** 2).mean()) if ref_out.size else 0.0
    rel_rms = float(np.sqrt((d ** 2).mean() / denom)) if denom > 0 else float(np.sqrt((d ** 2).mean()))
    lse_abs = 0.0
    if lse is not None:
        l = lse if isinstance(lse, np.ndarray) else to64(lse)
        both_inf = np.isneginf(l) & np.isneginf(ref_lse)
        assert np.array_equal(np.isneginf(l), np.isneginf(ref_lse)), "empty-row pattern differs"
        dl = np.where(both_inf, 0.0, l - np.where(both_inf, 0.0, ref_lse))
        lse_abs = float(np.abs(dl).max()) if dl.size else 0.0
    return max_abs, rel_rms, lse_abs


def assert_close(out, ref_out, lse=None, ref_lse=None, what=""):
    max_abs, rel_rms, lse_abs = errors(out, ref_out, lse, ref_lse)
    assert max_abs <= MAX_ABS, f"{what}: max_abs {max_abs:.3e}"
    assert rel_rms <= REL_RMS, f"{what}: rel_rms {rel_rms:.3e}"
    assert lse_abs <= LSE_ABS, f"{what}: lse_abs {lse_abs:.3e}"
    return max_abs, rel_rms, lse_abs


def assert_close_device(out, ref_out, lse=None, ref_lse=None, what=""):
    """Same tolerances, with the statistics computed on the device (large tensors)."""
    import torch

    d = out.double() - ref_out.double()
    max_abs = d.abs().max().item()
    rel_rms = (d.square().mean() / ref_out.double().square().mean()).sqrt().item()
    lse_abs = 0.0
    if lse is not None:
        a, b = lse.double(), ref_lse.double()
        assert torch.equal(torch.isneginf(a), torch.isneginf(b)), "empty-row pattern differs"
        fin = torch.isfinite(b)
        lse_abs = (a[fin] - b[fin]).abs().max().item() if fin.any() else 0.0
    assert max_abs <= MAX_ABS, f"{what}: max_abs {max_abs:.3e}"
    assert rel_rms <= REL_RMS, f"{what}: rel_rms {rel_rms:.3e}"
    assert lse_abs <= LSE_ABS, f"{what}: lse_abs {lse_abs:.3e}"
    return max_abs, rel_rms, lse_abs
