"""Seeded synthetic workloads shared by the tests, the bench and the smoke run.

This module only draws random inputs and tile patterns. It holds none of the
attention or radial-mask arithmetic, so both the CUDA path and the CPU oracle
can take their inputs from here without sharing any of the method's code.

The shapes stand in for the video-DiT workloads the pages measure on
(Wan2.1-14B, HunyuanVideo; no model weights or latents are used):

* ``tiny``     1x1 heads, D=64, 4 frames x 256 tokens, block 64, fp32 N(0,1)
               drawn on the CPU (seed 0) and rounded to bf16.
* ``wan``      1x40 heads, D=128, 21 x 1560 tokens (n=32760), block 128,
               bf16 N(0,1)/sqrt(128), seed 1.
* ``hunyuan``  1x24 heads, D=128, 33 x 3600 tokens (n=118800), block 128,
               bf16 N(0,1) * u, u ~ U(0.5, 1.5) per (tensor, head, token), seed 2.
* ``long4x``   1x40 heads, D=128, 84 x 1560 tokens (n=131040), block 128,
               bf16 N(0,1), seed 3.
* ``generic``  1x24 heads, D=128, n=32768, block 128, bf16 N(0,1)/sqrt(128),
               seed 4, one seeded tile pattern per head (diagonal,
               multi-diagonal, vertical stripes + diagonal, or a dual window),
               density 10-40 %.
* ``hunyuan_text``  the hunyuan grid followed by 256 joint text tokens
               (n=119056; HunyuanVideo-style joint text + video attention),
               same value recipe, seed 5.
* ``wan_b64``  the wan problem (same tensors, seed 1) with the radial mask cut
               at block 64.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    n: int
    block: int
    seed: int
    dist: str                  # "normal", "normal_scaled", "normal_token_scale"
    frames: int = 0            # radial workloads only
    tokens_per_frame: int = 0  # radial workloads only
    radial: bool = True
    text_tokens: int = 0       # joint text tokens appended after the video tokens

    @property
    def nqb(self) -> int:
        return -(-self.n // self.block)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 64, 4 * 256, 64, 0, "normal_fp32", 4, 256),
    "wan": Workload("wan", 1, 40, 128, 21 * 1560, 128, 1, "normal_scaled", 21, 1560),
    "hunyuan": Workload("hunyuan", 1, 24, 128, 33 * 3600, 128, 2, "normal_token_scale", 33, 3600),
    "long4x": Workload("long4x", 1, 40, 128, 84 * 1560, 128, 3, "normal", 84, 1560),
    "generic": Workload("generic", 1, 24, 128, 32768, 128, 4, "normal_scaled", radial=False),
    "hunyuan_text": Workload("hunyuan_text", 1, 24, 128, 33 * 3600 + 256, 128, 5,
                             "normal_token_scale", 33, 3600, text_tokens=256),
    "wan_b64": Workload("wan_b64", 1, 40, 128, 21 * 1560, 64, 1, "normal_scaled", 21, 1560),
}


def make_qkv(w: Workload, device="cpu", heads: int | None = None):
    """Seeded bf16 Q, K, V of shape ``[batch, heads, n, head_dim]`` on ``device``.

    ``heads`` overrides the head count (for reduced-size variants); the seed is
    the workload's. The same (workload, device) always gives the same tensors.
    """
    H = w.heads if heads is None else heads
    shape = (w.batch, H, w.n, w.head_dim)
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    out = []
    for _ in range(3):
        x = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        if w.dist == "normal_scaled":
            x = x / math.sqrt(w.head_dim)
        elif w.dist == "normal_token_scale":
            u = torch.rand((w.batch, H, w.n, 1), generator=g, device=dev, dtype=torch.float32)
            x = x * (0.5 + u)
        out.append(x.to(torch.bfloat16).contiguous())
    return tuple(out)


def make_random_qkv(batch, heads, n, head_dim, seed, device="cpu", scale=1.0):
    """Seeded bf16 N(0, scale^2) tensors for edge-case shapes."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return tuple((torch.randn((batch, heads, n, head_dim), generator=g, device=dev) * scale)
                 .to(torch.bfloat16).contiguous() for _ in range(3))


def make_module_inputs(batch, n, heads, head_dim, seed, device="cpu", bias=True):
    """Seeded bf16 inputs of the radial attention module: ``x [batch, n, C]``
    ~ N(0, 1); stacked ``w_qkv [3C, C]`` and ``w_out [C, C]`` ~ N(0, 1/C) (unit
    variance after projection, like a trained layer's scale); biases ~
    N(0, 0.1^2) or None. ``C = heads * head_dim``. Returns
    ``(x, w_qkv, b_qkv, w_out, b_out)``."""
    C = heads * head_dim
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)

    def draw(shape, std):
        return (torch.randn(shape, generator=g, device=dev) * std).to(torch.bfloat16).contiguous()

    x = draw((batch, n, C), 1.0)
    w_qkv = draw((3 * C, C), C ** -0.5)
    w_out = draw((C, C), C ** -0.5)
    b_qkv = draw((3 * C,), 0.1) if bias else None
    b_out = draw((C,), 0.1) if bias else None
    return x, w_qkv, b_qkv, w_out, b_out


# ----------------------------------------------------------------------------
# Per-head tile patterns for the generic workload (tile = one block).
# Families: the diagonal, multi-diagonal and vertical-stripe patterns of the
# Sparse-vDiT skill page ("Sparse attention patterns"), and the dual-window
# (local band plus an axial stripe) family of the Compact Attention abstract.
# ----------------------------------------------------------------------------

def _pattern(rng: np.random.Generator, nb: int) -> tuple[str, np.ndarray, dict]:
    """One seeded draw: ``(kind, mask, descriptor)``. The descriptor states the
    same pattern as data (``bands`` of ``kb - qb`` offsets, ``axial`` period
    and half-width, stripe ``columns``) for the device-side pattern builder."""
    qb = np.arange(nb)[:, None]
    kb = np.arange(nb)[None, :]
    kind = ("dual_window", "diagonal", "multi_diagonal", "stripe_diagonal")[rng.integers(4)]
    desc = {"bands": [], "axial": None, "columns": []}
    if kind == "diagonal":
        w = int(rng.integers(8, 64))
        m = np.abs(qb - kb) <= w
        desc["bands"].append((-w, w))
    elif kind == "multi_diagonal":
        c = int(rng.integers(1, 4))
        m = np.abs(qb - kb) <= c
        desc["bands"].append((-c, c))
        for off in rng.integers(-nb // 2, nb // 2, size=int(rng.integers(3, 9))):
            h = int(rng.integers(2, 9))
            m |= np.abs(kb - qb - int(off)) <= h
            desc["bands"].append((int(off) - h, int(off) + h))
    elif kind == "stripe_diagonal":
        c = int(rng.integers(1, 5))
        m = np.abs(qb - kb) <= c
        cols = rng.choice(nb, size=int(rng.integers(20, 90)), replace=False)
        m |= np.isin(kb, cols)
        desc["bands"].append((-c, c))
        desc["columns"] = sorted(int(x) for x in cols)
    else:  # dual window: local band of total width 2..16 tiles plus an axial stripe
        width = int(rng.integers(2, 17))
        period = int(rng.choice([8, 16, 32]))
        a = int(rng.integers(0, 2))
        rel = kb - qb
        m = (rel >= -(width // 2)) & (rel < width - width // 2)
        md = np.mod(rel, period)
        m |= (md <= a) | (md >= period - a)
        desc["bands"].append((-(width // 2), width - width // 2 - 1))
        desc["axial"] = (period, a)
    return kind, np.broadcast_to(m, (nb, nb)).copy(), desc


def _draw_generic(heads: int, nqb: int, seed_base: int, density):
    draws = []
    for h in range(heads):
        rng = np.random.default_rng(seed_base + h)
        while True:
            kind, m, desc = _pattern(rng, nqb)
            if density[0] <= m.mean() <= density[1]:
                break
        m[np.arange(nqb), np.arange(nqb)] = True
        desc["bands"].append((0, 0))  # the diagonal tile every row keeps
        draws.append((kind, m, desc))
    return draws


def make_generic_lists(heads: int, nqb: int, seed_base: int = 1000,
                       density=(0.10, 0.40)):
    """One seeded tile pattern per head, redrawn until its density is in range.

    Returns ``(row_ptr int32[heads*nqb+1], col_idx int32[nnz], kinds)``; head
    ``h``'s rows start at ``h * nqb``. Every row keeps its diagonal tile, so no
    row is empty.
    """
    draws = _draw_generic(heads, nqb, seed_base, density)
    allm = np.concatenate([m for _, m, _ in draws], axis=0)
    counts = allm.sum(axis=1)
    row_ptr = np.zeros(allm.shape[0] + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    _, cols = np.nonzero(allm)
    return row_ptr.astype(np.int32), cols.astype(np.int32), [k for k, _, _ in draws]


def generic_tile_patterns(heads: int, nqb: int, seed_base: int = 1000,
                          density=(0.10, 0.40)) -> list[dict]:
    """The descriptors of :func:`make_generic_lists`'s patterns (same draws),
    diagonal tile included, for building the same lists from the patterns."""
    return [d for _, _, d in _draw_generic(heads, nqb, seed_base, density)]


def random_block_lists(num_rows: int, nkb: int, density: float, seed: int,
                       empty_rows=(), force=None):
    """Seeded random CSR lists (sorted, unique) for edge-case tests.

    ``empty_rows``: rows left empty. ``force``: dict row -> list of blocks that
    replaces the random draw for that row.
    """
    rng = np.random.default_rng(seed)
    m = rng.random((num_rows, nkb)) < density
    for r in empty_rows:
        m[r] = False
    for r, cols in (force or {}).items():
        m[r] = False
        m[r, list(cols)] = True
    counts = m.sum(axis=1)
    row_ptr = np.zeros(num_rows + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    _, cols = np.nonzero(m)
    return row_ptr.astype(np.int32), cols.astype(np.int32)


def sample_rows(n: int, block: int, tokens_per_frame: int, count: int, seed: int) -> np.ndarray:
    """Query rows to check at full size: seeded rows plus the first and last row,
    every row of the ragged last block, and rows next to frame boundaries."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(n, size=min(count, n), replace=False).tolist())
    rows |= {0, n - 1}
    last = (n - 1) // block * block
    rows |= set(range(last, n))
    if tokens_per_frame:
        for f in range(1, n // tokens_per_frame):
            b = f * tokens_per_frame
            rows |= {b - 1, b}
    return np.array(sorted(r for r in rows if 0 <= r < n), dtype=np.int64)
