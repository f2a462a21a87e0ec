"""Radial block-sparse softmax attention (forward) for NVIDIA B200 / sm_100a.

A thin Python binding over libbsa's C ABI (include/bsa.h). The functions named
``bsa_*`` mirror the C entry points one to one and only marshal arguments;
PyTorch supplies device memory and the current CUDA stream. Every step of the
computation runs in the library's CUDA kernels.

Typical use::

    import block_sparse_attention_radial_b200 as bsa
    lists = bsa.radial_block_lists(frames=21, tokens_per_frame=1560, block=128)
    out, lse = bsa.attention(q, k, v, lists)      # q, k, v: bf16 [B, H, n, D] on cuda
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import TILE_PATTERN_MAX_BANDS, BlockListsC, LayoutC, STATUS_NAMES, TilePatternC

__all__ = [
    "BsaError", "BlockLists", "bsa_radial_mask_build", "bsa_attn_fwd_workspace_bytes",
    "bsa_attn_fwd", "bsa_attn_dense_masked_ref", "bsa_validate_lists", "bsa_get_device_status",
    "bsa_get_timeout_detail", "bsa_status_string", "bsa_last_cuda_error", "bsa_set_test_hooks",
    "radial_block_lists", "block_lists_from_csr", "attention", "dense_masked_reference",
    "computed_flops", "bsa_attn_fwd_noalloc", "bsa_selftest_exp2", "NOALLOC_MAX_ORDER_ENTRIES",
    "bsa_gemm_bf16", "bsa_joint_mask_build_varlen", "bsa_attn_fwd_varlen",
    "bsa_attn_fwd_varlen_workspace_bytes", "radial_block_lists_varlen", "attention_varlen",
    "bsa_attn_bwd_varlen", "bsa_attn_bwd_varlen_workspace_bytes", "attention_varlen_backward",
    "bsa_attn_bwd_one_pass", "bsa_attn_bwd_one_pass_workspace_bytes",
    "bsa_attn_fwd_patterns", "bsa_attn_fwd_radial",
    "bsa_attn_fwd_strided", "bsa_attn_module_workspace_bytes", "bsa_joint_mask_build",
    "bsa_attn_fwd_host", "bsa_attn_fwd_host_workspace_bytes", "bsa_attn_bwd_strided",
    "bsa_attn_module_bwd", "bsa_attn_module_bwd_workspace_bytes", "attention_module_backward", "bsa_attn_module_fwd",
    "attention_module", "module_flops", "bsa_attn_bwd", "bsa_attn_bwd_workspace_bytes",
    "attention_backward", "bsa_tile_pattern_lists_build", "tile_pattern_block_lists",
    "pack_tile_patterns", "bsa_attn_bwd_host", "bsa_attn_bwd_host_workspace_bytes",
]

# Size of the fixed scratch array behind bsa_attn_fwd_noalloc (int32 entries).
NOALLOC_MAX_ORDER_ENTRIES = 65536


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _lib.load()
        msg = lib.bsa_status_string(status).decode()
        extra = lib.bsa_last_cuda_error().decode() if status == 3 else ""
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({msg}) {extra}".strip())
        self.status = status


def _check(status: int, where: str) -> int:
    if status != 0:
        raise BsaError(status, where)
    return status


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


@dataclass
class BlockLists:
    """CSR key-block lists on the device (see ``bsa_block_lists`` in include/bsa.h)."""

    row_ptr: torch.Tensor       # int32 [num_lists * num_q_blocks + 1]
    col_idx: torch.Tensor       # int32 [nnz]
    num_lists: int
    num_q_blocks: int
    block: int
    k_blocks: int = 0           # key blocks when they differ from num_q_blocks (varlen: the widest item)

    @property
    def num_k_blocks(self) -> int:
        return self.k_blocks or self.num_q_blocks

    @property
    def nnz(self) -> int:
        return int(self.col_idx.numel())

    def c_struct(self) -> BlockListsC:
        return BlockListsC(self.num_lists, self.num_q_blocks, self.num_k_blocks, self.block,
                           self.nnz, self.row_ptr.data_ptr(),
                           self.col_idx.data_ptr() if self.nnz else 0)


# ------------------------------------------------------------- C entry points

def bsa_radial_mask_build(frames: int, tokens_per_frame: int, block: int, row_ptr: torch.Tensor,
                          col_idx: torch.Tensor | None = None, col_capacity: int = 0,
                          want_nnz: bool = True, stream=None) -> int | None:
    """Radial block lists into caller-owned int32 device tensors; returns nnz when asked
    (that synchronises the stream)."""
    lib = _lib.load()
    nnz = ctypes.c_int64(-1)
    st = lib.bsa_radial_mask_build(frames, tokens_per_frame, block, _ptr(row_ptr), _ptr(col_idx),
                                   col_capacity if col_idx is not None else 0,
                                   ctypes.byref(nnz) if want_nnz else None, _stream(stream))
    _check(st, "bsa_radial_mask_build")
    return int(nnz.value) if want_nnz else None


def bsa_joint_mask_build(frames: int, tokens_per_frame: int, text_tokens: int, block: int,
                         row_ptr: torch.Tensor, col_idx: torch.Tensor | None = None,
                         col_capacity: int = 0, want_nnz: bool = True,
                         stream=None) -> int | None:
    """Joint text + video block lists (text tokens after the video tokens, attended
    globally) into caller-owned int32 device tensors; returns nnz when asked."""
    lib = _lib.load()
    nnz = ctypes.c_int64(-1)
    st = lib.bsa_joint_mask_build(frames, tokens_per_frame, text_tokens, block, _ptr(row_ptr),
                                  _ptr(col_idx), col_capacity if col_idx is not None else 0,
                                  ctypes.byref(nnz) if want_nnz else None, _stream(stream))
    _check(st, "bsa_joint_mask_build")
    return int(nnz.value) if want_nnz else None


def bsa_joint_mask_build_varlen(items, block: int, row_ptr: torch.Tensor,
                                col_idx: torch.Tensor | None = None, col_capacity: int = 0,
                                want_nnz: bool = True, stream=None) -> int | None:
    """Concatenated joint lists of a variable-length batch: ``items`` is a list of
    (frames, tokens_per_frame, text_tokens); returns nnz when asked."""
    lib = _lib.load()
    k = len(items)
    arr = ctypes.c_int32 * max(k, 1)
    fr, tp, tx = (arr(*[int(it[i]) for it in items]) for i in range(3))
    nnz = ctypes.c_int64(-1)
    st = lib.bsa_joint_mask_build_varlen(k, fr, tp, tx, block, _ptr(row_ptr), _ptr(col_idx),
                                         col_capacity if col_idx is not None else 0,
                                         ctypes.byref(nnz) if want_nnz else None, _stream(stream))
    _check(st, "bsa_joint_mask_build_varlen")
    return int(nnz.value) if want_nnz else None


def bsa_tile_pattern_lists_build(num_lists: int, num_q_blocks: int, patterns: torch.Tensor,
                                 columns: torch.Tensor | None, row_ptr: torch.Tensor,
                                 col_idx: torch.Tensor | None = None, col_capacity: int = 0,
                                 want_nnz: bool = True, stream=None) -> int | None:
    """Per-head tile-pattern lists into caller-owned int32 device tensors.

    ``patterns``: device bytes of ``bsa_tile_pattern[num_lists]`` (see
    :func:`pack_tile_patterns`); ``columns``: device int32 stripe columns or
    None. Returns nnz when asked (that synchronises the stream)."""
    lib = _lib.load()
    nnz = ctypes.c_int64(-1)
    ncols = 0 if columns is None else int(columns.numel())
    st = lib.bsa_tile_pattern_lists_build(num_lists, num_q_blocks, _ptr(patterns),
                                          _ptr(columns if ncols else None), ncols, _ptr(row_ptr),
                                          _ptr(col_idx),
                                          col_capacity if col_idx is not None else 0,
                                          ctypes.byref(nnz) if want_nnz else None,
                                          _stream(stream))
    _check(st, "bsa_tile_pattern_lists_build")
    return int(nnz.value) if want_nnz else None


def bsa_attn_fwd_workspace_bytes(batch: int, heads: int, lists: BlockLists) -> int:
    return int(_lib.load().bsa_attn_fwd_workspace_bytes(batch, heads, ctypes.byref(lists.c_struct())))


def bsa_attn_fwd(q, k, v, lists: BlockLists, out, lse=None, workspace=None,
                 softmax_scale: float = 0.0, stream=None) -> None:
    """Block-sparse attention forward on the tensor cores (asynchronous)."""
    B, H, n, D = q.shape
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_fwd_workspace_bytes(B, H, ctypes.byref(ls)), 16),
                                dtype=torch.uint8, device=q.device)
    st = lib.bsa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, H, n, D, float(softmax_scale),
                          ctypes.byref(ls), _ptr(out), _ptr(lse), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_fwd")


def _layout(t) -> LayoutC:
    """bsa_layout of a [batch, heads, n, head_dim] view with a contiguous last axis."""
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [batch, heads, n, head_dim] view with a contiguous last axis")
    return LayoutC(t.stride(0), t.stride(1), t.stride(2))


def bsa_attn_fwd_strided(q, k, v, lists: BlockLists, out, lse=None, workspace=None,
                         softmax_scale: float = 0.0, stream=None) -> None:
    """bsa_attn_fwd on strided [B, H, n, D] views (e.g. ``x.view(B, n, H, D).transpose(1, 2)``):
    the kernels read q, k, v and write out through their strides, no copy."""
    B, H, n, D = q.shape
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_fwd_workspace_bytes(B, H, ctypes.byref(ls)), 16),
                                dtype=torch.uint8, device=q.device)
    lq, lk, lv, lo = (_layout(t) for t in (q, k, v, out))
    st = lib.bsa_attn_fwd_strided(_ptr(q), ctypes.byref(lq), _ptr(k), ctypes.byref(lk), _ptr(v),
                                  ctypes.byref(lv), B, H, n, D, float(softmax_scale),
                                  ctypes.byref(ls), _ptr(out), ctypes.byref(lo), _ptr(lse),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream))
    _check(st, "bsa_attn_fwd_strided")


def bsa_attn_fwd_patterns(q, k, v, patterns, columns, out, lse=None, head_pattern=None,
                          workspace=None, softmax_scale: float = 0.0, stream=None) -> None:
    """Forward over per-head tile patterns generated inside the kernel (no
    column list): ``patterns`` / ``columns`` as packed by
    :func:`pack_tile_patterns`; ``head_pattern`` an int32 device tensor mapping
    heads to patterns, or None (one pattern, or one per head)."""
    B, H, n, D = q.shape
    lib = _lib.load()
    L = int(patterns.numel() * patterns.element_size() // ctypes.sizeof(TilePatternC))
    nqb = -(-n // 128)
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_fwd_patterns_workspace_bytes(L, nqb), 16),
                                dtype=torch.uint8, device=q.device)
    st = lib.bsa_attn_fwd_patterns(_ptr(q), _ptr(k), _ptr(v), B, H, n, D, float(softmax_scale),
                                   L, _ptr(patterns), _ptr(columns),
                                   0 if columns is None else columns.numel(), _ptr(head_pattern),
                                   _ptr(out), _ptr(lse), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_fwd_patterns")


def bsa_attn_fwd_radial(q, k, v, frames: int, tokens_per_frame: int, out, lse=None,
                        text_tokens: int = 0, workspace=None, softmax_scale: float = 0.0,
                        stream=None) -> None:
    """Forward over the (joint) radial mask generated inside the kernel."""
    B, H, n, D = q.shape
    lib = _lib.load()
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_fwd_radial_workspace_bytes(
            frames, tokens_per_frame, text_tokens), 16), dtype=torch.uint8, device=q.device)
    st = lib.bsa_attn_fwd_radial(_ptr(q), _ptr(k), _ptr(v), B, H, frames, tokens_per_frame,
                                 text_tokens, D, float(softmax_scale), _ptr(out), _ptr(lse),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(st, "bsa_attn_fwd_radial")


def _cu_array(cu_seqlens):
    cu = [int(c) for c in cu_seqlens]
    return len(cu) - 1, (ctypes.c_int32 * len(cu))(*cu)


def _packed_layout(t):
    """Layout of a packed [total, heads, head_dim] view (contiguous last axis)."""
    if t.dim() != 3 or t.stride(2) != 1:
        raise ValueError("expected a [total, heads, head_dim] view with a contiguous last axis")
    return LayoutC(0, t.stride(1), t.stride(0))


def bsa_attn_fwd_varlen_workspace_bytes(cu_seqlens, heads: int, lists: BlockLists) -> int:
    k, cu = _cu_array(cu_seqlens)
    return int(_lib.load().bsa_attn_fwd_varlen_workspace_bytes(k, cu, heads,
                                                               ctypes.byref(lists.c_struct())))


def bsa_attn_fwd_varlen(q, k, v, cu_seqlens, lists: BlockLists, out, lse=None, workspace=None,
                        softmax_scale: float = 0.0, stream=None) -> None:
    """Variable-length batch forward on packed [total, heads, head_dim] tensors
    (item b = tokens cu_seqlens[b]..cu_seqlens[b+1]); lse is [heads, total]."""
    total, H, D = q.shape
    lib = _lib.load()
    ls = lists.c_struct()
    nitems, cu = _cu_array(cu_seqlens)
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_fwd_varlen_workspace_bytes(
            nitems, cu, H, ctypes.byref(ls)), 16), dtype=torch.uint8, device=q.device)

    lq, lk, lv, lo = (_packed_layout(t) for t in (q, k, v, out))
    st = lib.bsa_attn_fwd_varlen(_ptr(q), ctypes.byref(lq), _ptr(k), ctypes.byref(lk), _ptr(v),
                                 ctypes.byref(lv), nitems, cu, H, D, float(softmax_scale),
                                 ctypes.byref(ls), _ptr(out), ctypes.byref(lo), _ptr(lse),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(st, "bsa_attn_fwd_varlen")


def bsa_attn_bwd_varlen_workspace_bytes(cu_seqlens, heads: int, lists: BlockLists) -> int:
    k, cu = _cu_array(cu_seqlens)
    return int(_lib.load().bsa_attn_bwd_varlen_workspace_bytes(k, cu, heads,
                                                               ctypes.byref(lists.c_struct())))


def bsa_attn_bwd_varlen(q, k, v, out, dout, lse, cu_seqlens, lists: BlockLists, dq, dk, dv,
                        workspace=None, softmax_scale: float = 0.0, stream=None) -> None:
    """Variable-length batch backward on packed [total, heads, head_dim] tensors;
    lse is the forward's [heads, total]."""
    total, H, D = q.shape
    lib = _lib.load()
    ls = lists.c_struct()
    nitems, cu = _cu_array(cu_seqlens)
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_bwd_varlen_workspace_bytes(
            nitems, cu, H, ctypes.byref(ls)), 16), dtype=torch.uint8, device=q.device)
    lay = [_packed_layout(t) for t in (q, k, v, out, dout, dq, dk, dv)]
    st = lib.bsa_attn_bwd_varlen(
        _ptr(q), ctypes.byref(lay[0]), _ptr(k), ctypes.byref(lay[1]), _ptr(v), ctypes.byref(lay[2]),
        _ptr(out), ctypes.byref(lay[3]), _ptr(dout), ctypes.byref(lay[4]), _ptr(lse), nitems, cu,
        H, D, float(softmax_scale), ctypes.byref(ls), _ptr(dq), ctypes.byref(lay[5]), _ptr(dk),
        ctypes.byref(lay[6]), _ptr(dv), ctypes.byref(lay[7]), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_bwd_varlen")


def bsa_attn_fwd_host_workspace_bytes(batch: int, heads: int, n: int, head_dim: int,
                                      lists: BlockLists) -> int:
    return int(_lib.load().bsa_attn_fwd_host_workspace_bytes(batch, heads, n, head_dim,
                                                             ctypes.byref(lists.c_struct())))


def bsa_attn_fwd_host(q, k, v, lists: BlockLists, out, lse=None, workspace=None,
                      softmax_scale: float = 0.0, stream=None, device=None) -> None:
    """bsa_attn_fwd on CPU tensors (pin them for copy/compute overlap): q, k, v
    and out bf16 [B, H, n, D] in host memory, lse float [B, H, n] or None. The
    copies and kernels are enqueued on ``stream``; synchronise it before
    reading ``out``."""
    B, H, n, D = q.shape
    for t in (q, k, v, out, lse):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("bsa_attn_fwd_host takes contiguous host tensors")
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        dev = lists.row_ptr.device if device is None else torch.device(device)
        workspace = torch.empty(lib.bsa_attn_fwd_host_workspace_bytes(B, H, n, D, ctypes.byref(ls)),
                                dtype=torch.uint8, device=dev)
    st = lib.bsa_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), B, H, n, D, float(softmax_scale),
                               ctypes.byref(ls), _ptr(out), _ptr(lse), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_fwd_host")


def bsa_attn_module_workspace_bytes(batch: int, n: int, heads: int, head_dim: int,
                                    lists: BlockLists) -> int:
    return int(_lib.load().bsa_attn_module_workspace_bytes(batch, n, heads, head_dim,
                                                           ctypes.byref(lists.c_struct())))


def bsa_attn_module_fwd(x, w_qkv, b_qkv, w_out, b_out, heads: int, lists: BlockLists, y,
                        workspace=None, softmax_scale: float = 0.0, stream=None) -> None:
    """Radial attention module forward (projections, attention, out projection):
    x, y bf16 [B, n, C]; w_qkv [3C, C]; w_out [C, C]; biases [3C] / [C] or None."""
    B, n, C = x.shape
    D = C // heads
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        workspace = torch.empty(lib.bsa_attn_module_workspace_bytes(B, n, heads, D,
                                                                    ctypes.byref(ls)),
                                dtype=torch.uint8, device=x.device)
    for t in (x, w_qkv, b_qkv, w_out, b_out, y):
        if t is not None and not t.is_contiguous():
            raise ValueError("bsa_attn_module_fwd takes contiguous tensors")
    st = lib.bsa_attn_module_fwd(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(w_out), _ptr(b_out), B, n,
                                 heads, D, float(softmax_scale), ctypes.byref(ls), _ptr(y),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(st, "bsa_attn_module_fwd")


def bsa_attn_module_bwd_workspace_bytes(batch: int, n: int, heads: int, head_dim: int,
                                        lists: BlockLists) -> int:
    return int(_lib.load().bsa_attn_module_bwd_workspace_bytes(batch, n, heads, head_dim,
                                                               ctypes.byref(lists.c_struct())))


def bsa_attn_module_bwd(x, w_qkv, w_out, dy, heads: int, lists: BlockLists, fwd_workspace,
                        dx, dw_qkv, db_qkv, dw_out, db_out, workspace=None,
                        softmax_scale: float = 0.0, stream=None) -> None:
    """Gradients of the module forward whose workspace is ``fwd_workspace``:
    dx [B, n, C], dw_qkv [3C, C], db_qkv [3C] (or None), dw_out [C, C],
    db_out [C] (or None), all bf16."""
    B, n, C = x.shape
    D = C // heads
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        workspace = torch.empty(lib.bsa_attn_module_bwd_workspace_bytes(B, n, heads, D,
                                                                        ctypes.byref(ls)),
                                dtype=torch.uint8, device=x.device)
    for t in (x, w_qkv, w_out, dy, dx, dw_qkv, db_qkv, dw_out, db_out):
        if t is not None and not t.is_contiguous():
            raise ValueError("bsa_attn_module_bwd takes contiguous tensors")
    st = lib.bsa_attn_module_bwd(
        _ptr(x), _ptr(w_qkv), _ptr(w_out), _ptr(dy), B, n, heads, D, float(softmax_scale),
        ctypes.byref(ls), _ptr(fwd_workspace), fwd_workspace.numel() * fwd_workspace.element_size(),
        _ptr(dx), _ptr(dw_qkv), _ptr(db_qkv), _ptr(dw_out), _ptr(db_out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_module_bwd")


def bsa_attn_fwd_noalloc(q, k, v, lists: BlockLists, out, lse=None,
                         softmax_scale: float = 0.0, stream=None) -> None:
    """bsa_attn_fwd without a workspace, for callers that cannot allocate device
    memory (a plugin given only its input and output buffers, a runtime with a
    memory plan fixed at start-up). Its scratch is a fixed array inside the
    library, so it needs num_lists * num_q_blocks <= NOALLOC_MAX_ORDER_ENTRIES;
    calls overlapping on the GPU race on that array. The first call on a device
    resolves the array's address; make it before any stream capture."""
    B, H, n, D = q.shape
    st = _lib.load().bsa_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), B, H, n, D,
                                          float(softmax_scale), ctypes.byref(lists.c_struct()),
                                          _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "bsa_attn_fwd_noalloc")


def bsa_attn_bwd_workspace_bytes(batch: int, heads: int, n: int, lists: BlockLists) -> int:
    return int(_lib.load().bsa_attn_bwd_workspace_bytes(batch, heads, n,
                                                         ctypes.byref(lists.c_struct())))


def bsa_attn_bwd(q, k, v, out, dout, lse, lists: BlockLists, dq, dk, dv, workspace=None,
                 softmax_scale: float = 0.0, stream=None) -> None:
    """Backward pass of :func:`bsa_attn_fwd` on the tensor cores (asynchronous)."""
    B, H, n, D = q.shape
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_bwd_workspace_bytes(B, H, n, ctypes.byref(ls)), 16),
                                dtype=torch.uint8, device=q.device)
    st = lib.bsa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), B, H, n, D,
                          float(softmax_scale), ctypes.byref(ls), _ptr(dq), _ptr(dk), _ptr(dv),
                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                          _stream(stream))
    _check(st, "bsa_attn_bwd")


def bsa_attn_bwd_host_workspace_bytes(batch: int, heads: int, n: int, head_dim: int,
                                      lists: BlockLists) -> int:
    return int(_lib.load().bsa_attn_bwd_host_workspace_bytes(batch, heads, n, head_dim,
                                                             ctypes.byref(lists.c_struct())))


def bsa_attn_bwd_host(q, k, v, out, dout, lse, lists: BlockLists, dq, dk, dv, workspace=None,
                      softmax_scale: float = 0.0, stream=None, device=None) -> None:
    """bsa_attn_bwd on CPU tensors (pin them for copy/compute overlap): q, k, v,
    out, dout and the gradients dq, dk, dv bf16 [B, H, n, D], lse float
    [B, H, n], all contiguous in host memory. Enqueued on ``stream``;
    synchronise it before reading the gradients."""
    B, H, n, D = q.shape
    for t in (q, k, v, out, dout, lse, dq, dk, dv):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("bsa_attn_bwd_host takes contiguous host tensors")
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        dev = lists.row_ptr.device if device is None else torch.device(device)
        workspace = torch.empty(lib.bsa_attn_bwd_host_workspace_bytes(B, H, n, D, ctypes.byref(ls)),
                                dtype=torch.uint8, device=dev)
    st = lib.bsa_attn_bwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), B, H, n,
                               D, float(softmax_scale), ctypes.byref(ls), _ptr(dq), _ptr(dk),
                               _ptr(dv), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_bwd_host")


def bsa_attn_bwd_one_pass_workspace_bytes(batch: int, heads: int, n: int,
                                          lists: BlockLists) -> int:
    return int(_lib.load().bsa_attn_bwd_one_pass_workspace_bytes(batch, heads, n,
                                                                 ctypes.byref(lists.c_struct())))


def bsa_attn_bwd_one_pass(q, k, v, out, dout, lse, lists: BlockLists, dq, dk, dv, workspace=None,
                          softmax_scale: float = 0.0, stream=None) -> None:
    """The backward from one kernel (block 128; dQ parts added in row order)."""
    B, H, n, D = q.shape
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_bwd_one_pass_workspace_bytes(
            B, H, n, ctypes.byref(ls)), 16), dtype=torch.uint8, device=q.device)
    st = lib.bsa_attn_bwd_one_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), B,
                                   H, n, D, float(softmax_scale), ctypes.byref(ls), _ptr(dq),
                                   _ptr(dk), _ptr(dv), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_bwd_one_pass")


def bsa_attn_bwd_strided(q, k, v, out, dout, lse, lists: BlockLists, dq, dk, dv, workspace=None,
                         softmax_scale: float = 0.0, stream=None) -> None:
    """bsa_attn_bwd on strided [B, H, n, D] views (contiguous last axis): reads
    and writes every tensor through its strides, no copy."""
    B, H, n, D = q.shape
    lib = _lib.load()
    ls = lists.c_struct()
    if workspace is None:
        workspace = torch.empty(max(lib.bsa_attn_bwd_workspace_bytes(B, H, n, ctypes.byref(ls)), 16),
                                dtype=torch.uint8, device=q.device)
    lay = [_layout(t) for t in (q, k, v, out, dout, dq, dk, dv)]
    st = lib.bsa_attn_bwd_strided(
        _ptr(q), ctypes.byref(lay[0]), _ptr(k), ctypes.byref(lay[1]), _ptr(v), ctypes.byref(lay[2]),
        _ptr(out), ctypes.byref(lay[3]), _ptr(dout), ctypes.byref(lay[4]), _ptr(lse), B, H, n, D,
        float(softmax_scale), ctypes.byref(ls), _ptr(dq), ctypes.byref(lay[5]), _ptr(dk),
        ctypes.byref(lay[6]), _ptr(dv), ctypes.byref(lay[7]), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bsa_attn_bwd_strided")


def bsa_attn_dense_masked_ref(q, k, v, lists: BlockLists, out, lse=None,
                              softmax_scale: float = 0.0, stream=None) -> None:
    """Same result from the plain fp32 CUDA-core reference kernel (asynchronous)."""
    B, H, n, D = q.shape
    st = _lib.load().bsa_attn_dense_masked_ref(_ptr(q), _ptr(k), _ptr(v), B, H, n, D,
                                               float(softmax_scale), ctypes.byref(lists.c_struct()),
                                               _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "bsa_attn_dense_masked_ref")


def bsa_validate_lists(lists: BlockLists, stream=None) -> int:
    """Returns the status (0 = well formed, 5 = BSA_ERR_BAD_LISTS); raises on other errors."""
    st = _lib.load().bsa_validate_lists(ctypes.byref(lists.c_struct()), _stream(stream))
    if st not in (0, 5):
        _check(st, "bsa_validate_lists")
    return st


def bsa_get_device_status(stream=None) -> int:
    st = _lib.load().bsa_get_device_status(_stream(stream))
    if st == 3:
        _check(st, "bsa_get_device_status")
    return st


def bsa_get_timeout_detail() -> list[int]:
    out = (ctypes.c_int32 * 4)()
    _check(_lib.load().bsa_get_timeout_detail(out), "bsa_get_timeout_detail")
    return list(out)


def bsa_status_string(status: int) -> str:
    return _lib.load().bsa_status_string(status).decode()


def bsa_last_cuda_error() -> str:
    return _lib.load().bsa_last_cuda_error().decode()


def bsa_gemm_bf16(a, b, out, bias=None, a_mn_major: bool = False, b_mn_major: bool = False,
                  stream=None) -> None:
    """out[m, n] = A[m, k] B[k, n] (+ bias[n]) on the library's tcgen05 GEMM.

    ``a`` is A stored as [m, k] (``a_mn_major=False``) or as its transpose
    [k, m]; ``b`` is B stored as [n, k] (``b_mn_major=False``, an nn.Linear
    weight) or as [k, n]. 2-D bf16 device tensors with a contiguous last axis;
    the row strides are passed through."""
    m, n = out.shape
    k = a.shape[0] if a_mn_major else a.shape[1]
    st = _lib.load().bsa_gemm_bf16(_ptr(a), a.stride(0), int(a_mn_major), _ptr(b), b.stride(0),
                                   int(b_mn_major), _ptr(bias), _ptr(out), out.stride(0), m, n, k,
                                   _stream(stream))
    _check(st, "bsa_gemm_bf16")


def bsa_selftest_exp2(x: torch.Tensor):
    """(poly, mufu, exp2f) results of the softmax's exponential paths on float32 ``x``."""
    ys = [torch.empty_like(x) for _ in range(3)]
    _check(_lib.load().bsa_selftest_exp2(_ptr(x), *(_ptr(y) for y in ys), x.numel(),
                                         _stream(None)), "bsa_selftest_exp2")
    return tuple(ys)


def bsa_set_test_hooks(wait_limit_ns: int = 0, fault_flags: int = 0) -> None:
    _check(_lib.load().bsa_set_test_hooks(wait_limit_ns, fault_flags), "bsa_set_test_hooks")


# ------------------------------------------------------------- conveniences

def radial_block_lists(frames: int, tokens_per_frame: int, block: int = 128,
                       device=None, stream=None, text_tokens: int = 0) -> BlockLists:
    """Build the radial lists on the GPU (two calls: count, then fill). With
    ``text_tokens`` > 0, the joint lists of the video tokens followed by that
    many text tokens (:func:`bsa_joint_mask_build`)."""
    device = torch.device("cuda") if device is None else torch.device(device)
    n = frames * tokens_per_frame + text_tokens
    nqb = -(-n // block)
    row_ptr = torch.empty(nqb + 1, dtype=torch.int32, device=device)
    nnz = bsa_joint_mask_build(frames, tokens_per_frame, text_tokens, block, row_ptr,
                               stream=stream)
    col_idx = torch.empty(max(nnz, 1), dtype=torch.int32, device=device)
    got = bsa_joint_mask_build(frames, tokens_per_frame, text_tokens, block, row_ptr, col_idx,
                               col_idx.numel(), stream=stream)
    assert got == nnz
    return BlockLists(row_ptr, col_idx[:nnz], 1, nqb, block)


def radial_block_lists_varlen(items, block: int = 128, device=None, stream=None) -> BlockLists:
    """Concatenated joint lists of a variable-length batch on the GPU; ``items``
    is a list of (frames, tokens_per_frame, text_tokens)."""
    device = torch.device("cuda") if device is None else torch.device(device)
    nqbs = [-(-(f * s + t) // block) for f, s, t in items]
    row_ptr = torch.empty(sum(nqbs) + 1, dtype=torch.int32, device=device)
    nnz = bsa_joint_mask_build_varlen(items, block, row_ptr, stream=stream)
    col_idx = torch.empty(max(nnz, 1), dtype=torch.int32, device=device)
    got = bsa_joint_mask_build_varlen(items, block, row_ptr, col_idx, col_idx.numel(),
                                      stream=stream)
    assert got == nnz
    return BlockLists(row_ptr, col_idx[:nnz], 1, sum(nqbs), block, k_blocks=max(nqbs))


def attention_varlen(q, k, v, cu_seqlens, lists: BlockLists, softmax_scale: float = 0.0,
                     want_lse: bool = True, stream=None):
    """Variable-length batch on packed [total, heads, head_dim] q, k, v; returns
    ``(out [total, heads, head_dim], lse [heads, total])``."""
    total, H, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((H, total), dtype=torch.float32, device=q.device) if want_lse else None
    bsa_attn_fwd_varlen(q, k, v, cu_seqlens, lists, out, lse, None, softmax_scale, stream)
    return out, lse


def attention_varlen_backward(q, k, v, out, dout, lse, cu_seqlens, lists: BlockLists,
                              softmax_scale: float = 0.0, stream=None):
    """Gradients ``(dq, dk, dv)`` of :func:`attention_varlen` (packed
    [total, heads, head_dim]; lse [heads, total] from the forward)."""
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    bsa_attn_bwd_varlen(q, k, v, out, dout, lse, cu_seqlens, lists, dq, dk, dv, None,
                        softmax_scale, stream)
    return dq, dk, dv


def pack_tile_patterns(patterns, device=None):
    """Lay out per-head pattern descriptors as ``bsa_tile_pattern[]`` and the
    shared stripe-column array, both on ``device``.

    Each descriptor is a dict with ``bands`` (list of ``(lo, hi)`` offsets
    ``kb - qb``, at most 16), ``axial`` (``None`` or ``(period, halfwidth)``)
    and ``columns`` (stripe key blocks). Returns ``(patterns_u8, columns_i32
    or None)``."""
    device = torch.device("cuda") if device is None else torch.device(device)
    arr = (TilePatternC * len(patterns))()
    cols: list[int] = []
    for c, p in zip(arr, patterns):
        bands = list(p.get("bands", ()))
        if len(bands) > TILE_PATTERN_MAX_BANDS:
            raise ValueError(f"at most {TILE_PATTERN_MAX_BANDS} bands per pattern")
        c.num_bands = len(bands)
        for t, (lo, hi) in enumerate(bands):
            c.band_lo[t], c.band_hi[t] = int(lo), int(hi)
        axial = p.get("axial")
        if axial is not None and (int(axial[0]) < 1 or int(axial[1]) < 0):
            raise ValueError("axial term needs a period >= 1 and a half-width >= 0 (None: no term)")
        c.axial_period, c.axial_halfwidth = (0, 0) if axial is None else (int(axial[0]), int(axial[1]))
        c.columns_begin = len(cols)
        cols.extend(int(x) for x in p.get("columns", ()))
        c.columns_end = len(cols)
    raw = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)
    col_t = torch.tensor(cols, dtype=torch.int32, device=device) if cols else None
    return raw, col_t


def tile_pattern_block_lists(patterns, num_q_blocks: int, block: int = 128, device=None,
                             stream=None) -> BlockLists:
    """Build one list per head from its tile pattern on the GPU (two calls:
    count, then fill); ``num_lists = len(patterns)``."""
    device = torch.device("cuda") if device is None else torch.device(device)
    raw, cols = pack_tile_patterns(patterns, device)
    rows = len(patterns) * num_q_blocks
    row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=device)
    nnz = bsa_tile_pattern_lists_build(len(patterns), num_q_blocks, raw, cols, row_ptr,
                                       stream=stream)
    col_idx = torch.empty(max(nnz, 1), dtype=torch.int32, device=device)
    got = bsa_tile_pattern_lists_build(len(patterns), num_q_blocks, raw, cols, row_ptr, col_idx,
                                       col_idx.numel(), stream=stream)
    assert got == nnz
    return BlockLists(row_ptr, col_idx[:nnz], len(patterns), num_q_blocks, block)


def block_lists_from_csr(row_ptr, col_idx, num_lists: int, num_q_blocks: int, block: int,
                         device=None) -> BlockLists:
    """Wrap host or device CSR arrays (copied to ``device`` as int32)."""
    device = torch.device("cuda") if device is None else torch.device(device)
    rp = torch.as_tensor(row_ptr, dtype=torch.int32).to(device).contiguous()
    ci = torch.as_tensor(col_idx, dtype=torch.int32).to(device).contiguous()
    return BlockLists(rp, ci, num_lists, num_q_blocks, block)


def attention(q, k, v, lists: BlockLists, softmax_scale: float = 0.0, want_lse: bool = True,
              workspace=None, stream=None, out=None):
    """Run the forward on [B, H, n, D] tensors; returns ``(out, lse)``.

    Contiguous q, k, v (and ``out``, allocated contiguous when not given) go to
    :func:`bsa_attn_fwd`; strided views (a contiguous last axis, e.g. heads
    split off a [B, n, H*D] projection by ``view(B, n, H, D).transpose(1, 2)``)
    to :func:`bsa_attn_fwd_strided`, which reads and writes them in place."""
    B, H, n, D = q.shape
    if out is None:
        out = torch.empty((B, H, n, D), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device) if want_lse else None
    if all(t.is_contiguous() for t in (q, k, v, out)):
        bsa_attn_fwd(q, k, v, lists, out, lse, workspace, softmax_scale, stream)
    else:
        bsa_attn_fwd_strided(q, k, v, lists, out, lse, workspace, softmax_scale, stream)
    return out, lse


def attention_module(x, w_qkv, b_qkv, w_out, b_out, heads: int, lists: BlockLists,
                     softmax_scale: float = 0.0, workspace=None, stream=None):
    """Allocate y and run :func:`bsa_attn_module_fwd`; returns y (bf16 [B, n, C]).
    Pass ``workspace`` (of :func:`bsa_attn_module_workspace_bytes`) to keep the
    saved q/k/v, attention output and lse for :func:`attention_module_backward`."""
    y = torch.empty_like(x)
    bsa_attn_module_fwd(x, w_qkv, b_qkv, w_out, b_out, heads, lists, y, workspace, softmax_scale,
                        stream)
    return y


def attention_module_backward(x, w_qkv, w_out, dy, heads: int, lists: BlockLists, fwd_workspace,
                              softmax_scale: float = 0.0, biases: bool = True, workspace=None,
                              stream=None):
    """Allocate the gradients and run :func:`bsa_attn_module_bwd`; returns
    ``(dx, dw_qkv, db_qkv, dw_out, db_out)`` (the bias gradients None when
    ``biases`` is False)."""
    C = x.shape[-1]
    dx, dwq, dwo = torch.empty_like(x), torch.empty_like(w_qkv), torch.empty_like(w_out)
    dbq = torch.empty(3 * C, dtype=x.dtype, device=x.device) if biases else None
    dbo = torch.empty(C, dtype=x.dtype, device=x.device) if biases else None
    bsa_attn_module_bwd(x, w_qkv, w_out, dy, heads, lists, fwd_workspace, dx, dwq, dbq, dwo, dbo,
                        workspace, softmax_scale, stream)
    return dx, dwq, dbq, dwo, dbo


def module_flops(batch: int, n: int, heads: int, head_dim: int, attention_flops: int) -> int:
    """FLOPs of one module forward: the two projection GEMMs (2*rows*C*3C and
    2*rows*C*C) plus the attention's computed-block FLOPs."""
    C = heads * head_dim
    return 8 * batch * n * C * C + int(attention_flops)


def attention_backward(q, k, v, out, dout, lse, lists: BlockLists, softmax_scale: float = 0.0,
                       workspace=None, stream=None, grads=None):
    """Gradients of :func:`attention`; returns ``(dq, dk, dv)``. ``grads`` may
    give the three output tensors (any views with a contiguous last axis);
    otherwise they are allocated contiguous. All-contiguous calls go to
    :func:`bsa_attn_bwd`, others to :func:`bsa_attn_bwd_strided`."""
    if grads is None:
        shape = tuple(q.shape)
        grads = tuple(torch.empty(shape, dtype=q.dtype, device=q.device) for _ in range(3))
    dq, dk, dv = grads
    if all(t.is_contiguous() for t in (q, k, v, out, dout, dq, dk, dv)):
        bsa_attn_bwd(q, k, v, out, dout, lse, lists, dq, dk, dv, workspace, softmax_scale, stream)
    else:
        bsa_attn_bwd_strided(q, k, v, out, dout, lse, lists, dq, dk, dv, workspace, softmax_scale,
                             stream)
    return dq, dk, dv


def dense_masked_reference(q, k, v, lists: BlockLists, softmax_scale: float = 0.0, stream=None):
    B, H, n, _ = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    bsa_attn_dense_masked_ref(q, k, v, lists, out, lse, softmax_scale, stream)
    return out, lse


def computed_flops(row_ptr, col_idx, n: int, block: int, head_dim: int, batch: int,
                   heads: int, num_lists: int) -> int:
    """FLOPs on computed blocks: 4 * D * sum over listed (qb, kb) of valid rows x valid cols,
    over every batch item and head (host arrays)."""
    import numpy as np

    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx, dtype=np.int64)
    nqb = -(-n // block)
    valid = np.minimum(block, n - np.arange(nqb) * block)
    total = 0
    for lst in range(num_lists):
        rows = np.arange(nqb) + lst * nqb
        counts = np.diff(rp[lst * nqb: lst * nqb + nqb + 1])
        qv = np.repeat(valid, counts)
        kv = valid[ci[rp[rows[0]]:rp[rows[-1] + 1]]]
        total += int((qv * kv).sum())
    mult = heads if num_lists == 1 else 1
    return 4 * head_dim * batch * mult * total
