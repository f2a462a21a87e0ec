"""ctypes declarations of libbsa's C ABI (include/bsa.h).

Only argument marshalling lives here: every step of the computation runs in
the library's CUDA kernels. Loading fails loudly when the library has not been
built; there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

# Names exported by the library; kept in the same order as include/bsa.h.
EXPORTS = (
    "bsa_radial_mask_build",
    "bsa_joint_mask_build",
    "bsa_joint_mask_build_varlen",
    "bsa_tile_pattern_lists_build",
    "bsa_attn_fwd_workspace_bytes",
    "bsa_attn_fwd",
    "bsa_attn_fwd_strided",
    "bsa_attn_fwd_patterns_workspace_bytes",
    "bsa_attn_fwd_patterns",
    "bsa_attn_fwd_radial_workspace_bytes",
    "bsa_attn_fwd_radial",
    "bsa_attn_fwd_varlen_workspace_bytes",
    "bsa_attn_fwd_varlen",
    "bsa_attn_fwd_host_workspace_bytes",
    "bsa_attn_fwd_host",
    "bsa_attn_module_workspace_bytes",
    "bsa_attn_module_fwd",
    "bsa_attn_module_bwd_workspace_bytes",
    "bsa_attn_module_bwd",
    "bsa_gemm_bf16",
    "bsa_attn_dense_masked_ref",
    "bsa_attn_bwd",
    "bsa_attn_bwd_strided",
    "bsa_attn_bwd_varlen_workspace_bytes",
    "bsa_attn_bwd_varlen",
    "bsa_attn_bwd_workspace_bytes",
    "bsa_attn_bwd_one_pass_workspace_bytes",
    "bsa_attn_bwd_one_pass",
    "bsa_attn_bwd_host_workspace_bytes",
    "bsa_attn_bwd_host",
    "bsa_validate_lists",
    "bsa_get_device_status",
    "bsa_get_timeout_detail",
    "bsa_status_string",
    "bsa_last_cuda_error",
    "bsa_set_test_hooks",
    "bsa_selftest_exp2",
    "bsa_attn_fwd_noalloc",
)

STATUS_NAMES = {
    0: "BSA_OK",
    1: "BSA_ERR_INVALID_ARG",
    2: "BSA_ERR_UNSUPPORTED",
    3: "BSA_ERR_CUDA",
    4: "BSA_ERR_DEVICE_TIMEOUT",
    5: "BSA_ERR_BAD_LISTS",
    6: "BSA_ERR_CAPACITY",
    7: "BSA_ERR_SCRATCH_LIMIT",
}


TILE_PATTERN_MAX_BANDS = 16


class TilePatternC(ctypes.Structure):
    """Mirror of ``bsa_tile_pattern``."""

    _fields_ = [
        ("num_bands", ctypes.c_int32),
        ("band_lo", ctypes.c_int32 * TILE_PATTERN_MAX_BANDS),
        ("band_hi", ctypes.c_int32 * TILE_PATTERN_MAX_BANDS),
        ("axial_period", ctypes.c_int32),
        ("axial_halfwidth", ctypes.c_int32),
        ("columns_begin", ctypes.c_int32),
        ("columns_end", ctypes.c_int32),
    ]


class BlockListsC(ctypes.Structure):
    """Mirror of ``bsa_block_lists``."""

    _fields_ = [
        ("num_lists", ctypes.c_int32),
        ("num_q_blocks", ctypes.c_int32),
        ("num_k_blocks", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("nnz", ctypes.c_int32),
        ("row_ptr", ctypes.c_void_p),
        ("col_idx", ctypes.c_void_p),
    ]


class LayoutC(ctypes.Structure):
    """Mirror of ``bsa_layout`` (element strides; head_dim contiguous)."""

    _fields_ = [
        ("batch_stride", ctypes.c_int64),
        ("head_stride", ctypes.c_int64),
        ("token_stride", ctypes.c_int64),
    ]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbsa and declare its signatures (cached)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libbsa.so not found at {path}; build it with `python -c 'import __graft_entry__ as g; g.build()'` "
            "(the CUDA library is required: there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    i32, i64, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    lp = ctypes.POINTER(BlockListsC)
    yp = ctypes.POINTER(LayoutC)
    sig = {
        "bsa_radial_mask_build": (ctypes.c_int, [i32, i32, i32, vp, vp, i64, ctypes.POINTER(i64), vp]),
        "bsa_joint_mask_build": (ctypes.c_int, [i32, i32, i32, i32, vp, vp, i64,
                                                ctypes.POINTER(i64), vp]),
        "bsa_tile_pattern_lists_build": (ctypes.c_int, [i32, i32, vp, vp, i64, vp, vp, i64,
                                                        ctypes.POINTER(i64), vp]),
        "bsa_joint_mask_build_varlen": (ctypes.c_int, [i32, vp, vp, vp, i32, vp, vp, i64,
                                                       ctypes.POINTER(i64), vp]),
        "bsa_attn_fwd_varlen_workspace_bytes": (sz, [i32, vp, i32, lp]),
        "bsa_attn_fwd_patterns_workspace_bytes": (sz, [i32, i32]),
        "bsa_attn_fwd_patterns": (ctypes.c_int, [vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                                 i32, vp, vp, i64, vp, vp, vp, vp, sz, vp]),
        "bsa_attn_fwd_radial_workspace_bytes": (sz, [i32, i32, i32]),
        "bsa_attn_fwd_radial": (ctypes.c_int, [vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                               ctypes.c_float, vp, vp, vp, sz, vp]),
        "bsa_attn_fwd_varlen": (ctypes.c_int, [vp, yp, vp, yp, vp, yp, i32, vp, i32, i32,
                                               ctypes.c_float, lp, vp, yp, vp, vp, sz, vp]),
        "bsa_attn_fwd_workspace_bytes": (sz, [i32, i32, lp]),
        "bsa_attn_fwd": (ctypes.c_int, [vp, vp, vp, i32, i32, i32, i32, ctypes.c_float, lp,
                                        vp, vp, vp, sz, vp]),
        "bsa_attn_fwd_strided": (ctypes.c_int, [vp, yp, vp, yp, vp, yp, i32, i32, i32, i32,
                                                ctypes.c_float, lp, vp, yp, vp, vp, sz, vp]),
        "bsa_attn_module_workspace_bytes": (sz, [i32, i32, i32, i32, lp]),
        "bsa_attn_fwd_host_workspace_bytes": (sz, [i32, i32, i32, i32, lp]),
        "bsa_attn_module_bwd_workspace_bytes": (sz, [i32, i32, i32, i32, lp]),
        "bsa_attn_module_bwd": (ctypes.c_int, [vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                               lp, vp, sz, vp, vp, vp, vp, vp, vp, sz, vp]),
        "bsa_attn_fwd_host": (ctypes.c_int, [vp, vp, vp, i32, i32, i32, i32, ctypes.c_float, lp,
                                             vp, vp, vp, sz, vp]),
        "bsa_attn_module_fwd": (ctypes.c_int, [vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                               ctypes.c_float, lp, vp, vp, sz, vp]),
        "bsa_attn_dense_masked_ref": (ctypes.c_int, [vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                                     lp, vp, vp, vp]),
        "bsa_validate_lists": (ctypes.c_int, [lp, vp]),
        "bsa_get_device_status": (ctypes.c_int, [vp]),
        "bsa_get_timeout_detail": (ctypes.c_int, [ctypes.POINTER(i32)]),
        "bsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "bsa_last_cuda_error": (ctypes.c_char_p, []),
        "bsa_set_test_hooks": (ctypes.c_int, [i64, i32]),
        "bsa_gemm_bf16": (ctypes.c_int, [vp, i64, i32, vp, i64, i32, vp, vp, i64, i64, i64, i64,
                                         vp]),
        "bsa_selftest_exp2": (ctypes.c_int, [vp, vp, vp, vp, i32, vp]),
        "bsa_attn_fwd_noalloc": (ctypes.c_int, [vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                                lp, vp, vp, vp]),
        "bsa_attn_bwd": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                        lp, vp, vp, vp, vp, sz, vp]),
        "bsa_attn_bwd_workspace_bytes": (sz, [i32, i32, i32, lp]),
        "bsa_attn_bwd_one_pass_workspace_bytes": (sz, [i32, i32, i32, lp]),
        "bsa_attn_bwd_one_pass": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                                 ctypes.c_float, lp, vp, vp, vp, vp, sz, vp]),
        "bsa_attn_bwd_host_workspace_bytes": (sz, [i32, i32, i32, i32, lp]),
        "bsa_attn_bwd_host": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                             ctypes.c_float, lp, vp, vp, vp, vp, sz, vp]),
        "bsa_attn_bwd_strided": (ctypes.c_int, [vp, yp, vp, yp, vp, yp, vp, yp, vp, yp, vp, i32,
                                                i32, i32, i32, ctypes.c_float, lp, vp, yp, vp, yp,
                                                vp, yp, vp, sz, vp]),
        "bsa_attn_bwd_varlen_workspace_bytes": (sz, [i32, vp, i32, lp]),
        "bsa_attn_bwd_varlen": (ctypes.c_int, [vp, yp, vp, yp, vp, yp, vp, yp, vp, yp, vp, i32,
                                               vp, i32, i32, ctypes.c_float, lp, vp, yp, vp, yp,
                                               vp, yp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
