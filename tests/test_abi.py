"""The C ABI library loads on a machine without a GPU, exports every entry point
include/bsa.h declares, and rejects bad arguments on the host before any CUDA
call (CPU only: nothing here launches a kernel)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_radial_b200 import _lib

    if not os.path.exists(_lib.LIB_PATH):
        from block_sparse_attention_radial_b200.build import build

        build()
    return _lib.load()


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("bsa_radial_mask_build", "bsa_attn_fwd", "bsa_attn_dense_masked_ref",
              "bsa_attn_fwd_workspace_bytes", "bsa_get_device_status", "bsa_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from block_sparse_attention_radial_b200._lib import EXPORTS

    names = _declared()
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(EXPORTS) == names


def test_status_strings(lib):
    for code in range(7):
        s = lib.bsa_status_string(code).decode()
        assert s and s != "unknown status"
    assert lib.bsa_status_string(99).decode() == "unknown status"


def test_workspace_bytes(lib):
    from block_sparse_attention_radial_b200._lib import BlockListsC

    # the work order (one int per query block and list, 256-byte aligned) and
    # 256 bytes for the work counter
    ls = BlockListsC(1, 256, 256, 128, 1000, 0, 0)
    assert lib.bsa_attn_fwd_workspace_bytes(1, 40, ctypes.byref(ls)) == 1024 + 256
    ls = BlockListsC(24, 256, 256, 128, 1000, 0, 0)
    assert lib.bsa_attn_fwd_workspace_bytes(1, 24, ctypes.byref(ls)) == 24 * 256 * 4 + 256
    ls = BlockListsC(3, 256, 256, 128, 1000, 0, 0)   # neither 1 nor heads
    assert lib.bsa_attn_fwd_workspace_bytes(1, 24, ctypes.byref(ls)) == 0


def test_host_side_argument_checks(lib):
    from block_sparse_attention_radial_b200._lib import BlockListsC

    vp = ctypes.c_void_p
    fake = vp(1 << 20)   # never dereferenced: every call below fails its host checks
    ls = BlockListsC(1, 8, 8, 128, 10, 1 << 22, 1 << 23)
    call = lambda q, n, D, lst, out, ws=fake, wsb=1 << 12: lib.bsa_attn_fwd(
        q, fake, fake, 1, 1, n, D, 0.0, ctypes.byref(lst), out, None, ws, wsb, None)
    assert call(vp(0), 1024, 128, ls, vp(1 << 24)) == 1                       # null q
    assert call(fake, 1024, 96, ls, vp(1 << 24)) == 2                         # head_dim
    assert call(fake, 2000, 128, ls, vp(1 << 24)) == 1                        # n vs num_q_blocks
    bad_block = BlockListsC(1, 8, 8, 32, 10, 1 << 22, 1 << 23)
    assert call(fake, 256, 128, bad_block, vp(1 << 24)) == 2                  # block size
    assert call(vp((1 << 20) + 8), 1024, 128, ls, vp(1 << 24)) == 1           # misaligned q
    assert call(fake, 1024, 128, ls, vp(1 << 20)) == 1                        # out aliases q
    assert call(fake, 1024, 128, ls, vp(1 << 24), ws=vp(0)) == 1              # no workspace
    assert call(fake, 1024, 128, ls, vp(1 << 24), wsb=4) == 1                 # workspace too small
    two = BlockListsC(2, 8, 8, 128, 10, 1 << 22, 1 << 23)
    assert call(fake, 1024, 128, two, vp(1 << 24)) == 1                       # num_lists
    assert lib.bsa_attn_dense_masked_ref(fake, fake, fake, 1, 1, 1024, 64, 0.0, ctypes.byref(ls),
                                         vp(0), None, None) == 1              # null out


def test_mask_build_argument_checks(lib):
    vp = ctypes.c_void_p
    assert lib.bsa_radial_mask_build(0, 256, 64, vp(1 << 20), None, 0, None, None) == 1
    assert lib.bsa_radial_mask_build(4, 256, 64, vp(0), None, 0, None, None) == 1
    assert lib.bsa_radial_mask_build(4, 256, 32, vp(1 << 20), None, 0, None, None) == 2
    assert lib.bsa_radial_mask_build(1 << 16, 1 << 16, 128, vp(1 << 20), None, 0, None, None) == 1
    assert lib.bsa_joint_mask_build(4, 256, -1, 64, vp(1 << 20), None, 0, None, None) == 1
    assert lib.bsa_joint_mask_build(4, 256, 77, 32, vp(1 << 20), None, 0, None, None) == 2
    assert lib.bsa_joint_mask_build(1 << 15, 1 << 16, 1 << 30, 128, vp(1 << 20), None, 0, None,
                                    None) == 1
    assert lib.bsa_set_test_hooks(-1, 0) == 1
    assert lib.bsa_set_test_hooks(0, 0) == 0


def test_tile_pattern_build_argument_checks(lib):
    """Bad tile-pattern build arguments are rejected before any launch."""
    import ctypes

    from block_sparse_attention_radial_b200._lib import TilePatternC

    assert ctypes.sizeof(TilePatternC) == (5 + 2 * 16) * 4
    vp = ctypes.c_void_p
    pat, rp, cols = vp(1 << 20), vp(2 << 20), vp(3 << 20)
    f = lib.bsa_tile_pattern_lists_build
    assert f(0, 16, pat, None, 0, rp, None, 0, None, None) == 1          # no lists
    assert f(2, 0, pat, None, 0, rp, None, 0, None, None) == 1           # no rows
    assert f(2, 16, None, None, 0, rp, None, 0, None, None) == 1         # no patterns
    assert f(2, 16, pat, None, 0, None, None, 0, None, None) == 1        # no row_ptr
    assert f(2, 16, pat, None, 5, rp, None, 0, None, None) == 1          # columns missing
    assert f(2, 16, pat, cols, -1, rp, None, 0, None, None) == 1         # negative count
    assert f(2, 16, vp((1 << 20) + 2), None, 0, rp, None, 0, None, None) == 1  # misaligned
    assert f(2, 16, pat, None, 0, rp, vp(4 << 20), -1, None, None) == 1  # negative capacity
    assert f(2, 262145, pat, None, 0, rp, None, 0, None, None) == 2      # too many blocks
    assert f(1 << 14, 1 << 17, pat, None, 0, rp, None, 0, None, None) == 1  # rows >= 2^31 - 1


def test_backward_workspace_and_host_checks(lib):
    from block_sparse_attention_radial_b200._lib import BlockListsC

    ls = BlockListsC(1, 256, 256, 128, 1000, 0, 0)
    # lse2 + delta: 2 x 40 x 256 x 128 floats; 256 bytes of work counters;
    # offsets 257 ints; 1000 entries
    common = 2 * 40 * 256 * 128 * 4 + 256 + 1280 + 4096
    expect = common
    assert lib.bsa_attn_bwd_workspace_bytes(1, 40, 32760, ctypes.byref(ls)) == expect
    # the one-pass kernel: plus the entries' row positions, 4 dQ part
    # counters per query block, fp32 dQ rows of 128 per padded query row
    one = common + 4096 + 40 * 256 * 4 * 4 + 40 * 256 * 128 * 128 * 4
    assert lib.bsa_attn_bwd_one_pass_workspace_bytes(1, 40, 32760, ctypes.byref(ls)) == one
    assert lib.bsa_attn_bwd_workspace_bytes(1, 40, 32769, ctypes.byref(ls)) == 0  # nqb mismatch
    # block 64: masks of the transposed entries and the 128-row tile lists
    ls64 = BlockListsC(1, 512, 512, 64, 1000, 0, 0)
    expect64 = common + 1024 + 1280 + 4096 + 1024
    assert lib.bsa_attn_bwd_workspace_bytes(1, 40, 32760, ctypes.byref(ls64)) == expect64
    assert lib.bsa_attn_bwd_one_pass_workspace_bytes(1, 40, 32760, ctypes.byref(ls64)) == 0
    assert lib.bsa_attn_bwd_workspace_bytes(1, 40, 32769, ctypes.byref(ls64)) == 0  # nqb mismatch
    # bad arguments are rejected on the host, before any CUDA call
    p = ctypes.c_void_p(4096)
    ls = BlockListsC(1, 8, 8, 128, 10, 4096, 4096)
    args = [p, p, p, p, p, p, 1, 2, 1000, 128, ctypes.c_float(0.0), ctypes.byref(ls),
            ctypes.c_void_p(1 << 30), ctypes.c_void_p(1 << 31), ctypes.c_void_p(3 << 30),
            ctypes.c_void_p(1 << 33), 1 << 30, None]
    ovl = list(args)
    ovl[14] = p  # dv on top of the inputs
    assert lib.bsa_attn_bwd(*ovl) == 1
    ovl = list(args)
    ovl[13] = ctypes.c_void_p(1 << 30)  # dk on top of dq
    assert lib.bsa_attn_bwd(*ovl) == 1
    ovl = list(args)
    ovl[16] = 16  # workspace too small
    assert lib.bsa_attn_bwd(*ovl) == 1
    bad = list(args)
    bad[9] = 96
    assert lib.bsa_attn_bwd(*bad) == 2  # head_dim
    bad32 = BlockListsC(1, 32, 32, 32, 10, 4096, 4096)
    bad = list(args)
    bad[11] = ctypes.byref(bad32)
    assert lib.bsa_attn_bwd(*bad) == 2  # block 32 unsupported


def test_strided_forward_host_checks(lib):
    """bsa_attn_fwd_strided: layouts are validated on the host (every call
    below is rejected before any CUDA call)."""
    from block_sparse_attention_radial_b200._lib import BlockListsC, LayoutC

    vp, ref = ctypes.c_void_p, ctypes.byref
    B, H, n, D = 2, 4, 1024, 128
    C = H * D
    ls = BlockListsC(1, 8, 8, 128, 10, 1 << 22, 1 << 23)
    base = 1 << 30                            # fake [B, n, 3, H, D] projection buffer
    lqkv = LayoutC(n * 3 * C, D, 3 * C)
    lo = LayoutC(n * C, D, C)                 # [B, n, H, D] output

    def call(q=base, k=base + 2 * C, v=base + 4 * C, o=1 << 34, lq=lqkv, lk=lqkv, lv=lqkv,
             lo_=lo, hd=D, wsb=1 << 12):
        return lib.bsa_attn_fwd_strided(vp(q), lq and ref(lq), vp(k), ref(lk), vp(v), ref(lv),
                                        B, H, n, hd, 0.0, ref(ls), vp(o), ref(lo_), None,
                                        vp(1 << 36), wsb, None)

    assert call(lq=None) == 1                                   # no layout
    assert call(hd=96) == 2                                     # head_dim
    assert call(k=base + 2 * C + 8) == 1                        # misaligned k
    assert call(lk=LayoutC(n * 3 * C, D, 3 * C + 4)) == 1       # token stride not 16-byte
    assert call(lv=LayoutC(n * 3 * C, 0, 3 * C)) == 1           # zero head stride, heads > 1
    assert call(lo_=LayoutC(n * C, D, D)) == 1                  # output rows overlap each other
    assert call(o=base + 6 * C) == 1                            # output inside the q/k/v span
    assert call(wsb=4) == 1                                     # workspace too small


def test_module_workspace_and_host_checks(lib):
    from block_sparse_attention_radial_b200._lib import BlockListsC

    vp, ref = ctypes.c_void_p, ctypes.byref
    ls = BlockListsC(1, 256, 256, 128, 1000, 0, 0)
    # work order and counter (1 KiB + 256) + q/k/v [32760, 15360] + attention out
    # [32760, 5120] bf16 + lse [40, 32760] fp32 (the GEMMs need no scratch)
    expect = 1280 + 32760 * 15360 * 2 + 32760 * 5120 * 2 + 40 * 32760 * 4
    assert lib.bsa_attn_module_workspace_bytes(1, 32760, 40, 128, ref(ls)) == expect
    # backward: dA [32760, 5120] + dQKV [32760, 15360] bf16 + the attention
    # backward's workspace + 32 x 15360 fp32 partial sums
    attn_bwd = lib.bsa_attn_bwd_workspace_bytes(1, 40, 32760, ref(ls))
    expect_b = 32760 * 5120 * 2 + 32760 * 15360 * 2 + attn_bwd + 32 * 15360 * 4
    assert lib.bsa_attn_module_bwd_workspace_bytes(1, 32760, 40, 128, ref(ls)) == expect_b
    assert lib.bsa_attn_module_workspace_bytes(1, 32760, 40, 128, None) == 0
    B, n, H, D = 1, 1000, 2, 64
    small = BlockListsC(1, 8, 8, 128, 10, 1 << 22, 1 << 23)
    ws = lib.bsa_attn_module_workspace_bytes(B, n, H, D, ref(small))
    x, wq, wo, y, w = (vp(a << 30) for a in (1, 2, 3, 4, 8))

    def call(x=x, wq=wq, wo=wo, y=y, hd=D, wsb=ws):
        return lib.bsa_attn_module_fwd(x, wq, None, wo, None, B, n, H, hd, 0.0, ref(small), y, w,
                                       wsb, None)

    assert call(wo=vp(0)) == 1                                  # null weight
    assert call(hd=96) == 2                                     # head_dim
    assert call(wsb=ws - 1) == 1                                # workspace too small
    assert call(y=x) == 1                                       # y on top of x
    assert call(y=vp((8 << 30) + 4096)) == 1                    # y inside the workspace
    assert call(x=vp((1 << 30) + 8)) == 1                       # misaligned x


def test_strided_backward_host_checks(lib):
    """bsa_attn_bwd_strided rejects bad layouts on the host; the gradient
    slices of one [B, n, 3, H, D] buffer are accepted as disjoint (checked
    through the forward's identical rules for a gradient that would overlap)."""
    from block_sparse_attention_radial_b200._lib import BlockListsC, LayoutC

    vp, ref = ctypes.c_void_p, ctypes.byref
    B, H, n, D = 1, 4, 1024, 64
    C = H * D
    ls = BlockListsC(1, 8, 8, 128, 10, 1 << 22, 1 << 23)
    lqkv = LayoutC(n * 3 * C, D, 3 * C)
    ltok = LayoutC(n * C, D, C)
    qkv, attn, dattn, dqkv = 1 << 30, 1 << 32, 3 << 32, 1 << 34

    def call(dq=dqkv, dk=dqkv + 2 * C, dv=dqkv + 4 * C, ldq=lqkv, ldk=lqkv, ldv=lqkv, wsb=16):
        return lib.bsa_attn_bwd_strided(
            vp(qkv), ref(lqkv), vp(qkv + 2 * C), ref(lqkv), vp(qkv + 4 * C), ref(lqkv),
            vp(attn), ref(ltok), vp(dattn), ref(ltok), vp(5 << 32), B, H, n, D, 0.0, ref(ls),
            vp(dq), ref(ldq), vp(dk), ref(ldk), vp(dv), ref(ldv), vp(1 << 36), wsb, None)

    assert call() == 1                                   # workspace too small (layouts fine)
    assert call(dk=dqkv + 2 * C - 64) == 1               # dk's rows reach into dq's
    assert call(ldv=LayoutC(n * 3 * C, D, 3 * C + 8)) == 1  # different layout, shared span
    assert call(dq=qkv) == 1                              # dq on top of the inputs
    assert call(ldq=LayoutC(n * 3 * C, 8, 3 * C)) == 1   # dq's own rows overlap


def test_host_buffer_forward_host_checks(lib):
    """bsa_attn_fwd_host: workspace size formula and argument checks on the
    host (all rejected before any CUDA call)."""
    from block_sparse_attention_radial_b200._lib import BlockListsC

    vp, ref = ctypes.c_void_p, ctypes.byref
    ls = BlockListsC(1, 256, 256, 128, 1000, 0, 0)
    t = 1 * 40 * 32760 * 128 * 2
    # attention scratch (order + counter) + q, k, v, out (bf16) + lse (fp32)
    expect = 1280 + 4 * t + 40 * 32760 * 4
    assert lib.bsa_attn_fwd_host_workspace_bytes(1, 40, 32760, 128, ref(ls)) == expect
    small = BlockListsC(1, 8, 8, 128, 10, 1 << 22, 1 << 23)
    ws = lib.bsa_attn_fwd_host_workspace_bytes(1, 2, 1000, 64, ref(small))
    h = vp(1 << 20)

    def call(q=h, hd=64, w=vp(1 << 32), wsb=ws):
        return lib.bsa_attn_fwd_host(q, h, h, 1, 2, 1000, hd, 0.0, ref(small), h, None, w, wsb,
                                     None)

    assert call(q=vp(0)) == 1                       # null input
    assert call(hd=96) == 2                         # head_dim
    assert call(wsb=ws - 1) == 1                    # workspace too small
    assert call(w=vp((1 << 32) + 16)) == 1          # workspace not 256-byte aligned


def test_host_buffer_backward_host_checks(lib):
    """bsa_attn_bwd_host: workspace size formula and argument checks on the
    host (all rejected before any CUDA call)."""
    from block_sparse_attention_radial_b200._lib import BlockListsC

    vp, ref = ctypes.c_void_p, ctypes.byref
    ls = BlockListsC(1, 256, 256, 128, 1000, 0, 0)
    t = 1 * 40 * 32760 * 128 * 2
    # 40 heads in groups of at most 7: the backward's scratch for 7 heads
    # (lse2 and delta per 128-row tile row, work counters, transposed offsets
    # and entries), then q, k, v, out, dout, dq, dk, dv (bf16) and lse (fp32)
    scratch = 2 * 7 * 256 * 128 * 4 + 256 + 1280 + 4096
    expect = scratch + 8 * t + 40 * 32760 * 4
    assert lib.bsa_attn_bwd_host_workspace_bytes(1, 40, 32760, 128, ref(ls)) == expect
    assert lib.bsa_attn_bwd_host_workspace_bytes(1, 40, 0, 128, ref(ls)) == 0
    bad = BlockListsC(3, 256, 256, 128, 1000, 0, 0)      # 3 lists for 40 heads
    assert lib.bsa_attn_bwd_host_workspace_bytes(1, 40, 32760, 128, ref(bad)) == 0
    small = BlockListsC(2, 8, 8, 128, 10, 1 << 22, 1 << 23)
    ws = lib.bsa_attn_bwd_host_workspace_bytes(1, 2, 1000, 64, ref(small))
    assert ws > 0
    h = vp(1 << 20)

    def call(q=h, lse=h, dv=h, hd=64, w=vp(1 << 32), wsb=ws):
        return lib.bsa_attn_bwd_host(q, h, h, h, h, lse, 1, 2, 1000, hd, 0.0, ref(small), h, h, dv,
                                     w, wsb, None)

    assert call(q=vp(0)) == 1                       # null input
    assert call(lse=None) == 1                      # lse is required
    assert call(dv=None) == 1                       # null output
    assert call(hd=96) == 2                         # head_dim
    assert call(wsb=ws - 1) == 1                    # workspace too small
    assert call(w=vp((1 << 32) + 16)) == 1          # workspace not 256-byte aligned


def test_tile_pattern_packing():
    """Descriptors are laid out as bsa_tile_pattern[] (stripe columns in one
    shared array, each pattern's range recorded); malformed terms are refused
    on the host."""
    import pytest
    import torch

    import block_sparse_attention_radial_b200 as bsa

    pats = [{"bands": [(-2, 3), (7, 7)], "axial": (8, 1), "columns": [5, 1]}, {},
            {"columns": [9]}]
    raw, cols = bsa.pack_tile_patterns(pats, device="cpu")
    words = raw.view(torch.int32).view(3, 37)
    assert words[0, 0] == 2 and words[0, 1:3].tolist() == [-2, 7]
    assert words[0, 17:19].tolist() == [3, 7]
    assert words[0, 33:37].tolist() == [8, 1, 0, 2]
    assert words[1].tolist() == [0] * 35 + [2, 2]      # empty range at offset 2
    assert words[2, 35:37].tolist() == [2, 3]
    assert cols.tolist() == [5, 1, 9]
    with pytest.raises(ValueError):
        bsa.pack_tile_patterns([{"bands": [(0, 0)] * 17}], device="cpu")
    with pytest.raises(ValueError):
        bsa.pack_tile_patterns([{"axial": (0, 1)}], device="cpu")


def test_plain_c_caller(lib, tmp_path):
    """A C99 program compiled against include/bsa.h and linked to libbsa.so
    calls host-only entry points: the header is plain C and the symbols link
    without C++ name mangling."""
    import shutil
    import subprocess

    from block_sparse_attention_radial_b200 import _lib

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(r"""
#include <stdio.h>
#include "bsa.h"
int main(void) {
  bsa_block_lists l = {1, 256, 256, 128, 1000, (const int32_t *)0, (const int32_t *)0};
  bsa_tile_pattern p = {0};
  printf("%zu\n", bsa_attn_fwd_workspace_bytes(1, 40, &l));
  printf("%s\n", bsa_status_string(BSA_ERR_CAPACITY));
  printf("%d\n", bsa_tile_pattern_lists_build(0, 16, &p, 0, 0, 0, 0, 0, 0, 0));
  printf("%zu\n", sizeof(bsa_tile_pattern));
  return 0;
}
""")
    exe = tmp_path / "caller"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L" + libdir, "-l:libbsa.so",
                    "-Wl,-rpath," + libdir], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    assert out[0] == "1280"                      # 128 pair entries, aligned, + the work counter
    assert out[1] == lib.bsa_status_string(6).decode()
    assert out[2] == "1"                         # BSA_ERR_INVALID_ARG, found on the host
    assert out[3] == str(37 * 4)


def test_gemm_host_checks(lib):
    """bsa_gemm_bf16 rejects bad shapes, strides, alignment and overlapping
    output on the host, before any CUDA call."""
    vp = ctypes.c_void_p
    a, b, d, bias = (vp(x << 30) for x in (1, 2, 3, 4))

    def call(a=a, lda=256, amn=0, b=b, ldb=256, bmn=0, bias=None, d=d, ldd=512, m=100, n=512,
             k=256):
        return lib.bsa_gemm_bf16(a, lda, amn, b, ldb, bmn, bias, d, ldd, m, n, k, None)

    assert call(m=0) == 1 and call(n=0) == 1 and call(k=0) == 1
    assert call(n=500, ldd=504) == 1                 # n not a multiple of 8
    assert call(lda=252, k=250) == 1                 # lda not a multiple of 8
    assert call(lda=128) == 1                        # K-major A: lda < k
    assert call(amn=1, lda=96) == 1                  # MN-major A: lda < m
    assert call(ldb=128) == 1                        # B stored [n][k]: ldb < k
    assert call(bmn=1, ldb=256) == 1                 # B stored [k][n]: ldb < n
    assert call(ldd=256) == 1                        # ldd < n
    assert call(a=vp((1 << 30) + 8)) == 1            # misaligned A
    assert call(d=vp((3 << 30) + 2)) == 1            # misaligned D
    assert call(d=vp((1 << 30) + 1024)) == 1         # D inside A's span
    assert call(d=vp((2 << 30) + 4096)) == 1         # D inside B's span
    assert call(bias=vp((3 << 30) + 64)) == 1        # bias inside D's span
    assert call(a=None) == 1


def test_varlen_host_checks(lib):
    """bsa_attn_fwd_varlen and its list builder reject malformed per-item
    arguments on the host, before any CUDA call."""
    from block_sparse_attention_radial_b200._lib import BlockListsC, LayoutC

    vp, ref = ctypes.c_void_p, ctypes.byref
    H, D = 2, 128
    cu_ok = (ctypes.c_int32 * 4)(0, 300, 300, 700)        # nqb 3, 0, 4 at block 128
    lay = LayoutC(0, D, H * D)                            # packed [total, H, D]
    q, k, v, o, w = (vp(a << 30) for a in (1, 2, 3, 4, 8))

    def lists(nq=7, nk=4, block=128, L=1):
        return BlockListsC(L, nq, nk, block, 10, 1 << 22, 1 << 23)

    def call(ls=None, cu=cu_ok, items=3, wsb=1 << 20, out=o, hd=D):
        ls = lists() if ls is None else ls
        return lib.bsa_attn_fwd_varlen(q, ref(lay), k, ref(lay), v, ref(lay), items, cu, H, hd,
                                       0.0, ref(ls), out, ref(lay), None, w, wsb, None)

    assert lib.bsa_attn_fwd_varlen_workspace_bytes(3, cu_ok, H, ref(lists())) == 256 + 256
    # block 64: plus the items' tile lists (7 + 1 offsets, 10 entries, 10 masks)
    assert lib.bsa_attn_fwd_varlen_workspace_bytes(3, cu_ok, H, ref(lists(block=64))) == \
        256 + 256 + 256 + 256 + 256
    assert call(items=0) == 1 and call(items=65) == 1
    assert call(cu=(ctypes.c_int32 * 4)(1, 300, 300, 700)) == 1      # cu[0] != 0
    assert call(cu=(ctypes.c_int32 * 4)(0, 300, 200, 700)) == 1      # decreasing
    assert call(cu=(ctypes.c_int32 * 2)(0, 0), items=1) == 1          # no tokens at all
    assert call(ls=lists(nq=6)) == 1                                  # row count mismatch
    assert call(ls=lists(nk=7)) == 1                                  # widest item is 4
    assert call(ls=lists(block=64, nq=14, nk=7)) == 1                 # 12 blocks of 64, not 14
    assert call(ls=lists(block=32, nq=24, nk=13)) == 2                # block 32 unsupported
    assert call(ls=lists(L=3)) == 1                                   # num_lists not 1 or H
    assert call(hd=96) == 2
    assert call(wsb=256) == 1                                         # workspace too small
    assert call(out=vp((4 << 30) + 8)) == 1                           # misaligned out
    assert call(out=vp((1 << 30) + 4096)) == 1                        # out inside q's span
    # list builder: bad item geometry, too many items
    fr, tp, tx = ((ctypes.c_int32 * 2)(*x) for x in ((2, 0), (100, 100), (0, 0)))
    rp = vp(1 << 22)
    assert lib.bsa_joint_mask_build_varlen(2, fr, tp, tx, 128, rp, None, 0, None, None) == 1
    fr2 = (ctypes.c_int32 * 2)(2, 3)
    assert lib.bsa_joint_mask_build_varlen(65, fr2, tp, tx, 128, rp, None, 0, None, None) == 1
    assert lib.bsa_joint_mask_build_varlen(2, fr2, tp, tx, 96, rp, None, 0, None, None) == 2


def test_varlen_backward_host_checks(lib):
    """bsa_attn_bwd_varlen rejects malformed arguments on the host, before any
    CUDA call."""
    from block_sparse_attention_radial_b200._lib import BlockListsC, LayoutC

    vp, ref = ctypes.c_void_p, ctypes.byref
    H, D = 2, 128
    cu_ok = (ctypes.c_int32 * 4)(0, 300, 300, 700)        # nqb 3, 0, 4 at block 128
    lay = LayoutC(0, D, H * D)                            # packed [total, H, D]
    bufs = [vp(a << 30) for a in range(1, 9)]             # q k v out dout dq dk dv
    lse, w = vp(9 << 30), vp(10 << 30)

    def lists(nq=7, nk=4, block=128, L=1):
        return BlockListsC(L, nq, nk, block, 10, 1 << 22, 1 << 23)

    def call(ls=None, cu=cu_ok, items=3, wsb=1 << 24, hd=D, lse_=lse, dq=None):
        ls = lists() if ls is None else ls
        p = list(bufs)
        if dq is not None:
            p[5] = dq
        return lib.bsa_attn_bwd_varlen(p[0], ref(lay), p[1], ref(lay), p[2], ref(lay), p[3],
                                       ref(lay), p[4], ref(lay), lse_, items, cu, H, hd, 0.0,
                                       ref(ls), p[5], ref(lay), p[6], ref(lay), p[7], ref(lay), w,
                                       wsb, None)

    ws = lib.bsa_attn_bwd_varlen_workspace_bytes(3, cu_ok, H, ref(lists()))
    # every item's padded rows (7 blocks of 128, 2 heads): lse2 + delta for
    # 1792 rows each, counters, 7 + 1 column pointers, 10 entries, each part
    # 256-byte aligned
    assert ws == 7168 + 7168 + 256 + 256 + 256
    assert lib.bsa_attn_bwd_varlen_workspace_bytes(3, cu_ok, H, ref(lists(block=32))) == 0
    # block 64: plus the tile lists (7 + 1 offsets, 10 entries, 10 mask
    # bytes) and one mask byte per transposed entry
    assert lib.bsa_attn_bwd_varlen_workspace_bytes(3, cu_ok, H, ref(lists(block=64))) == \
        ws + 256 + 256 + 256 + 256
    assert call(items=0) == 1 and call(items=65) == 1
    assert call(cu=(ctypes.c_int32 * 4)(1, 300, 300, 700)) == 1      # cu[0] != 0
    assert call(cu=(ctypes.c_int32 * 4)(0, 300, 200, 700)) == 1      # decreasing
    assert call(ls=lists(nq=6)) == 1                                  # row count mismatch
    assert call(ls=lists(nk=5)) == 1                                  # widest item is 4
    assert call(ls=lists(block=64, nq=14, nk=7)) == 1                 # 12 blocks of 64, not 14
    assert call(ls=lists(block=32, nq=24, nk=13)) == 2                # block 32 unsupported
    assert call(ls=lists(L=3)) == 1                                   # num_lists not 1 or H
    assert call(hd=96) == 2
    assert call(lse_=None) == 1                                       # lse required
    assert call(lse_=vp((9 << 30) + 2)) == 1                          # misaligned lse
    assert call(wsb=ws - 1) == 1                                      # workspace too small
    assert call(dq=vp((6 << 30) + 8)) == 1                            # misaligned dq
    assert call(dq=vp((1 << 30) + 4096)) == 1                         # dq inside q's span
    assert call(dq=bufs[6]) == 1                                      # dq and dk the same


def test_generated_rows_host_checks(lib):
    """bsa_attn_fwd_patterns / bsa_attn_fwd_radial reject bad arguments on the
    host, before any CUDA call."""
    vp = ctypes.c_void_p
    B, H, n, D = 1, 4, 1000, 128
    q, k, v, o, pat, cols, w = (vp(a << 30) for a in (1, 2, 3, 4, 5, 6, 8))
    ws = lib.bsa_attn_fwd_patterns_workspace_bytes(2, 8)
    # row lengths (2*8+1 ints -> 256 B) + order and pair costs (2*4 ints -> 256 B
    # each) + counter
    assert ws == 256 + 256 + 256 + 256
    assert lib.bsa_attn_fwd_patterns_workspace_bytes(0, 8) == 0

    def pcall(L=H, p=pat, c=cols, nc=10, hp=None, wsb=1 << 20, hd=D, nn=n):
        return lib.bsa_attn_fwd_patterns(q, k, v, B, H, nn, hd, 0.0, L, p, c, nc, hp, o, None, w,
                                         wsb, None)

    assert pcall(L=0) == 1 and pcall(L=4097) == 1
    assert pcall(L=3) == 1                       # neither 1 nor heads, and no head map
    assert pcall(p=None) == 1
    assert pcall(c=None) == 1                    # columns missing while num_columns > 0
    assert pcall(nc=-1) == 1
    assert pcall(wsb=256) == 1
    assert pcall(hd=96) == 2
    assert pcall(nn=0) == 1

    def rcall(F=4, S=250, T=0, wsb=1 << 20):
        return lib.bsa_attn_fwd_radial(q, k, v, B, H, F, S, T, D, 0.0, o, None, w, wsb, None)

    assert rcall(F=0) == 1 and rcall(S=0) == 1 and rcall(T=-1) == 1
    assert rcall(S=9000) == 2                    # a frame wider than the generator's window
    assert rcall(wsb=256) == 1
    assert lib.bsa_attn_fwd_radial_workspace_bytes(4, 250, 0) > 0
    assert lib.bsa_attn_fwd_radial_workspace_bytes(0, 250, 0) == 0
